"""The parity checker itself (CPU only): it must accept what the tolerances excuse and
reject planted mistakes.

Records that stand in for the GPU's output are built by the oracle on the CPU and then
altered by hand: a code moved one cell across the threshold it lies next to (excused), a
code moved two cells, a code moved one cell across the other threshold of its cell, a
stray padding bit, a sign flipped far from zero. The tolerances are the method's parity
bounds: codes bit-exact except within 1e-5 of a threshold, norms to 1e-5.
"""

import numpy as np
import pytest

from oracle import codebook as ocb
from oracle import turboquant as otq
from tests import _parity as par


def _haar(d, rng):
    a = rng.standard_normal((d, d))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def _vector_near_threshold(d, Pi, t_j, delta, rng):
    """x whose rotated unit vector has y_0 = t_j + delta exactly (up to float64 rounding)."""
    y = rng.standard_normal(d)
    y[0] = 0.0
    y *= np.sqrt(1.0 - (t_j + delta) ** 2) / np.linalg.norm(y)
    y[0] = t_j + delta
    return 2.5 * (y @ Pi)          # x = n Pi^T y with n = 2.5


def _gpu_like(x, Pi, S, c, d, bits, qjl, codes=None):
    """Records as a correct implementation would write them for the given codes (the
    oracle's own codes by default): norms, and for keys rho and signs of the residual
    of those codes."""
    enc = otq.quantize(x, Pi, c, S if qjl else None)
    gi = enc["idx"] if codes is None else codes
    if not qjl:
        return otq.pack(gi, None, d, bits, False), enc["norm"], None
    u = x / enc["norm"][:, None]
    r = u - np.asarray(c, dtype=np.float64)[gi] @ Pi
    s = r @ np.asarray(S, dtype=np.float64).T
    return (otq.pack(gi, (s >= 0).astype(np.int64), d, bits, True), enc["norm"],
            np.sqrt(np.sum(r * r, axis=1)))


@pytest.fixture(scope="module")
def setup():
    d, bits = 64, 2
    rng = np.random.default_rng(41)
    Pi = _haar(d, rng)
    S = rng.standard_normal((d, d))
    c = ocb.fit_codebook(d, bits)[0]
    t = otq.thresholds_of(c)
    return d, bits, Pi, S, c, t, rng


@pytest.mark.parametrize("qjl", [False, True])
def test_one_cell_move_across_nearby_threshold_is_excused(setup, qjl):
    d, bits, Pi, S, c, t, rng = setup
    x = np.stack([_vector_near_threshold(d, Pi, t[1], 4e-6, rng) for _ in range(3)])
    codes = otq.quantize(x, Pi, c)["idx"].copy()
    assert np.all(codes[:, 0] == 2)            # just above t_1: cell 2
    codes[:, 0] = 1                            # moved across t_1 into cell 1
    rec, n, rho = _gpu_like(x, Pi, S, c, d, bits, qjl, codes)
    # the excused flips of this small case are above the 1e-4 rate budget, so relax it here only
    old = par.FLIP_RATE_MAX
    par.FLIP_RATE_MAX = 1.0
    try:
        out = par.check_encoding(x, rec, n, rho, Pi, S, c, d, bits, qjl)
    finally:
        par.FLIP_RATE_MAX = old
    assert out["index_flips"] == 3


@pytest.mark.parametrize("new_code", [0, 3])
def test_two_cell_move_or_wrong_threshold_is_rejected(setup, new_code):
    # y_0 sits 4e-6 above t_1 (cell 2). Cell 0 is two cells away; cell 3 is one cell away
    # but across t_2, which is far from y_0. Both must fail.
    d, bits, Pi, S, c, t, rng = setup
    x = _vector_near_threshold(d, Pi, t[1], 4e-6, rng)[None, :]
    codes = otq.quantize(x, Pi, c)["idx"].copy()
    codes[0, 0] = new_code
    rec, n, rho = _gpu_like(x, Pi, S, c, d, bits, True, codes)
    with pytest.raises(AssertionError, match="code mismatches"):
        par.check_encoding(x, rec, n, rho, Pi, S, c, d, bits, True)


def test_move_far_from_any_threshold_is_rejected(setup):
    d, bits, Pi, S, c, t, rng = setup
    x = _vector_near_threshold(d, Pi, t[1], 3e-3, rng)[None, :]
    codes = otq.quantize(x, Pi, c)["idx"].copy()
    codes[0, 0] = 1
    rec, n, rho = _gpu_like(x, Pi, S, c, d, bits, False, codes)
    with pytest.raises(AssertionError, match="code mismatches"):
        par.check_encoding(x, rec, n, rho, Pi, S, c, d, bits, False)


def test_exact_records_pass_and_stray_bits_or_signs_fail(setup):
    d, bits, Pi, S, c, t, rng = setup
    x = rng.standard_normal((40, d))
    rec, n, rho = _gpu_like(x, Pi, S, c, d, bits, True)
    out = par.check_encoding(x, rec, n, rho, Pi, S, c, d, bits, True)
    assert out["index_flips"] == 0 and out["sign_flips"] == 0
    # a stray bit in the unused high bits of the sign field's last word (d = 64: none in
    # the index field, 2 * 64 = 128 bits fill 4 words) -> use d = 40 for that
    d2 = 40
    Pi2, S2 = _haar(d2, rng), rng.standard_normal((d2, d2))
    c2 = ocb.fit_codebook(d2, bits)[0]
    x2 = rng.standard_normal((5, d2))
    rec2, n2, rho2 = _gpu_like(x2, Pi2, S2, c2, d2, bits, True)
    for word, bit in ((2, 31), (4, 9)):         # index field word 2 holds bits 64..95 (80 used); sign word 1
        bad = rec2.copy()
        bad[3, word] |= np.uint32(1 << bit)
        with pytest.raises(AssertionError, match="padding"):
            par.check_encoding(x2, bad, n2, rho2, Pi2, S2, c2, d2, bits, True)
    # a sign bit flipped where |s_i| is far from zero
    enc = otq.quantize(x, Pi, c, S)
    a, i = np.unravel_index(np.argmax(np.abs(enc["s"])), enc["s"].shape)
    bad = rec.copy()
    iw = otq.index_words(d, bits)
    bad[a, iw + i // 32] ^= np.uint32(1 << (i % 32))
    with pytest.raises(AssertionError, match="sign mismatches"):
        par.check_encoding(x, bad, n, rho, Pi, S, c, d, bits, True)
    # a norm off by 1e-4 relative
    n_bad = n.copy()
    n_bad[7] *= 1 + 1e-4
    with pytest.raises(AssertionError, match="norm mismatch"):
        par.check_encoding(x, rec, n_bad, rho, Pi, S, c, d, bits, True)
