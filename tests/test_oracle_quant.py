"""Pins for the oracle's encoder, record layout, logit estimator and softmax.V (CPU only).

Independent checks: hand-worked records, brute force over the full product
codebook at d = 8, the identity rotation (textbook nearest-centroid scalar
quantization), exact round trips on codewords, the zero vector, unbiasedness
of the estimator over 10^4 random sketches and rotations, the closed-form bias
of the MSE-only estimator, and one-hot / uniform softmax limits.
"""

import itertools
import math
import os

import numpy as np
import pytest

from oracle import codebook as cb
from oracle import turboquant as tq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _haar(d, rng):
    a = rng.standard_normal((d, d))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def _read_layout():
    cases = []
    with open(os.path.join(GOLDEN, "layout_records.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, d, bits, qjl, codes, signs, words = (p.strip() for p in line.split("|"))
            cases.append((name, int(d), int(bits), bool(int(qjl)),
                          [int(v) for v in codes.split()],
                          None if signs == "-" else [int(v) for v in signs.split()],
                          [int(w, 16) for w in words.split()]))
    return cases


@pytest.mark.parametrize("case", _read_layout(), ids=lambda c: c[0])
def test_layout_hand_worked(case):
    name, d, bits, qjl, codes, signs, words = case
    got = tq.pack(np.array([codes]), None if signs is None else np.array([signs]), d, bits, qjl)
    assert got.tolist() == [words]
    idx, sg = tq.unpack(np.array([words], dtype=np.uint32), d, bits, qjl)
    assert idx.tolist() == [codes]
    if qjl:
        assert sg.tolist() == [signs]


@pytest.mark.parametrize("d,bits,qjl", [(8, 1, True), (128, 2, True), (128, 3, True), (200, 3, True),
                                        (200, 4, False), (128, 4, False), (8, 3, False)])
def test_pack_roundtrip_and_padding(d, bits, qjl):
    rng = np.random.default_rng(d * 10 + bits)
    idx = rng.integers(0, 1 << bits, size=(64, d))
    sign = rng.integers(0, 2, size=(64, d)) if qjl else None
    rec = tq.pack(idx, sign, d, bits, qjl)
    assert rec.shape == (64, tq.record_words(d, bits, qjl))
    i2, s2 = tq.unpack(rec, d, bits, qjl)
    assert np.array_equal(i2, idx)
    if qjl:
        assert np.array_equal(s2, sign)
    assert tq.padding_is_zero(rec, d, bits, qjl)


def test_record_sizes_d128():
    # bytes per key at b = 2/3/4 total bits (index bits = b-1, plus the sign bit),
    # and per value at b index bits: the planes only (norms are stored apart)
    assert [4 * tq.record_words(128, b - 1, True) for b in (2, 3, 4)] == [32, 48, 64]
    assert [4 * tq.record_words(128, b, False) for b in (2, 3, 4)] == [32, 48, 64]


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_identity_rotation_is_nearest_centroid(bits):
    d = 64
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((300, d))
    c32, _ = cb.fit_codebook(d, bits)
    enc = tq.quantize(x, np.eye(d), c32)
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    c = c32.astype(np.float64)
    brute = np.argmin(np.abs(u[:, :, None] - c[None, None, :]), axis=2)
    assert np.array_equal(enc["idx"], brute)


def test_product_codebook_brute_force_d8():
    # Exhaustive nearest codeword over all 4^8 = 65536 vectors of the product
    # codebook equals the per-coordinate decision of the encoder.
    d, bits = 8, 2
    rng = np.random.default_rng(5)
    Pi = _haar(d, rng)
    c32, _ = cb.fit_codebook(d, bits)
    c = c32.astype(np.float64)
    words = np.array(list(itertools.product(range(4), repeat=d)))
    book = c[words]
    x = rng.standard_normal((40, d))
    enc = tq.quantize(x, Pi, c32)
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    y = u @ Pi.T
    for a in range(len(x)):
        best = np.argmin(np.sum((book - y[a]) ** 2, axis=1))
        assert np.array_equal(words[best], enc["idx"][a])


def test_codeword_round_trip_is_exact():
    # Take a codeword w = c[idx*] and x = n Pi^T w/||w||. Then y = Pi u = w/||w||
    # lies exactly on the codebook scaled by 1/||w||, so the encoder must return
    # idx*, a zero residual, and an estimate equal to <q, x> (the QJL term
    # vanishes with rho = 0).
    d, bits = 128, 2
    rng = np.random.default_rng(7)
    Pi = _haar(d, rng)
    S = rng.standard_normal((d, d))
    c = cb.fit_codebook(d, bits)[0].astype(np.float64)
    want = rng.integers(0, 4, size=(20, d))
    n = rng.uniform(0.5, 3.0, size=20)
    for a in range(20):
        w = c[want[a]]
        x = n[a] * (w @ Pi) / np.linalg.norm(w)
        scaled = c / np.linalg.norm(w)
        enc = tq.quantize(x[None, :], Pi, scaled, S)
        assert np.array_equal(enc["idx"][0], want[a])
        assert enc["rnorm"][0] < 1e-12
        q = rng.standard_normal((3, d))
        lg = tq.logits(q, Pi, S, scaled, enc["norm"], enc["rnorm"], enc["idx"], enc["sign"])
        tol = 1e-10 * np.linalg.norm(x) * np.linalg.norm(q, axis=1).max()
        assert np.allclose(lg[:, 0], q @ x, rtol=0, atol=tol)


def test_zero_vector():
    d, bits = 32, 2
    rng = np.random.default_rng(3)
    Pi, S = _haar(d, rng), rng.standard_normal((d, d))
    c32, t = cb.fit_codebook(d, bits)
    enc = tq.quantize(np.zeros((1, d)), Pi, c32, S)
    assert enc["norm"][0] == 0 and enc["rnorm"][0] == 0
    assert np.all(enc["sign"] == 1)
    assert np.all(enc["idx"] == np.sum(t < 0))
    lg = tq.logits(rng.standard_normal((2, d)), Pi, S, c32, enc["norm"], enc["rnorm"], enc["idx"], enc["sign"])
    assert np.all(lg == 0)


def test_ties_go_to_lower_cell():
    # d = 1, Pi = [1], x = [1]: y = 1. With centroids {-1, 1} the threshold is 0 and
    # y is above it; with centroids {0, 2} the threshold is exactly 1 = y, which
    # the reading sends to the lower cell.
    one = np.array([[1.0]])
    assert tq.quantize(one, np.eye(1), np.array([-1.0, 1.0], dtype=np.float32))["idx"][0, 0] == 1
    assert tq.quantize(one, np.eye(1), np.array([0.0, 2.0], dtype=np.float32))["idx"][0, 0] == 0
    # sign of an exactly zero sketch coordinate is +1 (bit 1): S = 0 gives s = 0
    enc = tq.quantize(np.array([[3.0, 4.0]]), np.eye(2), np.array([-0.5, 0.5], dtype=np.float32), np.zeros((2, 2)))
    assert enc["sign"].tolist() == [[1, 1]]


def test_estimator_unbiased_over_sketches_and_rotations():
    # E over (Pi, S) of the estimator equals <q, k>; 10^4 independent draws.
    d, bits, n_draw = 128, 2, 10_000
    rng = np.random.default_rng(2024)
    k = rng.standard_normal(d)
    q = k + 0.7 * rng.standard_normal(d)
    truth = float(q @ k)
    c32, _ = cb.fit_codebook(d, bits)
    est = np.empty(n_draw)
    mse_only = np.empty(n_draw)
    for i in range(n_draw):
        Pi = _haar(d, rng)
        S = rng.standard_normal((d, d))
        enc = tq.quantize(k[None, :], Pi, c32, S)
        est[i] = tq.logits(q[None, :], Pi, S, c32, enc["norm"], enc["rnorm"], enc["idx"], enc["sign"])[0, 0]
        mse_only[i] = tq.logits_mse_only(q[None, :], Pi, c32, enc["norm"], enc["idx"])[0, 0]
    se = est.std() / math.sqrt(n_draw)
    assert abs(est.mean() - truth) < 4 * se, (est.mean(), truth, se)
    # without the QJL term the estimate is biased (shrunk)
    se_m = mse_only.std() / math.sqrt(n_draw)
    assert abs(mse_only.mean() - truth) > 10 * se_m


def test_one_bit_mse_only_bias_closed_form():
    # 1 bit: E_Pi[Pi^T c[idx(Pi u)]] = d c1^2 u, so the MSE-only estimate has mean
    # d c1^2 <q, k> (c1 = E|y|); the QJL term restores <q, k>.
    d, n_draw = 64, 6000
    rng = np.random.default_rng(11)
    k = rng.standard_normal(d)
    q = 0.5 * k + rng.standard_normal(d)
    truth = float(q @ k)
    c1 = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    c32 = np.array([-c1, c1], dtype=np.float32)
    vals = np.empty(n_draw)
    full = np.empty(n_draw)
    for i in range(n_draw):
        Pi = _haar(d, rng)
        S = rng.standard_normal((d, d))
        enc = tq.quantize(k[None, :], Pi, c32, S)
        vals[i] = tq.logits_mse_only(q[None, :], Pi, c32, enc["norm"], enc["idx"])[0, 0]
        full[i] = tq.logits(q[None, :], Pi, S, c32, enc["norm"], enc["rnorm"], enc["idx"], enc["sign"])[0, 0]
    want = d * float(c32[1]) ** 2 * truth
    assert abs(vals.mean() - want) < 4 * vals.std() / math.sqrt(n_draw)
    assert abs(full.mean() - truth) < 4 * full.std() / math.sqrt(n_draw)


def test_qjl_term_unbiased_and_variance_bound_for_fixed_rotation():
    # With Pi fixed, averaging over S alone: E[<Sq, sign(Sr)>] = d sqrt(2/pi) <q, r>/||r||,
    # and Var of the scaled term  sqrt(pi/2)/d * rho <Sq, sign(Sr)>  is at most (pi/2)/d ||q||^2 rho^2.
    d, bits, n_draw = 128, 2, 10_000
    rng = np.random.default_rng(77)
    Pi = _haar(d, rng)
    c32, _ = cb.fit_codebook(d, bits)
    k = rng.standard_normal(d)
    q = rng.standard_normal(d) + 0.3 * k
    enc0 = tq.quantize(k[None, :], Pi, c32, np.eye(d))
    r, rho, n = enc0["r"][0], enc0["rnorm"][0], enc0["norm"][0]
    terms = np.empty(n_draw)
    for i in range(n_draw):
        S = rng.standard_normal((d, d))
        terms[i] = math.sqrt(math.pi / 2) / d * rho * float((S @ q) @ np.where(S @ r >= 0, 1.0, -1.0))
    want = float(q @ r)
    assert abs(terms.mean() - want) < 4 * terms.std() / math.sqrt(n_draw)
    assert terms.var() <= (math.pi / 2) / d * float(q @ q) * rho ** 2 * 1.05
    del n


def test_softmax_limits():
    d, bits = 32, 3
    rng = np.random.default_rng(8)
    Pi = _haar(d, rng)
    c32, _ = cb.fit_codebook(d, bits)
    v = rng.standard_normal((50, d))
    enc = tq.quantize(v, Pi, c32)
    recon = tq.dequantize_mse(enc["norm"], enc["idx"], Pi, c32)
    lg = rng.standard_normal((3, 50))
    lg[0, 17] += 1e4
    out = tq.attend_v(lg, 1.0, enc["norm"], enc["idx"], Pi, c32)
    assert np.allclose(out[0], recon[17], atol=1e-12)
    flat = np.zeros((1, 50))
    out = tq.attend_v(flat, 0.3, enc["norm"], enc["idx"], Pi, c32)
    assert np.allclose(out[0], recon.mean(axis=0), atol=1e-12)
    assert tq.attend_v(np.zeros((2, 0)), 1.0, enc["norm"][:0], enc["idx"][:0], Pi, c32).tolist() == [[0.0] * d] * 2


def test_mse_only_reconstruction_error_matches_integral():
    # empirical per-vector MSE of the value path against the oracle's integral
    d, bits, n = 128, 3, 20_000
    rng = np.random.default_rng(21)
    Pi = _haar(d, rng)
    c32, _ = cb.fit_codebook(d, bits)
    x = rng.standard_normal((n, d))
    enc = tq.quantize(x, Pi, c32)
    u = x / enc["norm"][:, None]
    err = np.sum((u - tq.dequantize_mse(np.ones(n), enc["idx"], Pi, c32)) ** 2, axis=1)
    want = cb.mse_per_vector(d, c32.astype(np.float64))
    assert abs(err.mean() - want) < 4 * err.std() / math.sqrt(n)


def test_topk_orders_ties_by_index():
    s = np.array([[0.5, 0.9, 0.5, 0.9, 0.1]])
    assert tq.topk(s, 3).tolist() == [[1, 3, 0]]


def _used_bit_mask(d, bits, qjl):
    """Which bits of a record carry data, worked out from the layout's definition alone:
    the index stream's first bits*d bits, then (keys) the sign field's first d bits."""
    iw = (bits * d + 31) // 32
    sw = (d + 31) // 32 if qjl else 0
    used = np.zeros((iw + sw) * 32, dtype=bool)
    used[:bits * d] = True
    if qjl:
        used[iw * 32:iw * 32 + d] = True
    return used


@pytest.mark.parametrize("d,bits,qjl", [(8, 1, True), (8, 3, True), (200, 1, True), (200, 3, True),
                                        (8, 3, False), (200, 3, False)])
def test_padding_check_rejects_every_single_stray_bit(d, bits, qjl):
    # zubnet.ai news, paragraph 2: a record holds the indices and the sign bits and nothing
    # else, so every other bit must be 0. Plant one stray bit at each unused position (in
    # the index field's last word and in the sign field's last word) of an otherwise valid
    # record: the check must fail every time, and pass on a record whose used bits are all 1.
    rng = np.random.default_rng(d + 10 * bits + int(qjl))
    idx = rng.integers(0, 1 << bits, size=(1, d))
    sign = rng.integers(0, 2, size=(1, d)) if qjl else None
    rec = tq.pack(idx, sign, d, bits, qjl)
    assert tq.padding_is_zero(rec, d, bits, qjl)
    used = _used_bit_mask(d, bits, qjl)
    pad = np.nonzero(~used)[0]
    assert len(pad) > 0
    for pos in pad:
        bad = rec.copy()
        bad[0, pos // 32] |= np.uint32(1 << (pos % 32))
        assert not tq.padding_is_zero(bad, d, bits, qjl), f"stray bit {pos} not caught"
        # also as the second row of a batch (the check covers every row)
        assert not tq.padding_is_zero(np.concatenate([rec, bad]), d, bits, qjl)
    full = np.zeros_like(rec)
    for pos in np.nonzero(used)[0]:
        full[0, pos // 32] |= np.uint32(1 << (pos % 32))
    assert tq.padding_is_zero(full, d, bits, qjl)
