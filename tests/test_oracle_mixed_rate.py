"""Pins for the mixed-rate (fractional bits per channel) oracle, CPU only.

zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5 bits per channel",
title and paragraph 2, quote 3.5 and 2.5 bits per channel without a mechanism; the
oracle reads it as two coordinate groups at adjacent widths (oracle/mixed_rate.py).
Independent checks: hand-worked records, a stray bit at every unused position, the
integer-rate encoder (itself pinned) at m = 0 and m = d, exhaustive nearest codeword
over the whole mixed product codebook at d = 8, exact codeword round trips, the MSE mix
of the two integer-rate integrals against Monte Carlo, and unbiasedness of the logit
estimator over 10^4 rotations and sketches.
"""

import itertools
import math
import os

import numpy as np
import pytest

from oracle import codebook as cb
from oracle import mixed_rate as mr
from oracle import turboquant as tq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _haar(d, rng):
    a = rng.standard_normal((d, d))
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def _books(d, beta):
    return cb.fit_codebook(d, beta)[0], cb.fit_codebook(d, beta + 1)[0]


def _read_layout():
    cases = []
    with open(os.path.join(GOLDEN, "layout_records_mixed_rate.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, d, beta, m, qjl, codes, signs, words = (p.strip() for p in line.split("|"))
            cases.append((name, int(d), int(beta), int(m), bool(int(qjl)), [int(v) for v in codes.split()],
                          None if signs == "-" else [int(v) for v in signs.split()],
                          [int(w, 16) for w in words.split()]))
    return cases


@pytest.mark.parametrize("case", _read_layout(), ids=lambda c: c[0])
def test_layout_hand_worked(case):
    name, d, beta, m, qjl, codes, signs, words = case
    got = mr.pack(np.array([codes]), None if signs is None else np.array([signs]), d, beta, m, qjl)
    assert got.tolist() == [words]
    idx, sg = mr.unpack(np.array([words], dtype=np.uint32), d, beta, m, qjl)
    assert idx.tolist() == [codes]
    if qjl:
        assert sg.tolist() == [signs]


@pytest.mark.parametrize("d,beta,m,qjl", [(64, 1, 32, True), (128, 2, 64, True), (128, 3, 64, False),
                                          (200, 2, 96, True), (8, 1, 4, False)])
def test_pack_round_trip_and_every_stray_bit(d, beta, m, qjl):
    rng = np.random.default_rng(d + beta + m)
    idx = np.concatenate([rng.integers(0, 2 << beta, size=(16, m)), rng.integers(0, 1 << beta, size=(16, d - m))],
                         axis=1)
    sign = rng.integers(0, 2, size=(16, d)) if qjl else None
    rec = mr.pack(idx, sign, d, beta, m, qjl)
    assert rec.shape == (16, mr.record_words(d, beta, m, qjl))
    i2, s2 = mr.unpack(rec, d, beta, m, qjl)
    assert np.array_equal(i2, idx) and (not qjl or np.array_equal(s2, sign))
    assert mr.padding_is_zero(rec, d, beta, m, qjl)
    iw = mr.index_words(d, beta, m)
    used = np.zeros(rec.shape[1] * 32, dtype=bool)
    used[:(beta + 1) * m + beta * (d - m)] = True
    if qjl:
        used[iw * 32:iw * 32 + d] = True
    for pos in np.nonzero(~used)[0]:
        bad = rec[:1].copy()
        bad[0, pos // 32] |= np.uint32(1 << (pos % 32))
        assert not mr.padding_is_zero(bad, d, beta, m, qjl), pos


def test_record_sizes_d128():
    # keys at 2.5 / 3.5 bits per channel: 1.5 / 2.5 code bits + the sign bit; values at
    # 2.5 / 3.5: 2.5 / 3.5 code bits. Bytes of the records (norms apart).
    assert 4 * mr.record_words(128, 1, 64, True) == 128 * (1.5 + 1) / 8
    assert 4 * mr.record_words(128, 2, 64, True) == 128 * (2.5 + 1) / 8
    assert 4 * mr.record_words(128, 2, 64, False) == 128 * 2.5 / 8
    assert 4 * mr.record_words(128, 3, 64, False) == 128 * 3.5 / 8


@pytest.mark.parametrize("m_is_d", [False, True])
def test_limits_equal_the_integer_rate_encoder(m_is_d):
    # m = 0: every coordinate at beta bits; m = d: every coordinate at beta + 1 bits. Both
    # must reproduce the integer-rate oracle exactly (records, norms, logits, softmax.V).
    d, beta = 64, 2
    rng = np.random.default_rng(3 + m_is_d)
    Pi, S = _haar(d, rng), rng.standard_normal((d, d))
    c_lo, c_hi = _books(d, beta)
    m = d if m_is_d else 0
    c_int, b_int = (c_hi, beta + 1) if m_is_d else (c_lo, beta)
    x = rng.standard_normal((30, d))
    a = mr.quantize(x, Pi, c_lo, c_hi, m, S)
    b = tq.quantize(x, Pi, c_int, S)
    for key in ("norm", "idx", "rnorm", "sign"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(mr.pack(a["idx"], a["sign"], d, beta, m, True), tq.pack(b["idx"], b["sign"], d, b_int, True))
    q = rng.standard_normal((3, d))
    la = mr.logits(q, Pi, S, c_lo, c_hi, m, a["norm"], a["rnorm"], a["idx"], a["sign"])
    lb = tq.logits(q, Pi, S, c_int, b["norm"], b["rnorm"], b["idx"], b["sign"])
    assert np.allclose(la, lb, rtol=0, atol=1e-12)
    oa = mr.attend_v(la, 0.3, a["norm"], a["idx"], Pi, c_lo, c_hi, m)
    ob = tq.attend_v(lb, 0.3, b["norm"], b["idx"], Pi, c_int)
    assert np.allclose(oa, ob, rtol=0, atol=1e-12)


def test_mixed_product_codebook_brute_force_d8():
    # Exhaustive nearest codeword over all 4^4 x 2^4 = 4096 vectors of the mixed product
    # codebook (coordinates 0..3 at 2 bits, 4..7 at 1 bit) equals the encoder's decision.
    d, beta, m = 8, 1, 4
    rng = np.random.default_rng(5)
    Pi = _haar(d, rng)
    c_lo, c_hi = _books(d, beta)
    words = np.array(list(itertools.product(*([range(4)] * m + [range(2)] * (d - m)))))
    book = mr.centroids_per_coordinate(words, c_lo, c_hi, m)
    x = rng.standard_normal((40, d))
    enc = mr.quantize(x, Pi, c_lo, c_hi, m)
    y = (x / np.linalg.norm(x, axis=1, keepdims=True)) @ Pi.T
    for a in range(len(x)):
        assert np.array_equal(words[np.argmin(np.sum((book - y[a]) ** 2, axis=1))], enc["idx"][a])


def test_codeword_round_trip_is_exact():
    d, beta, m = 128, 2, 64
    rng = np.random.default_rng(7)
    Pi, S = _haar(d, rng), rng.standard_normal((d, d))
    c_lo, c_hi = _books(d, beta)
    for a in range(10):
        want = np.concatenate([rng.integers(0, 8, m), rng.integers(0, 4, d - m)])
        w = mr.centroids_per_coordinate(want, c_lo, c_hi, m)
        nw = np.linalg.norm(w)
        x = rng.uniform(0.5, 3.0) * (w @ Pi) / nw
        enc = mr.quantize(x[None, :], Pi, np.asarray(c_lo, np.float64) / nw, np.asarray(c_hi, np.float64) / nw, m, S)
        assert np.array_equal(enc["idx"][0], want)
        assert enc["rnorm"][0] < 1e-12
        q = rng.standard_normal((2, d))
        lg = mr.logits(q, Pi, S, np.asarray(c_lo) / nw, np.asarray(c_hi) / nw, m, enc["norm"], enc["rnorm"],
                       enc["idx"], enc["sign"])
        assert np.allclose(lg[:, 0], q @ x, rtol=0, atol=1e-10 * np.linalg.norm(x) * np.abs(q).sum())


@pytest.mark.parametrize("d,beta,m", [(128, 2, 64), (128, 1, 64), (128, 3, 32)])
def test_mse_is_the_coordinate_weighted_mix(d, beta, m):
    # Monte Carlo of the mixed MSE stage over 2 x 10^4 unit vectors (Haar rotation) against
    # (m/d) MSE_d(beta+1) + (1 - m/d) MSE_d(beta), each term the oracle's pinned integral.
    n = 20_000
    rng = np.random.default_rng(d + 10 * beta + m)
    Pi = _haar(d, rng)
    c_lo, c_hi = _books(d, beta)
    x = rng.standard_normal((n, d))
    enc = mr.quantize(x, Pi, c_lo, c_hi, m)
    u = x / enc["norm"][:, None]
    err = np.sum((u - mr.centroids_per_coordinate(enc["idx"], c_lo, c_hi, m) @ Pi) ** 2, axis=1)
    want = mr.mse_mix(d, m, cb.mse_per_vector(d, c_hi), cb.mse_per_vector(d, c_lo))
    assert abs(err.mean() - want) < 4 * err.std() / math.sqrt(n), (err.mean(), want)
    # and it lies strictly between the two integer rates
    assert cb.mse_per_vector(d, c_hi) < want < cb.mse_per_vector(d, c_lo)


def test_estimator_unbiased_over_sketches_and_rotations():
    # keys at 2.5 bits per channel (1.5 code bits + QJL): E over (Pi, S) of the estimate is <q, k>
    d, beta, m, n_draw = 64, 1, 32, 10_000
    rng = np.random.default_rng(2025)
    k = rng.standard_normal(d)
    q = k + 0.7 * rng.standard_normal(d)
    c_lo, c_hi = _books(d, beta)
    est = np.empty(n_draw)
    for i in range(n_draw):
        Pi, S = _haar(d, rng), rng.standard_normal((d, d))
        enc = mr.quantize(k[None, :], Pi, c_lo, c_hi, m, S)
        est[i] = mr.logits(q[None, :], Pi, S, c_lo, c_hi, m, enc["norm"], enc["rnorm"], enc["idx"], enc["sign"])[0, 0]
    assert abs(est.mean() - q @ k) < 4 * est.std() / math.sqrt(n_draw)
