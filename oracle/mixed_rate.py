"""Fractional bit-rates: TurboQuant with two coordinate groups at adjacent widths (float64).

Test infrastructure (see ``oracle/__init__``).

Pages: zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5 bits
per channel" (es/pt/fr), title and paragraph 2: the cache is stored at 3.5 bits
per channel with no measurable quality loss, and 2.5 bits per channel loses a
little. The pages do not say how a fractional number of bits per channel is
reached with a per-coordinate scalar quantizer.

Reading taken here (the plainest one the rest of the pages supports): "b bits per
channel" is the average over the d coordinates
of the bits stored per coordinate. After the random rotation every coordinate of
y = Pi u has the same law f_d, so which coordinates get the extra bit does not
matter for the error; the first m rotated coordinates get beta + 1 code bits and
the other d - m get beta, each group quantized with the Lloyd-Max codebook of
f_d at its own width (the same fit as the integer rates). Then

    average code bits per coordinate = beta + m / d,

keys add their one QJL sign bit per coordinate (keys at 3.5 bits: beta = 2,
m = d/2 plus the sign; values at 3.5 bits: beta = 3, m = d/2), and since the
coordinate-wise errors add up, the per-vector MSE of the MSE stage is the
coordinate-weighted mix

    MSE = (m/d) MSE_d(beta + 1) + (1 - m/d) MSE_d(beta).

The residual, its norm, the QJL sketch and the estimator are those of the
integer-rate method with yhat_i = c_hi[idx_i] for i < m and c_lo[idx_i] otherwise.

Record layout (our specification, an extension of the integer-rate one): the
code of coordinate i < m sits at stream bits [(beta+1) i, (beta+1) i + beta + 1),
the code of coordinate i >= m at stream bits [(beta+1) m + beta (i - m), ... + beta),
least significant bit first; index_words = ceil(((beta+1) m + beta (d - m)) / 32);
the sign field (keys) follows exactly as at integer rates. Unused bits are 0.
"""

from __future__ import annotations

import math

import numpy as np


def index_bits(d: int, beta: int, m: int) -> int:
    """Code bits of one record: m coordinates at beta + 1 bits, d - m at beta bits."""
    return (beta + 1) * m + beta * (d - m)


def index_words(d: int, beta: int, m: int) -> int:
    return (index_bits(d, beta, m) + 31) // 32


def record_words(d: int, beta: int, m: int, qjl: bool) -> int:
    return index_words(d, beta, m) + ((d + 31) // 32 if qjl else 0)


def code_positions(d: int, beta: int, m: int):
    """(first stream bit, width) of every coordinate's code."""
    start = np.empty(d, dtype=np.int64)
    width = np.empty(d, dtype=np.int64)
    i = np.arange(d)
    hi = i < m
    start[hi] = (beta + 1) * i[hi]
    width[hi] = beta + 1
    start[~hi] = (beta + 1) * m + beta * (i[~hi] - m)
    width[~hi] = beta
    return start, width


def pack(idx, sign, d: int, beta: int, m: int, qjl: bool) -> np.ndarray:
    """Rows of codes (and sign bits) -> uint32 records, bit by bit per the layout above."""
    idx = np.asarray(idx, dtype=np.int64).reshape(-1, d)
    n = idx.shape[0]
    iw = index_words(d, beta, m)
    start, width = code_positions(d, beta, m)
    stream = np.zeros((n, iw * 32), dtype=np.uint64)
    for i in range(d):
        for b in range(width[i]):
            stream[:, start[i] + b] = (idx[:, i] >> b) & 1
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    words = (stream.reshape(n, iw, 32) * weights).sum(axis=2)
    if qjl:
        sw = (d + 31) // 32
        sbits = np.zeros((n, sw * 32), dtype=np.uint64)
        sbits[:, :d] = np.asarray(sign, dtype=np.uint64).reshape(-1, d)
        words = np.concatenate([words, (sbits.reshape(n, sw, 32) * weights).sum(axis=2)], axis=1)
    return words.astype(np.uint32)


def unpack(records, d: int, beta: int, m: int, qjl: bool):
    """uint32 records -> (codes [n, d] int64, sign bits [n, d] or None)."""
    rec = np.asarray(records, dtype=np.uint64).reshape(-1, record_words(d, beta, m, qjl))
    n = rec.shape[0]
    iw = index_words(d, beta, m)
    shifts = np.arange(32, dtype=np.uint64)
    stream = ((rec[:, :iw, None] >> shifts) & np.uint64(1)).reshape(n, iw * 32).astype(np.int64)
    start, width = code_positions(d, beta, m)
    idx = np.zeros((n, d), dtype=np.int64)
    for i in range(d):
        for b in range(width[i]):
            idx[:, i] |= stream[:, start[i] + b] << b
    sign = None
    if qjl:
        sbits = ((rec[:, iw:, None] >> shifts) & np.uint64(1)).reshape(n, -1)
        sign = sbits[:, :d].astype(np.int64)
    return idx, sign


def padding_is_zero(records, d: int, beta: int, m: int, qjl: bool) -> bool:
    """True when every bit outside the codes and the signs is 0."""
    rec = np.asarray(records, dtype=np.uint64).reshape(-1, record_words(d, beta, m, qjl))
    iw = index_words(d, beta, m)
    used = np.zeros(rec.shape[1] * 32, dtype=bool)
    used[:index_bits(d, beta, m)] = True
    if qjl:
        used[iw * 32:iw * 32 + d] = True
    shifts = np.arange(32, dtype=np.uint64)
    bits = ((rec[:, :, None] >> shifts) & np.uint64(1)).reshape(rec.shape[0], -1)
    return bool(np.all(bits[:, ~used] == 0))


def centroids_per_coordinate(idx, c_lo, c_hi, m: int) -> np.ndarray:
    """yhat_i = c_hi[idx_i] for i < m, c_lo[idx_i] otherwise."""
    idx = np.asarray(idx)
    out = np.empty(idx.shape, dtype=np.float64)
    out[..., :m] = np.asarray(c_hi, dtype=np.float64)[idx[..., :m]]
    out[..., m:] = np.asarray(c_lo, dtype=np.float64)[idx[..., m:]]
    return out


def quantize(x, Pi, c_lo, c_hi, m: int, S=None):
    """Encode rows of x at the mixed rate. Same steps as the integer-rate encoder (norm,
    rotation, per-coordinate nearest cell, residual, sign sketch), with coordinate i < m
    quantized against c_hi and the rest against c_lo. Ties go to the lower cell; a zero
    vector has u = 0, r = 0, rho = 0 and all sign bits 1."""
    x = np.asarray(x, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    t_lo = (np.asarray(c_lo, np.float64)[:-1] + np.asarray(c_lo, np.float64)[1:]) / 2.0
    t_hi = (np.asarray(c_hi, np.float64)[:-1] + np.asarray(c_hi, np.float64)[1:]) / 2.0
    norm = np.sqrt(np.sum(x * x, axis=1))
    u = np.zeros_like(x)
    nz = norm > 0
    u[nz] = x[nz] / norm[nz, None]
    y = u @ Pi.T
    idx = np.empty(y.shape, dtype=np.int64)
    idx[:, :m] = np.searchsorted(t_hi, y[:, :m], side="left")
    idx[:, m:] = np.searchsorted(t_lo, y[:, m:], side="left")
    out = {"norm": norm, "idx": idx, "y": y}
    if S is not None:
        yhat = centroids_per_coordinate(idx, c_lo, c_hi, m)
        r = u - yhat @ Pi
        r[~nz] = 0.0
        s = r @ np.asarray(S, dtype=np.float64).T
        out.update(rnorm=np.sqrt(np.sum(r * r, axis=1)), sign=(s >= 0).astype(np.int64), s=s, r=r)
    return out


def logits(q, Pi, S, c_lo, c_hi, m: int, norm, rnorm, idx, sign):
    """l[a, t] = n_t ( <Pi q_a, yhat_t> + rho_t sqrt(pi/2)/d <S q_a, 2 sign_t - 1> ), yhat per group."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[1]
    q_rot = q @ np.asarray(Pi, dtype=np.float64).T
    q_sk = q @ np.asarray(S, dtype=np.float64).T
    yhat = centroids_per_coordinate(idx, c_lo, c_hi, m)
    pm = 2.0 * np.asarray(sign, dtype=np.float64) - 1.0
    qjl = (q_sk @ pm.T) * (math.sqrt(math.pi / 2.0) / d) * np.asarray(rnorm, dtype=np.float64)[None, :]
    return np.asarray(norm, dtype=np.float64)[None, :] * (q_rot @ yhat.T + qjl)


def attend_v(lg, scale, v_norm, v_idx, Pi, c_lo, c_hi, m: int):
    """out[a] = Pi^T sum_t softmax(scale * lg[a])_t n_t yhat_t; no keys -> zeros."""
    lg = np.asarray(lg, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    nq, nt = lg.shape
    if nt == 0:
        return np.zeros((nq, Pi.shape[0]))
    z = scale * lg
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    vals = centroids_per_coordinate(v_idx, c_lo, c_hi, m) * np.asarray(v_norm, dtype=np.float64)[:, None]
    return (p @ vals) @ Pi


def mse_mix(d: int, m: int, mse_hi: float, mse_lo: float) -> float:
    """Per-vector MSE of the mixed-rate MSE stage from the two integer-rate per-vector MSEs."""
    return (m / d) * mse_hi + (1.0 - m / d) * mse_lo
