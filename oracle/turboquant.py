"""TurboQuant encoder, packed record, logit estimator and softmax.V (float64).

Test infrastructure (see ``oracle/__init__``). Plain NumPy, one vector or one
(query, key) pair at a time in spirit; vectorised over rows only where the
row operations are independent. No blocking, fusion or reordering.

Pages followed:
  [Z] zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5 bits
      per channel" (es/pt/fr), paragraph 2: stage one randomly rotates the
      vector; stage two applies an MSE quantizer and then a 1-bit quantized
      Johnson-Lindenstrauss transform of the residual; each token stores
      quantization indices, sign bits and an L2-norm scalar.
  [W] winningdata.io, "TurboQuant: Google comprime KV cache para 3 bits sem
      perder acuracia", "Como o TurboQuant funciona": "1. PolarQuant" (the
      rotation is a product with a random orthogonal matrix) and "2. QJL
      Residual" (one extra bit per value removes the inner-product bias).
  [U] usedby.ai, "TurboQuant: Compresion de KV Cache a 3 bits y aceleracion
      de inferencia en H100", "El Pitch": the attention logits are computed
      on the compressed keys.

Notation: x input vector (dimension d), n = ||x||, u = x/n, y = Pi u,
L = 2**bits centroids c (ascending), thresholds t_j = (c_j + c_{j+1})/2,
idx_i = #{j : y_i > t_j}, yhat_i = c[idx_i], r = u - Pi^T yhat, rho = ||r||,
s = S r, sign bit_i = [s_i >= 0].

Readings where the pages are silent:
  * keys carry bits-1 index bits + 1 sign bit per coordinate; values carry
    `bits` index bits and no sketch (MSE only).
  * keys store both n and rho; values store n only.
  * S is d x d (one sign bit per coordinate, [W] "1 bit extra por valor").
  * estimator: l = n * ( <Pi q, c[idx]> + rho * sqrt(pi/2)/d * <S q, 2 bit - 1> ).
    E_S[<Sq, sign(Sr)>] = d sqrt(2/pi) <q, r>/||r|| for Gaussian S, so the
    second term is unbiased for n <q, r> and the whole for <q, x>.
  * ties: y_i equal to a threshold goes to the lower cell; s_i = 0 gives bit 1.
  * zero vector: n = 0, u = 0, y = 0, r = 0, rho = 0 (all sign bits 1).
  * softmax.V: p = softmax(scale * l) over the keys, out = Pi^T sum_t p_t n_t c_V[idx_t]
    (the rotation is undone once, after the weighted sum); no keys -> zeros.
  * query head h reads KV head h // (n_q_heads / n_kv_heads).

Record layout (our specification; the pages give none):
  a record is `index_words + sign_words` little-endian uint32 words,
  index_words = ceil(bits*d/32), sign_words = ceil(d/32) for keys, 0 for values.
  The index field is a bit stream: bit k of the stream is bit (k mod 32) of
  word floor(k/32); the code of coordinate i occupies stream bits
  [bits*i, bits*i + bits), least significant bit first. The sign field holds
  bit_i at bit (i mod 32) of word index_words + floor(i/32). Unused bits are 0.
"""

from __future__ import annotations

import math

import numpy as np


# ----------------------------------------------------------------------------
# layout
# ----------------------------------------------------------------------------

def index_words(d: int, bits: int) -> int:
    return (bits * d + 31) // 32


def sign_words(d: int, qjl: bool) -> int:
    return (d + 31) // 32 if qjl else 0


def record_words(d: int, bits: int, qjl: bool) -> int:
    return index_words(d, bits) + sign_words(d, qjl)


def pack(idx, sign, d: int, bits: int, qjl: bool) -> np.ndarray:
    """Rows of codes (and sign bits) -> uint32 records, per the layout above."""
    idx = np.asarray(idx, dtype=np.int64).reshape(-1, d)
    n = idx.shape[0]
    iw = index_words(d, bits)
    stream = np.zeros((n, iw * 32), dtype=np.uint64)
    for b in range(bits):
        stream[:, np.arange(d) * bits + b] = (idx >> b) & 1
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    words = (stream.reshape(n, iw, 32) * weights).sum(axis=2)
    if qjl:
        sw = sign_words(d, True)
        sbits = np.zeros((n, sw * 32), dtype=np.uint64)
        sbits[:, :d] = np.asarray(sign, dtype=np.uint64).reshape(-1, d)
        words = np.concatenate([words, (sbits.reshape(n, sw, 32) * weights).sum(axis=2)], axis=1)
    return words.astype(np.uint32)


def unpack(records, d: int, bits: int, qjl: bool):
    """uint32 records -> (codes [n, d] int64, sign bits [n, d] or None)."""
    rec = np.asarray(records, dtype=np.uint64).reshape(-1, record_words(d, bits, qjl))
    n = rec.shape[0]
    iw = index_words(d, bits)
    shifts = np.arange(32, dtype=np.uint64)
    stream = ((rec[:, :iw, None] >> shifts) & np.uint64(1)).reshape(n, iw * 32)
    idx = np.zeros((n, d), dtype=np.int64)
    for b in range(bits):
        idx |= stream[:, np.arange(d) * bits + b].astype(np.int64) << b
    sign = None
    if qjl:
        sbits = ((rec[:, iw:, None] >> shifts) & np.uint64(1)).reshape(n, -1)
        sign = sbits[:, :d].astype(np.int64)
    return idx, sign


def padding_is_zero(records, d: int, bits: int, qjl: bool) -> bool:
    """True when every bit outside the codes and signs of the layout is 0."""
    rec = np.asarray(records, dtype=np.uint64).reshape(-1, record_words(d, bits, qjl))
    iw = index_words(d, bits)
    used = bits * d
    ok = True
    for w in range(iw):
        lo = w * 32
        nbits = max(0, min(32, used - lo))
        mask = (1 << nbits) - 1
        ok &= bool(np.all((rec[:, w] & np.uint64(~mask & 0xFFFFFFFF)) == 0))
    if qjl:
        for w in range(sign_words(d, True)):
            nbits = max(0, min(32, d - 32 * w))
            mask = (1 << nbits) - 1
            ok &= bool(np.all((rec[:, iw + w] & np.uint64(~mask & 0xFFFFFFFF)) == 0))
    return ok


# ----------------------------------------------------------------------------
# encoder  ([Z] stage one and two; [W] PolarQuant and QJL Residual)
# ----------------------------------------------------------------------------

def thresholds_of(codebook) -> np.ndarray:
    """Midpoints of adjacent centroids, exact in float64 for float32 centroids."""
    c = np.asarray(codebook, dtype=np.float64)
    return (c[:-1] + c[1:]) / 2.0


def quantize(x, Pi, codebook, S=None):
    """Encode rows of x. Returns dict(norm, idx, and for keys rnorm, sign, s, y).

    x: [n, d] (any real dtype; widened to float64), Pi: [d, d] orthogonal,
    codebook: 2**bits ascending centroids, S: [d, d] Gaussian sketch or None
    for the MSE-only (value) path.
    """
    x = np.asarray(x, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    c = np.asarray(codebook, dtype=np.float64)
    t = thresholds_of(c)
    n_rows, d = x.shape
    norm = np.sqrt(np.sum(x * x, axis=1))
    u = np.zeros_like(x)
    nz = norm > 0
    u[nz] = x[nz] / norm[nz, None]
    y = u @ Pi.T                                   # y = Pi u, row by row
    idx = np.searchsorted(t, y, side="left")       # #{j : t_j < y_i}; ties -> lower cell
    out = {"norm": norm, "idx": idx.astype(np.int64), "y": y}
    if S is not None:
        S = np.asarray(S, dtype=np.float64)
        yhat = c[idx]
        r = u - yhat @ Pi                          # r = u - Pi^T yhat
        r[~nz] = 0.0
        s = r @ S.T                                # s = S r
        out["rnorm"] = np.sqrt(np.sum(r * r, axis=1))
        out["sign"] = (s >= 0).astype(np.int64)
        out["s"] = s
        out["r"] = r
    return out


def dequantize_mse(norm, idx, Pi, codebook):
    """n * Pi^T c[idx]: the MSE-stage reconstruction of each row."""
    c = np.asarray(codebook, dtype=np.float64)
    return np.asarray(norm, dtype=np.float64)[:, None] * (c[np.asarray(idx)] @ np.asarray(Pi, dtype=np.float64))


# ----------------------------------------------------------------------------
# estimator on the packed cache  ([U] "El Pitch"; [W] "2. QJL Residual")
# ----------------------------------------------------------------------------

def logits(q, Pi, S, codebook, norm, rnorm, idx, sign):
    """l[a, t] = n_t ( <Pi q_a, c[idx_t]> + rho_t sqrt(pi/2)/d <S q_a, 2 sign_t - 1> ).

    q: [nq, d]; norm, rnorm: [nt]; idx, sign: [nt, d]. Returns [nq, nt].
    """
    q = np.asarray(q, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    c = np.asarray(codebook, dtype=np.float64)
    d = q.shape[1]
    q_rot = q @ Pi.T                                # Pi q
    q_sk = q @ S.T                                  # S q
    yhat = c[np.asarray(idx)]                       # [nt, d]
    pm = 2.0 * np.asarray(sign, dtype=np.float64) - 1.0
    mse_term = q_rot @ yhat.T                       # [nq, nt]
    qjl_term = (q_sk @ pm.T) * (math.sqrt(math.pi / 2.0) / d) * np.asarray(rnorm, dtype=np.float64)[None, :]
    return np.asarray(norm, dtype=np.float64)[None, :] * (mse_term + qjl_term)


def logits_mse_only(q, Pi, codebook, norm, idx):
    """The first term alone: n_t <Pi q, c[idx_t]> (biased; used to show QJL matters)."""
    q_rot = np.asarray(q, dtype=np.float64) @ np.asarray(Pi, dtype=np.float64).T
    yhat = np.asarray(codebook, dtype=np.float64)[np.asarray(idx)]
    return np.asarray(norm, dtype=np.float64)[None, :] * (q_rot @ yhat.T)


def attend_v(lg, scale, v_norm, v_idx, Pi, codebook_v):
    """out[a] = Pi^T sum_t softmax(scale * lg[a])_t * n_t * c_V[idx_t]   ([Z]: KV = keys and values).

    lg: [nq, nt] logits; v_norm: [nt]; v_idx: [nt, d]. Returns [nq, d].
    """
    lg = np.asarray(lg, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    nq, nt = lg.shape
    d = Pi.shape[0]
    if nt == 0:
        return np.zeros((nq, d))
    z = scale * lg
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    vals = np.asarray(codebook_v, dtype=np.float64)[np.asarray(v_idx)] * np.asarray(v_norm, dtype=np.float64)[:, None]
    acc = p @ vals                                  # rotated domain, [nq, d]
    return acc @ Pi                                 # Pi^T acc, row by row


def walsh_hadamard(x):
    """Unnormalised fast Walsh-Hadamard transform over the last axis (length a power of two):
    returns x H with H the Sylvester-Hadamard matrix, by log2(d) rounds of pairwise sums and
    differences. The structured rotation the pages' "O(d) per vector" cost refers to
    ([W] "1. PolarQuant"; a Hadamard product costs O(d log d)) is Pi = H diag(s) / sqrt(d)."""
    y = np.array(x, dtype=np.float64, copy=True)
    d = y.shape[-1]
    if d < 1 or d & (d - 1):
        raise ValueError(f"length {d} is not a power of two")
    h = 1
    while h < d:
        y = y.reshape(y.shape[:-1] + (d // (2 * h), 2, h))
        a, b = y[..., 0, :].copy(), y[..., 1, :].copy()
        y[..., 0, :], y[..., 1, :] = a + b, a - b
        y = y.reshape(y.shape[:-3] + (d,))
        h *= 2
    return y


def structured_rotate(u, signs):
    """Rows of u rotated by Pi = H diag(signs) / sqrt(d): (Pi u_row) = H (signs * u_row) / sqrt(d)."""
    u = np.asarray(u, dtype=np.float64)
    return walsh_hadamard(u * np.asarray(signs, dtype=np.float64)) / math.sqrt(u.shape[-1])


def kv_head_of(q_head: int, n_q_heads: int, n_kv_heads: int) -> int:
    """Contiguous grouped-query mapping (reading; winningdata.io, "Limitacoes e trade-offs"
    leaves GQA open)."""
    return q_head // (n_q_heads // n_kv_heads)


# ----------------------------------------------------------------------------
# nearest-neighbour search (zubnet.ai paragraph 3; winningdata.io "Os numeros que importam")
# ----------------------------------------------------------------------------

def topk(scores, k: int):
    """Per row, indices of the k largest scores; equal scores -> lower index first."""
    scores = np.asarray(scores, dtype=np.float64)
    out = np.empty((scores.shape[0], k), dtype=np.int64)
    for a in range(scores.shape[0]):
        order = np.lexsort((np.arange(scores.shape[1]), -scores[a]))
        out[a] = order[:k]
    return out
