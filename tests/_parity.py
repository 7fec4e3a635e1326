"""Comparison of the CUDA path's packed cache, logits and outputs with the oracle.

Tolerances (the method's parity bounds):
  * codes and sign bits bit-exact, except a code that moved exactly one cell across
    the threshold t_j between its two cells while the rotated value lies within 1e-5
    of that threshold (|y_i - t_j| <= 1e-5 with ||u|| = 1 and ||Pi_i|| = 1), or a sign
    whose sketch value lies within 1e-5 ||S_i|| rho of zero;
    such excused flips must be at most 1e-4 of all coordinates;
  * norms (||x|| and rho) to 1e-5 relative;
  * logits to 2e-3 * ||q|| * n_t, with the oracle evaluated on the GPU's cache;
  * softmax.V to 2e-3 * max_t n_t (infinity norm), oracle on the GPU's cache and logits;
  * nearest-neighbour top-k: each returned score within the logit tolerance of the
    oracle's score of that database vector, the r-th returned score within the
    tolerance of the oracle's r-th largest score (order statistics move by at most
    the largest score error), indices distinct, scores non-increasing, equal scores
    in index order, and (-inf, -1) exactly where the database has fewer than k vectors.
Where the GPU moved a code across a threshold (excused), rho and the sign bits
are checked against the oracle re-run on the GPU's codes.
"""

from __future__ import annotations

import numpy as np

from oracle import turboquant as otq

FLIP_BAND = 1e-5
FLIP_RATE_MAX = 1e-4
NORM_RTOL = 1e-5
LOGIT_TOL = 2e-3
OUT_TOL = 2e-3


def as_u32(records_i32) -> np.ndarray:
    return np.ascontiguousarray(records_i32).view(np.uint32)


def check_encoding(x, rec, norm, rnorm, Pi, S, codebook, d, bits, qjl):
    """x: [n, d] float64 inputs (widened exactly), rec: [n, R] uint32, norm/rnorm [n].
    Returns a dict of counts; raises AssertionError on any violation."""
    x = np.asarray(x, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    c = np.asarray(codebook, dtype=np.float64)
    n = x.shape[0]
    assert rec.shape == (n, otq.record_words(d, bits, qjl)), rec.shape
    assert otq.padding_is_zero(rec, d, bits, qjl), "non-zero padding bits"
    enc = otq.quantize(x, Pi, codebook, S if qjl else None)
    # ||x||
    ref_n = enc["norm"]
    bad = np.abs(norm - ref_n) > NORM_RTOL * np.maximum(ref_n, 1e-30)
    assert not bad.any(), f"norm mismatch at rows {np.nonzero(bad)[0][:10]}: {norm[bad][:5]} vs {ref_n[bad][:5]}"
    gi, gs = otq.unpack(rec, d, bits, qjl)
    t = otq.thresholds_of(c)
    oi = enc["idx"]
    idiff = gi != oi
    # An excused code moved exactly one cell, across the threshold between the two cells
    # (t_j between cells j and j + 1), and y_i lies within the band of that threshold.
    one_cell = np.abs(gi - oi) == 1
    between = t[np.clip(np.minimum(gi, oi), 0, len(t) - 1)] if len(t) else np.zeros_like(enc["y"])
    near = np.abs(enc["y"] - between) <= FLIP_BAND
    unexcused = idiff & ~(one_cell & near)
    assert not unexcused.any(), (
        f"{unexcused.sum()} code mismatches that are not one-cell moves across a threshold within the band; "
        f"first at "
        f"{np.argwhere(unexcused)[:5].tolist()} y={enc['y'][unexcused][:5]} gpu={gi[unexcused][:5]} "
        f"oracle={enc['idx'][unexcused][:5]}")
    out = {"coords": n * d, "index_flips": int(idiff.sum()), "sign_flips": 0}
    if qjl:
        S64 = np.asarray(S, dtype=np.float64)
        nz = ref_n > 0
        u = np.zeros_like(x)
        u[nz] = x[nz] / ref_n[nz, None]
        r = u - c[gi] @ Pi
        r[~nz] = 0.0
        rho = np.sqrt(np.sum(r * r, axis=1))
        bad = np.abs(rnorm - rho) > NORM_RTOL * np.maximum(rho, 1e-30) + 1e-7 * (rho == 0)
        assert not bad.any(), f"rnorm mismatch at rows {np.nonzero(bad)[0][:10]}: {rnorm[bad][:5]} vs {rho[bad][:5]}"
        s = r @ S64.T
        want = (s >= 0).astype(np.int64)
        sdiff = gs != want
        band = FLIP_BAND * np.linalg.norm(S64, axis=1)[None, :] * rho[:, None]
        unexcused = sdiff & (np.abs(s) > band)
        assert not unexcused.any(), (
            f"{unexcused.sum()} sign mismatches outside the zero band; first at {np.argwhere(unexcused)[:5].tolist()}")
        out["sign_flips"] = int(sdiff.sum())
    for field in ("index_flips", "sign_flips"):
        assert out[field] <= FLIP_RATE_MAX * n * d, f"excused {field} {out[field]} exceed 1e-4 of {n * d} coordinates"
    return out


def check_logits(gpu, q, Pi, S, codebook, rec, norm, rnorm, d, bits):
    """gpu: [nq, nt] logits; q: [nq, d] for ONE kv head; rec/norm/rnorm: that head's GPU cache."""
    gi, gs = otq.unpack(rec, d, bits, True)
    ref = otq.logits(q, Pi, S, codebook, norm, rnorm, gi, gs)
    tol = LOGIT_TOL * np.linalg.norm(np.asarray(q, dtype=np.float64), axis=1)[:, None] * np.asarray(norm)[None, :]
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    assert np.all(err <= tol + 1e-30), f"logit error {np.max(err / (tol + 1e-30)):.3g} x tolerance"
    return float(np.max(err / (tol + 1e-30))) if err.size else 0.0


def check_attend(gpu, lg, scale, Pi, codebook, rec, norm, d, bits):
    """gpu: [nq, d] outputs; lg: [nq, nt] the logits fed to the GPU; rec/norm: one kv head's value cache."""
    gi, _ = otq.unpack(rec, d, bits, False)
    ref = otq.attend_v(lg, scale, norm, gi, Pi, codebook)
    tol = OUT_TOL * (float(np.max(norm)) if len(norm) else 1.0)
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    assert np.all(err <= tol), f"softmax.V error {np.max(err) / tol:.3g} x tolerance"
    return float(np.max(err) / tol) if err.size else 0.0


def nn_scores(q, Pi, S, codebook, rec, norm, rnorm, d, bits, rows=100_000):
    """Oracle estimator scores [nq, n_db] of queries q over a packed database, unpacked in row blocks."""
    n_db = rec.shape[0]
    ref = np.empty((np.asarray(q).shape[0], n_db), dtype=np.float64)
    for a in range(0, n_db, rows):
        gi, gs = otq.unpack(rec[a:a + rows], d, bits, True)
        ref[:, a:a + rows] = otq.logits(q, Pi, S, codebook, norm[a:a + rows], rnorm[a:a + rows], gi, gs)
    return ref


def check_nn(gpu_s, gpu_i, q, Pi, S, codebook, rec, norm, rnorm, d, bits, k):
    """gpu_s/gpu_i: [nq, k] top-k scores and ids; q: [nq, d]; rec/norm/rnorm: the GPU's database
    cache (already checked against the oracle's encoding). Returns the worst error / tolerance."""
    ref = nn_scores(q, Pi, S, codebook, rec, norm, rnorm, d, bits)   # [nq, n_db] float64
    n_db = ref.shape[1]
    kk = min(k, n_db)
    gpu_s = np.asarray(gpu_s, dtype=np.float64)
    gpu_i = np.asarray(gpu_i)
    assert np.all(gpu_i[:, kk:] == -1) and np.all(np.isneginf(gpu_s[:, kk:])), "padding entries"
    worst = 0.0
    qn = np.linalg.norm(np.asarray(q, dtype=np.float64), axis=1)
    nmax = float(np.max(norm)) if n_db else 0.0
    for a in range(gpu_s.shape[0]):
        ids, sc = gpu_i[a, :kk], gpu_s[a, :kk]
        assert np.all((ids >= 0) & (ids < n_db)), f"query {a}: ids out of range {ids}"
        assert len(set(ids.tolist())) == kk, f"query {a}: repeated ids {ids}"
        assert np.all(np.diff(sc) <= 0), f"query {a}: scores not sorted {sc}"
        ties = np.nonzero(np.diff(sc) == 0)[0]
        assert np.all(ids[ties] < ids[ties + 1]), f"query {a}: equal scores out of index order"
        tol_j = LOGIT_TOL * qn[a] * np.asarray(norm)[ids] + 1e-30
        err = np.abs(sc - ref[a, ids])
        assert np.all(err <= tol_j), f"query {a}: score error {np.max(err / tol_j):.3g} x tolerance"
        # a returned vector must not have an exactly equal oracle score with a lower index that was
        # left out (identical records tie exactly; the lower index ranks first)
        left_out = np.ones(n_db, dtype=bool)
        left_out[ids] = False
        for j in ids:
            tied = np.nonzero(left_out[:j] & (ref[a, :j] == ref[a, j]))[0]
            assert len(tied) == 0, f"query {a}: id {j} returned ahead of the equal-scored lower id {tied[0]}"
        tol = LOGIT_TOL * qn[a] * nmax + 1e-30
        order = np.sort(ref[a])[::-1][:kk]
        oerr = np.abs(sc - order)
        assert np.all(oerr <= tol), f"query {a}: rank error {np.max(oerr / tol):.3g} x tolerance"
        worst = max(worst, float(np.max(err / tol_j)), float(np.max(oerr / tol)))
    return worst


# ----------------------------------------------------------------------------
# mixed rate (the first m coordinates at beta + 1 code bits): the same tolerances,
# oracle/mixed_rate.py as the reference
# ----------------------------------------------------------------------------

def check_encoding_mixed(x, rec, norm, rnorm, Pi, S, c_lo, c_hi, d, beta, m, qjl):
    from oracle import mixed_rate as omr

    x = np.asarray(x, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    n = x.shape[0]
    assert rec.shape == (n, omr.record_words(d, beta, m, qjl)), rec.shape
    assert omr.padding_is_zero(rec, d, beta, m, qjl), "non-zero padding bits"
    enc = omr.quantize(x, Pi, c_lo, c_hi, m, S if qjl else None)
    ref_n = enc["norm"]
    bad = np.abs(norm - ref_n) > NORM_RTOL * np.maximum(ref_n, 1e-30)
    assert not bad.any(), f"norm mismatch at rows {np.nonzero(bad)[0][:10]}"
    gi, gs = omr.unpack(rec, d, beta, m, qjl)
    oi = enc["idx"]
    idiff = gi != oi
    t_lo = otq.thresholds_of(c_lo)
    t_hi = otq.thresholds_of(c_hi)
    lower = np.minimum(gi, oi)
    between = np.empty(gi.shape)
    between[:, :m] = t_hi[np.clip(lower[:, :m], 0, len(t_hi) - 1)]
    between[:, m:] = t_lo[np.clip(lower[:, m:], 0, len(t_lo) - 1)]
    near = np.abs(enc["y"] - between) <= FLIP_BAND
    unexcused = idiff & ~((np.abs(gi - oi) == 1) & near)
    assert not unexcused.any(), (
        f"{unexcused.sum()} code mismatches that are not one-cell moves across a threshold within the band; "
        f"first at {np.argwhere(unexcused)[:5].tolist()}")
    out = {"coords": n * d, "index_flips": int(idiff.sum()), "sign_flips": 0}
    if qjl:
        S64 = np.asarray(S, dtype=np.float64)
        nz = ref_n > 0
        u = np.zeros_like(x)
        u[nz] = x[nz] / ref_n[nz, None]
        r = u - omr.centroids_per_coordinate(gi, c_lo, c_hi, m) @ Pi
        r[~nz] = 0.0
        rho = np.sqrt(np.sum(r * r, axis=1))
        bad = np.abs(rnorm - rho) > NORM_RTOL * np.maximum(rho, 1e-30) + 1e-7 * (rho == 0)
        assert not bad.any(), f"rnorm mismatch at rows {np.nonzero(bad)[0][:10]}"
        s = r @ S64.T
        sdiff = gs != (s >= 0).astype(np.int64)
        band = FLIP_BAND * np.linalg.norm(S64, axis=1)[None, :] * rho[:, None]
        unexcused = sdiff & (np.abs(s) > band)
        assert not unexcused.any(), f"{unexcused.sum()} sign mismatches outside the zero band"
        out["sign_flips"] = int(sdiff.sum())
    for field in ("index_flips", "sign_flips"):
        assert out[field] <= FLIP_RATE_MAX * n * d, f"excused {field} {out[field]} exceed 1e-4 of {n * d} coordinates"
    return out


def check_logits_mixed(gpu, q, Pi, S, c_lo, c_hi, rec, norm, rnorm, d, beta, m):
    from oracle import mixed_rate as omr

    gi, gs = omr.unpack(rec, d, beta, m, True)
    ref = omr.logits(q, Pi, S, c_lo, c_hi, m, norm, rnorm, gi, gs)
    tol = LOGIT_TOL * np.linalg.norm(np.asarray(q, dtype=np.float64), axis=1)[:, None] * np.asarray(norm)[None, :]
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    assert np.all(err <= tol + 1e-30), f"logit error {np.max(err / (tol + 1e-30)):.3g} x tolerance"
    return float(np.max(err / (tol + 1e-30))) if err.size else 0.0


def check_attend_mixed(gpu, lg, scale, Pi, c_lo, c_hi, rec, norm, d, beta, m):
    from oracle import mixed_rate as omr

    gi, _ = omr.unpack(rec, d, beta, m, False)
    ref = omr.attend_v(lg, scale, norm, gi, Pi, c_lo, c_hi, m)
    tol = OUT_TOL * (float(np.max(norm)) if len(norm) else 1.0)
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    assert np.all(err <= tol), f"softmax.V error {np.max(err) / tol:.3g} x tolerance"
    return float(np.max(err) / tol) if err.size else 0.0
