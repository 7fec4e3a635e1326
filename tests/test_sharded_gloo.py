"""Multi-rank plumbing of the split data paths on CPU: two gloo ranks (kv_cache_vector_quantize_b200.sharded).

A nearest-neighbour database split by rows and a KV cache split by tokens each need one exchange:
per-shard top-k lists, or per-range softmax.V partials (M, L, A), all-gathered and merged. Here the
ranks' local results come from the float64 oracle and the merge steps are plain float64 restatements
(the library's merge kernels need a GPU; tests/test_gpu_sharded.py checks them), so what is tested
is the host side: the split, the global ids, the gather order and the layout the merges receive.
Both ranks must end with the single-process result.
"""

from __future__ import annotations

import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(d=32, n_db=301, n_q=5, bits=2, seed=3):
    from oracle import codebook as ocb
    from oracle import turboquant as otq
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((d, d))
    qm, r = np.linalg.qr(a)
    Pi = qm * np.sign(np.diag(r))[None, :]
    S = rng.standard_normal((d, d))
    c = ocb.fit_codebook(d, bits)[0]
    db = rng.standard_normal((n_db, d))
    db[7] = db[11]                      # equal vectors: equal scores, ranked by id across shards
    e = otq.quantize(db, Pi, c, S)
    q = rng.standard_normal((n_q, d))
    scores = otq.logits(q, Pi, S, c, e["norm"], e["rnorm"], e["idx"], e["sign"])
    return Pi, S, c, e, q, scores


def _topk_with_scores(scores, k):
    from oracle import turboquant as otq
    ids = otq.topk(scores, k)
    return np.take_along_axis(scores, ids, axis=1), ids


def _merge_lists_f64(ps, pi):
    """[parts, n_q, k] lists -> top-k by (score desc, id asc), empty places (-1) skipped."""
    parts, nq, k = ps.shape
    out_s = torch.full((nq, k), -math.inf, dtype=ps.dtype)
    out_i = torch.full((nq, k), -1, dtype=pi.dtype)
    for a in range(nq):
        cand = [(float(ps[p, a, j]), int(pi[p, a, j])) for p in range(parts) for j in range(k) if int(pi[p, a, j]) >= 0]
        cand.sort(key=lambda t: (-t[0], t[1]))
        for j, (sv, iv) in enumerate(cand[:k]):
            out_s[a, j], out_i[a, j] = sv, iv
    return out_s, out_i


def _partial_f64(lg, scale, norm, yhat):
    """(M, L, A) per row of a token range: the softmax.V pieces before the merge."""
    z = scale * lg
    if z.shape[1] == 0:
        out = np.zeros((lg.shape[0], yhat.shape[1] + 2))
        out[:, 0] = -math.inf
        return out
    M = z.max(axis=1)
    w = np.exp(z - M[:, None])
    A = (w * norm[None, :]) @ yhat
    return np.concatenate([M[:, None], w.sum(axis=1)[:, None], A], axis=1)


def _merge_partials_f64(parts, Pi):
    """[rows, n_parts, d + 2] -> Pi^T (sum_p e^{M_p - M} A_p) / (sum_p e^{M_p - M} L_p)."""
    parts = parts.numpy()
    M = parts[:, :, 0].max(axis=1)
    f = np.exp(parts[:, :, 0] - M[:, None])
    L = (f * parts[:, :, 1]).sum(axis=1)
    A = (f[:, :, None] * parts[:, :, 2:]).sum(axis=1)
    return torch.from_numpy((A / L[:, None]) @ np.asarray(Pi))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from kv_cache_vector_quantize_b200 import sharded as sh
    try:
        # ---- nearest-neighbour database split by rows ----
        k = 6
        Pi, S, c, e, q, scores = _case()
        b, en = sh.shard_range(scores.shape[1], world, rank)
        ls, li = _topk_with_scores(scores[:, b:en], k)
        got_s, got_i = sh.merge_topk_sharded(torch.from_numpy(ls), torch.from_numpy(li), b,
                                             merge=_merge_lists_f64)
        want_s, want_i = _topk_with_scores(scores, k)
        nn_ok = bool(np.array_equal(got_i.numpy(), want_i) and np.array_equal(got_s.numpy(), want_s))
        # ---- KV cache split by tokens ----
        T, nq = 257, 3
        rng = np.random.default_rng(9)
        lg = 4.0 * rng.standard_normal((nq, T))
        norm = np.exp(0.5 * rng.standard_normal(T))
        yhat = np.asarray(c, dtype=np.float64)[rng.integers(0, len(c), size=(T, Pi.shape[0]))]
        scale = 0.3
        ref = (np.exp(scale * lg - (scale * lg).max(axis=1, keepdims=True)) /
               np.exp(scale * lg - (scale * lg).max(axis=1, keepdims=True)).sum(axis=1, keepdims=True)) @ (
                   norm[:, None] * yhat) @ Pi
        b, en = sh.shard_range(T, world, rank)
        part = torch.from_numpy(_partial_f64(lg[:, b:en], scale, norm[b:en], yhat[b:en]))
        got = sh.merge_attend_sharded(part, torch.from_numpy(Pi), merge=_merge_partials_f64)
        att_ok = bool(np.allclose(got.numpy(), ref, rtol=0, atol=1e-12))
        # an empty range among the parts (every rank adds one)
        empty = torch.from_numpy(_partial_f64(lg[:, :0], scale, norm[:0], yhat[:0]))
        both = sh.gather_parts(part)
        parts = torch.cat([both, empty[None]]).transpose(0, 1).contiguous()
        got2 = _merge_partials_f64(parts, Pi)
        att_ok &= bool(np.allclose(got2.numpy(), ref, rtol=0, atol=1e-12))
        out.put((rank, nn_ok, att_ok))
    finally:
        dist.destroy_process_group()


def test_shard_range_partitions_exactly():
    from kv_cache_vector_quantize_b200 import sharded as sh
    for n in (0, 1, 7, 301, 1_000_000):
        for world in (1, 2, 3, 8):
            spans = [sh.shard_range(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sh.shard_range(5, 2, 2)


def test_globalize_ids_keeps_empty_places():
    from kv_cache_vector_quantize_b200 import sharded as sh
    ids = torch.tensor([[0, 5, -1], [2, -1, -1]])
    assert sh.globalize_ids(ids, 100).tolist() == [[100, 105, -1], [102, -1, -1]]


def test_two_gloo_ranks_merge_to_the_single_process_result():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, nn_ok, att_ok in res:
        assert nn_ok, f"rank {rank}: merged top-k differs from the single-process top-k"
        assert att_ok, f"rank {rank}: merged softmax.V differs from the single-process result"
