"""GPU checks of the merge steps of the split data paths, on one GPU (kv_cache_vector_quantize_b200.sharded).

A database split by rows: every shard gets its own cache and search, its ids are made global and
tq_nn_merge combines the lists; the result must be the unsplit search exactly (the scan scores a
(query, vector) pair the same way whichever tile holds the vector). A value cache split by tokens:
every token range gets tq_attend_v_partial, tq_attend_merge combines them; the result must match
tq_attend_v on the whole cache (rounding only) and the oracle's softmax.V within the parity
tolerance, with an empty range among the parts. Only the collective itself (an all-gather, tested
with gloo ranks on the CPU) is left out: the parts are stacked on one device.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import tq_synth as syn
from oracle import codebook as ocb
from tests import _parity as par

pytestmark = pytest.mark.gpu

cuda_ok = torch.cuda.is_available()
if cuda_ok:
    import kv_cache_vector_quantize_b200 as tqb
    from kv_cache_vector_quantize_b200 import sharded as sh


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok:
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("d,bits,n_db,k,world", [(200, 1, 5003, 10, 3), (128, 2, 1500, 16, 4), (128, 3, 37, 5, 2)])
def test_sharded_search_equals_unsharded(d, bits, n_db, k, world):
    dev = torch.device("cuda")
    db, qs = syn.nn_inputs(n_db, 300, d, device=dev)
    db[5] = db[n_db - 3]                     # equal vectors in different shards: ranked by global id
    Pi, S = syn.rotation(d).to(dev), syn.sketch(d).to(dev)
    cb = torch.from_numpy(ocb.fit_codebook(d, bits)[0]).to(dev)
    SPiT = tqb.tq_sketch_rotation(Pi, S)
    whole = tqb.PackedCache.empty(d, bits, True, 1, 1, n_db)
    tqb.tq_quantize_append(whole, db.reshape(1, 1, n_db, d), 0, Pi, SPiT, cb)
    want_s, want_i = tqb.tq_nn_search(whole, qs, n_db, Pi, S, cb, k)
    parts_s, parts_i = [], []
    for r in range(world):
        b, e = sh.shard_range(n_db, world, r)
        c = tqb.PackedCache.empty(d, bits, True, 1, 1, max(e - b, 1))
        if e > b:
            tqb.tq_quantize_append(c, db[b:e].reshape(1, 1, e - b, d).contiguous(), 0, Pi, SPiT, cb)
        s, i = tqb.tq_nn_search(c, qs, e - b, Pi, S, cb, k)
        parts_s.append(s)
        parts_i.append(sh.globalize_ids(i, b))
    got_s, got_i = tqb.tq_nn_merge(torch.stack(parts_s), torch.stack(parts_i))
    torch.cuda.synchronize()
    assert torch.equal(got_i, want_i)
    assert torch.equal(got_s, want_s)


def test_nn_merge_short_lists_and_padding():
    # two parts, k = 4: one part has 2 entries, the other none; ties by id
    dev = torch.device("cuda")
    ps = torch.tensor([[[3.0, 1.0, -math.inf, -math.inf]], [[-math.inf] * 4]], device=dev)
    pi = torch.tensor([[[7, 2, -1, -1]], [[-1, -1, -1, -1]]], dtype=torch.int64, device=dev)
    s, i = tqb.tq_nn_merge(ps, pi)
    assert i.tolist() == [[7, 2, -1, -1]] and s[0, :2].tolist() == [3.0, 1.0] and bool(torch.isneginf(s[0, 2:]).all())
    ps = torch.tensor([[[2.0, 2.0]], [[2.0, 1.0]]], device=dev)
    pi = torch.tensor([[[9, 12]], [[4, 1]]], dtype=torch.int64, device=dev)
    s, i = tqb.tq_nn_merge(ps, pi)
    assert i.tolist() == [[4, 9]] and s.tolist() == [[2.0, 2.0]]


@pytest.mark.parametrize("d,bits,B,H,G,T", [(128, 3, 1, 2, 4, 3000), (128, 2, 2, 1, 1, 1537), (64, 3, 1, 2, 2, 700)])
def test_sharded_softmax_v_matches_single_call(d, bits, B, H, G, T):
    dev = torch.device("cuda")
    Pi = syn.rotation(d).to(dev)
    cv = torch.from_numpy(ocb.fit_codebook(d, bits)[0]).to(dev)
    v = syn.lognormal_sphere((B, H, T, d), 81, dtype=torch.bfloat16, device=dev)
    vc = tqb.PackedCache.empty(d, bits, False, B, H, T)
    tqb.tq_quantize_append(vc, v, 0, Pi, None, cv)
    lg = 3.0 * syn.gaussian((B, H * G, T), 82, device=dev)
    sc = 1.0 / math.sqrt(d)
    want = tqb.tq_attend_v(vc, lg, sc, T, Pi, cv)
    # four token ranges, one of them empty, cut at multiples of 4 tokens: the cache seen from a token
    # offset (records and norms advanced, the same capacity stride between (sequence, head) rows)
    a1, a2 = (T // 3) & ~3, (2 * T // 3) & ~3
    bounds = [0, a1, a1, a2, T]
    parts = [_partial(vc, a, b, lg[:, :, a:b].contiguous(), sc, cv) for a, b in zip(bounds[:-1], bounds[1:])]
    got = tqb.tq_attend_merge(torch.stack(parts, dim=1).contiguous(), Pi).view(B, H * G, d)
    torch.cuda.synchronize()
    scale_ref = float(vc.norm.max())
    assert float((got - want).abs().max()) <= 1e-5 * scale_ref
    # and the oracle's softmax.V of the whole cache
    rec = par.as_u32(vc.records.cpu().numpy())
    for s_ in range(B):
        for h in range(H):
            par.check_attend(got[s_, h * G:(h + 1) * G].cpu().numpy(), lg[s_, h * G:(h + 1) * G].cpu().numpy().astype(np.float64),
                             sc, Pi.cpu().numpy(), cv.cpu().numpy(), rec[s_, h], vc.norm[s_, h].cpu().numpy(), d, bits)


def _partial(vc, a, b, lg, sc, cv):
    """tq_attend_v_partial through the C ABI for tokens [a, b) of vc (a descriptor offset by a tokens)."""
    import ctypes
    lib = tqb.raw_lib()
    rw = vc.records.shape[-1]
    desc = tqb.TqCacheDesc(vc.d, vc.idx_bits, 0, vc.n_seq, vc.n_kv_heads, 0, vc.capacity,
                           vc.records.data_ptr() + 4 * rw * a, vc.norm.data_ptr() + 4 * a, None)
    hq, n = lg.shape[1], b - a
    part = torch.empty((vc.n_seq * hq, vc.d + 2), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(256, lib.tq_attend_workspace_size(ctypes.byref(desc), hq, n)), dtype=torch.uint8,
                     device="cuda")
    st = lib.tq_attend_v_partial(ctypes.byref(desc), ctypes.c_void_p(lg.data_ptr()), ctypes.c_float(sc), hq, n,
                                 ctypes.c_void_p(cv.data_ptr()), ctypes.c_void_p(part.data_ptr()),
                                 ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == tqb.TQ_OK, tqb.tq_last_error()
    return part
