"""The path replayed from CUDA graphs: every call is stream-ordered and capturable.

A serving loop captures its per-token work once and replays it; the library's calls make no host
synchronisation and, after the first key quantize call, allocate nothing, and their kernels'
programmatic-dependent launches are captured as graph edges. Captured once after a warm-up call
(which also sets the kernels' shared-memory attributes), each graph is replayed several times and
must give the eager call's result bit for bit:
the one-call decode step for one and for four query heads per KV head, and quantize-append + logits +
softmax.V as one graph.
"""

from __future__ import annotations

import math

import pytest
import torch

import tq_synth as syn
from oracle import codebook as ocb

pytestmark = pytest.mark.gpu

cuda_ok = torch.cuda.is_available()
if cuda_ok:
    import kv_cache_vector_quantize_b200 as tqb


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok:
        pytest.skip("needs a CUDA device")


def _setup(H, G, T, seed):
    d = 128
    dev = torch.device("cuda")
    Pi, S = syn.rotation(d).to(dev), syn.sketch(d).to(dev)
    ck = torch.from_numpy(ocb.fit_codebook(d, 2)[0]).to(dev)
    cv = torch.from_numpy(ocb.fit_codebook(d, 3)[0]).to(dev)
    SPiT = tqb.tq_sketch_rotation(Pi, S)
    k = syn.gaussian((1, H, T, d), seed, device=dev).to(torch.bfloat16)
    v = syn.lognormal_sphere((1, H, T, d), seed + 1, dtype=torch.bfloat16, device=dev)
    q = syn.gaussian((1, H * G, d), seed + 2, device=dev)
    kc = tqb.PackedCache.empty(d, 2, True, 1, H, T)
    vc = tqb.PackedCache.empty(d, 3, False, 1, H, T)
    return dict(d=d, Pi=Pi, S=S, ck=ck, cv=cv, SPiT=SPiT, k=k, v=v, q=q, kc=kc, vc=vc)


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()                                   # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("G", [1, 4])
def test_decode_step_replays_bit_equal(G):
    H, T = 2, 3000
    c = _setup(H, G, T, 300 + G)
    tqb.tq_quantize_append(c["kc"], c["k"], 0, c["Pi"], c["SPiT"], c["ck"])
    tqb.tq_quantize_append(c["vc"], c["v"], 0, c["Pi"], None, c["cv"])
    sc = 1.0 / math.sqrt(c["d"])
    want = tqb.tq_decode_attend(c["kc"], c["vc"], c["q"], T, sc, c["Pi"], c["S"], c["ck"], c["cv"])
    torch.cuda.synchronize()
    out = torch.empty_like(want)
    ws = torch.zeros(max(256, tqb.tq_decode_workspace_size(c["kc"], c["vc"], H * G, T)), dtype=torch.uint8,
                     device="cuda")
    g = _capture(lambda: tqb.tq_decode_attend(c["kc"], c["vc"], c["q"], T, sc, c["Pi"], c["S"], c["ck"], c["cv"],
                                              out=out, workspace=ws))
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, want)
    tqb.tq_workspace_status(ws)


def test_quantize_logits_softmax_v_replay_bit_equal():
    H, G, T = 2, 4, 2049
    c = _setup(H, G, T, 310)
    sc = 1.0 / math.sqrt(c["d"])
    kc, vc = c["kc"], c["vc"]
    ws_l = torch.zeros(max(256, tqb.tq_logits_workspace_size(kc, H * G)), dtype=torch.uint8, device="cuda")
    ws_a = torch.zeros(max(256, tqb.tq_attend_workspace_size(vc, H * G, T)), dtype=torch.uint8, device="cuda")
    lg = torch.empty((1, H * G, T), dtype=torch.float32, device="cuda")
    out = torch.empty((1, H * G, c["d"]), dtype=torch.float32, device="cuda")

    def step():
        tqb.tq_quantize_append(kc, c["k"], 0, c["Pi"], c["SPiT"], c["ck"])
        tqb.tq_quantize_append(vc, c["v"], 0, c["Pi"], None, c["cv"])
        tqb.tq_logits(kc, c["q"], T, c["Pi"], c["S"], c["ck"], logits=lg, workspace=ws_l)
        tqb.tq_attend_v(vc, lg, sc, T, c["Pi"], c["cv"], out=out, workspace=ws_a)

    step()
    torch.cuda.synchronize()
    want_rec, want_out = kc.records.clone(), out.clone()
    g = _capture(step)
    for _ in range(3):
        kc.records.zero_()
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(kc.records, want_rec)
        assert torch.equal(out, want_out)
    tqb.tq_workspace_status(ws_l)
    tqb.tq_workspace_status(ws_a)
