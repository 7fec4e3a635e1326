"""The tensor-core quantizer's tile schedule: streams, repeats and graphs.

For keys its CTAs take 128-token tiles from a counter that the library hands out per stream
(and per launch recorded into a graph), and the launch's last CTA zeroes it again; values take
their tiles in a fixed order. Which CTA encodes a tile does not change the encoding, so every
launch must give the records, norms and rnorms of the first one bit for bit: back-to-back
launches on one stream (the counter is reset between them), launches on four streams at once
(each with its own counter) and a graph's replays. The first launch is checked against the
float64 oracle on sampled tokens.
"""

from __future__ import annotations

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


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok:
        pytest.skip("needs a CUDA device")


D, H, T = 128, 8, 40_000           # 2500 tiles: about 17 per CTA on a 148-SM part


def _setup(qjl, bits):
    dev = torch.device("cuda")
    Pi, S = syn.rotation(D), syn.sketch(D)
    cb = ocb.fit_codebook(D, bits)[0]
    x = syn.gaussian((1, H, T, D), 520 + bits, device=dev).to(torch.bfloat16)
    SPiT = tqb.tq_sketch_rotation(Pi.to(dev), S.to(dev)) if qjl else None
    return Pi, S, cb, x, SPiT


def _state(c):
    return [c.records.clone(), c.norm.clone()] + ([c.rnorm.clone()] if c.qjl else [])


@pytest.mark.parametrize("qjl,bits", [(True, 2), (False, 3)])
def test_schedule_repeats_streams_graph(qjl, bits):
    Pi, S, cb, x, SPiT = _setup(qjl, bits)
    dev = torch.device("cuda")
    Pid, cbd = Pi.to(dev), torch.from_numpy(cb).to(dev)
    mk = lambda: tqb.PackedCache.empty(D, bits, qjl, 1, H, T)
    c0 = mk()
    tqb.tq_quantize_append(c0, x, 0, Pid, SPiT, cbd)
    torch.cuda.synchronize()
    want = _state(c0)

    # the oracle on sampled tokens of the first launch
    rows = np.random.default_rng(5).choice(H * T, 300, replace=False)
    xs = x.reshape(H * T, D)[torch.from_numpy(rows).to(dev)].float().cpu().numpy().astype(np.float64)
    rec = par.as_u32(c0.records.reshape(H * T, -1)[torch.from_numpy(rows).to(dev)].cpu().numpy())
    nrm = c0.norm.reshape(-1)[torch.from_numpy(rows).to(dev)].cpu().numpy()
    rn = c0.rnorm.reshape(-1)[torch.from_numpy(rows).to(dev)].cpu().numpy() if qjl else None
    par.check_encoding(xs, rec, nrm, rn, Pi.double().numpy(), S.double().numpy(), cb, D, bits, qjl)

    # back to back on one stream
    for _ in range(4):
        c0.records.zero_()
        tqb.tq_quantize_append(c0, x, 0, Pid, SPiT, cbd)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(_state(c0), want))

    # four streams at once, three launches each
    caches = [mk() for _ in range(4)]
    streams = [torch.cuda.Stream() for _ in range(4)]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    for _ in range(3):
        for c, s in zip(caches, streams):
            with torch.cuda.stream(s):
                tqb.tq_quantize_append(c, x, 0, Pid, SPiT, cbd)
    for s in streams:
        torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for c in caches:
        assert all(torch.equal(a, b) for a, b in zip(_state(c), want))

    # a graph's replays
    cg = mk()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        tqb.tq_quantize_append(cg, x, 0, Pid, SPiT, cbd)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        tqb.tq_quantize_append(cg, x, 0, Pid, SPiT, cbd)
    for _ in range(3):
        cg.records.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert all(torch.equal(a, b) for a, b in zip(_state(cg), want))
