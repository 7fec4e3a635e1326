"""tq_attend_v_noalloc: softmax.V with the library's built-in scratch array.

Some callers cannot allocate device memory themselves: plugins inside a host
framework that owns all device memory through its own pool and gives them no
scratch buffer, or latency-critical decode loops that must not call cudaMalloc.
For them the library offers tq_attend_v_noalloc, which takes the same inputs
and outputs as tq_attend_v but uses a fixed array compiled into the library.

These tests call it through the C ABI and compare its output with the regular
tq_attend_v on the same inputs (with a caller workspace), for two calls in a
row with different shapes, so that nothing left in the shared array by the
first call can leak into the second. Both paths run the same kernels on the same
inputs, so the outputs must be bit-identical. After each call the array's status
word is read with tq_attend_v_noalloc_status, the only way a caller can see a
device-side failure of this entry point. The file is named so that pytest
collects it last.
"""

from __future__ import annotations

import ctypes
import math

import pytest
import torch

import tq_synth as syn

pytestmark = pytest.mark.gpu

cuda_ok = torch.cuda.is_available()
if cuda_ok:
    import kv_cache_vector_quantize_b200 as tqb


def _noalloc(vc, logits, scale, n_tokens, Pi, cb, out):
    lib = tqb.raw_lib()
    desc = vc.desc()
    return lib.tq_attend_v_noalloc(ctypes.byref(desc), ctypes.c_void_p(logits.data_ptr()), ctypes.c_float(scale),
                                   logits.shape[1], n_tokens, ctypes.c_void_p(Pi.data_ptr()),
                                   ctypes.c_void_p(cb.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _case(n_seq, hkv, group, T, d, bits, seed):
    dev = torch.device("cuda")
    Pi = syn.rotation(d).to(dev)
    cb = tqb.tq_codebook_fit(d, bits).to(dev)
    v = syn.lognormal_sphere((n_seq, hkv, T, d), seed, dtype=torch.bfloat16, device=dev)
    vc = tqb.PackedCache.empty(d, bits, False, n_seq, hkv, T, device=dev)
    tqb.tq_quantize_append(vc, v, 0, Pi, None, cb)
    logits = 3.0 * syn.gaussian((n_seq, hkv * group, T), seed + 1, device=dev)
    return vc, logits, Pi, cb


@pytest.mark.skipif(not cuda_ok, reason="needs a CUDA device")
def test_noalloc_matches_workspace_path_on_two_calls():
    shapes = [(1, 2, 4, 5000, 128, 3, 11), (2, 1, 3, 1200, 64, 2, 12)]
    for n_seq, hkv, group, T, d, bits, seed in shapes:
        vc, logits, Pi, cb = _case(n_seq, hkv, group, T, d, bits, seed)
        scale = 1.0 / math.sqrt(d)
        want = tqb.tq_attend_v(vc, logits, scale, T, Pi, cb)
        got = torch.full_like(want, float("nan"))
        status = _noalloc(vc, logits, scale, T, Pi, cb, got)
        assert status == tqb.TQ_OK, tqb.tq_last_error()
        st = tqb.raw_lib().tq_attend_v_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == tqb.TQ_OK, tqb.tq_last_error()
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert torch.equal(got, want), float((got - want).abs().max())


@pytest.mark.skipif(not cuda_ok, reason="needs a CUDA device")
def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 8 x 64 query heads x 131072 tokens would need ~68 MB of partials: rejected
    # before any launch. Placeholder addresses are never dereferenced; a fault is
    # armed so that a call that wrongly passed the size check returns instead.
    fake = 0x7F0000000000
    desc = tqb.TqCacheDesc(128, 3, 0, 8, 8, 0, 131072, fake, fake + 4096, None)
    need = tqb.raw_lib().tq_attend_workspace_size(ctypes.byref(desc), 64, 131072)
    assert need > (4 << 20)
    tqb.tq_debug_inject(tqb.TQ_ERR_CUDA, 1)
    try:
        st = tqb.raw_lib().tq_attend_v_noalloc(ctypes.byref(desc), fake, ctypes.c_float(0.1), 64, 131072, fake,
                                               fake, fake, None)
    finally:
        tqb.tq_debug_inject(tqb.TQ_OK, 0)
    assert st == tqb.TQ_ERR_WORKSPACE
    assert "built-in array" in tqb.tq_last_error()
