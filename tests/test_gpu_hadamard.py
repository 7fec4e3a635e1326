"""GPU parity of the structured-rotation quantizer (tq_quantize_append_hadamard) against the oracle.

winningdata.io, "TurboQuant: Google comprime KV cache para 3 bits sem perder acuracia", "1. PolarQuant"
prices the rotation per vector; with Pi = H diag(s) / sqrt(d) (H Sylvester-Hadamard) the library applies it
by a fast Walsh-Hadamard transform. The encoding must be the oracle's with the dense Pi of the same
rotation, and logits, softmax.V and the one-call decode step read the cache with that dense Pi. Shapes:
every supported d (32, 64, 128, 256), keys and values, three dtypes, ragged token counts, a zero vector,
a mixed-rate cache, and a check that the dense-Pi call encodes the same cache (up to excused flips).
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


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok:
        pytest.skip("needs a CUDA device")


# (d, key code bits, value code bits, n_seq, kv heads, group, tokens, dtype)
SHAPES = [
    (32, 1, 2, 1, 2, 1, 301, torch.float32),
    (64, 2, 3, 2, 1, 2, 130, torch.bfloat16),
    (128, 2, 3, 1, 2, 4, 777, torch.bfloat16),
    (128, 3, 4, 1, 1, 1, 257, torch.float16),
    (256, 2, 2, 1, 1, 2, 513, torch.float32),
    (256, 1, 3, 1, 2, 1, 129, torch.bfloat16),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"d{s[0]}-kb{s[1]}-vb{s[2]}-B{s[3]}-H{s[4]}-G{s[5]}-T{s[6]}")
def test_hadamard_quantize_path_parity(shape):
    d, kb, vb, B, H, G, T, dt = shape
    k = syn.gaussian((B, H, T, d), 61 + d)
    k[0, 0, 3] = 0.0                                      # a zero vector
    k = k.to(dt)
    v = syn.lognormal_sphere((B, H, T, d), 62 + d, dtype=dt)
    q = syn.gaussian((B, H * G, d), 63 + d)
    Pi, S, signs = syn.randomized_hadamard(d), syn.sketch(d), syn.hadamard_signs(d)
    ck, cv = ocb.fit_codebook(d, kb)[0], ocb.fit_codebook(d, vb)[0]
    dev = torch.device("cuda")
    Pig, Sg, sg = Pi.to(dev), S.to(dev), signs.to(dev)
    ckg, cvg = torch.from_numpy(ck).to(dev), torch.from_numpy(cv).to(dev)
    SPiT = tqb.tq_sketch_rotation(Pig, Sg)
    cap = T + 3
    kc = tqb.PackedCache.empty(d, kb, True, B, H, cap)
    vc = tqb.PackedCache.empty(d, vb, False, B, H, cap)
    tqb.tq_quantize_append_hadamard(kc, k.cuda(), 0, sg, SPiT, ckg)
    tqb.tq_quantize_append_hadamard(vc, v.cuda(), 0, sg, None, cvg)
    lg = tqb.tq_logits(kc, q.cuda(), T, Pig, Sg, ckg)
    sc = 1.0 / math.sqrt(d)
    out = tqb.tq_attend_v(vc, lg, sc, T, Pig, cvg)
    out_d = tqb.tq_decode_attend(kc, vc, q.cuda(), T, sc, Pig, Sg, ckg, cvg)
    # the dense-Pi quantizer on the same input
    kd = tqb.PackedCache.empty(d, kb, True, B, H, cap)
    tqb.tq_quantize_append(kd, k.cuda(), 0, Pig, SPiT, ckg)
    torch.cuda.synchronize()
    assert torch.equal(out_d, out)
    Pn, Sn = Pi.numpy(), S.numpy()
    krec, vrec = par.as_u32(kc.records.cpu().numpy()), par.as_u32(vc.records.cpu().numpy())
    kn, kr, vn = kc.norm.cpu().numpy(), kc.rnorm.cpu().numpy(), vc.norm.cpu().numpy()
    lg_np, out_np, qn = lg.cpu().numpy(), out.cpu().numpy(), q.numpy().astype(np.float64)
    kx, vx = k.float().numpy().astype(np.float64), v.float().numpy().astype(np.float64)
    for s_ in range(B):
        for h in range(H):
            par.check_encoding(kx[s_, h], krec[s_, h, :T], kn[s_, h, :T], kr[s_, h, :T], Pn, Sn, ck, d, kb, True)
            par.check_encoding(vx[s_, h], vrec[s_, h, :T], vn[s_, h, :T], None, Pn, None, cv, d, vb, False)
            rows = slice(h * G, (h + 1) * G)
            par.check_logits(lg_np[s_, rows], qn[s_, rows], Pn, Sn, ck, krec[s_, h, :T], kn[s_, h, :T],
                             kr[s_, h, :T], d, kb)
            par.check_attend(out_np[s_, rows], lg_np[s_, rows].astype(np.float64), sc, Pn, cv, vrec[s_, h, :T],
                             vn[s_, h, :T], d, vb)
    # the two rotation paths: the same norms to the parity tolerance and codes except a few rounding
    # flips at thresholds (each path is held to the oracle above)
    assert torch.allclose(kc.norm, kd.norm, rtol=1e-5, atol=0)
    differ = (kc.records != kd.records).any(dim=-1).float().mean().item()
    assert differ <= 0.02, differ
    assert not kc.records[:, :, T:].any() and not vc.records[:, :, T:].any()


def test_hadamard_quantize_mixed_rate():
    # 3.5 bits per channel at d = 128: the first 64 rotated coordinates one code bit wider
    d, kb, vb, T = 128, 2, 3, 300
    k = syn.gaussian((1, 1, T, d), 71).to(torch.bfloat16)
    v = syn.lognormal_sphere((1, 1, T, d), 72, dtype=torch.bfloat16)
    Pi, S, signs = syn.randomized_hadamard(d), syn.sketch(d), syn.hadamard_signs(d)
    books = {b: (ocb.fit_codebook(d, b)[0], ocb.fit_codebook(d, b + 1)[0]) for b in (kb, vb)}
    dev = torch.device("cuda")
    Pig, Sg, sg = Pi.to(dev), S.to(dev), signs.to(dev)
    SPiT = tqb.tq_sketch_rotation(Pig, Sg)
    kc = tqb.PackedCache.empty(d, kb, True, 1, 1, T, n_hi=64)
    vc = tqb.PackedCache.empty(d, vb, False, 1, 1, T, n_hi=64)
    tqb.tq_quantize_append_hadamard(kc, k.cuda(), 0, sg, SPiT, torch.from_numpy(np.concatenate(books[kb])).to(dev))
    tqb.tq_quantize_append_hadamard(vc, v.cuda(), 0, sg, None, torch.from_numpy(np.concatenate(books[vb])).to(dev))
    torch.cuda.synchronize()
    Pn, Sn = Pi.numpy(), S.numpy()
    par.check_encoding_mixed(k[0, 0].float().numpy().astype(np.float64), par.as_u32(kc.records[0, 0].cpu().numpy()),
                             kc.norm[0, 0].cpu().numpy(), kc.rnorm[0, 0].cpu().numpy(), Pn, Sn, *books[kb], d, kb, 64,
                             True)
    par.check_encoding_mixed(v[0, 0].float().numpy().astype(np.float64), par.as_u32(vc.records[0, 0].cpu().numpy()),
                             vc.norm[0, 0].cpu().numpy(), None, Pn, None, *books[vb], d, vb, 64, False)


def test_hadamard_rejects_other_d():
    d = 200
    c = tqb.PackedCache.empty(d, 2, False, 1, 1, 8)
    with pytest.raises(tqb.TQError) as e:
        tqb.tq_quantize_append_hadamard(c, torch.zeros((1, 1, 8, d), device="cuda"), 0,
                                        torch.ones(d, device="cuda"), None,
                                        torch.from_numpy(ocb.fit_codebook(d, 2)[0]).cuda())
    assert e.value.status == tqb.TQ_ERR_UNSUPPORTED
