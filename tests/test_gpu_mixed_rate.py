"""GPU parity of mixed-rate caches (fractional bits per channel) against the float64 oracle.

zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5 bits per channel", title
and paragraph 2: 3.5 bits per channel keep quality, 2.5 lose a little. Read as the first
n_hi rotated coordinates at one more code bit than the rest (oracle/mixed_rate.py). Every
call goes through kv_cache_vector_quantize_b200 -> libtq.so: quantize-append, logits,
softmax.V and the one-call decode step, on ragged token counts, three dtypes, grouped
queries, d = 64 / 128 / 200, a zero vector, and appends in two parts.
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


def _books(d, beta):
    c_lo = ocb.fit_codebook(d, beta)[0]
    c_hi = ocb.fit_codebook(d, beta + 1)[0]
    return c_lo, c_hi, torch.from_numpy(np.concatenate([c_lo, c_hi])).cuda()


# (d, key beta, key n_hi, value beta, value n_hi, n_seq, kv heads, group, tokens, dtype)
SHAPES = [
    (128, 2, 64, 3, 64, 1, 2, 1, 1037, torch.bfloat16),   # 3.5 bits per channel, keys and values
    (128, 1, 64, 2, 64, 2, 1, 4, 777, torch.float16),     # 2.5 bits per channel, grouped queries
    (64, 1, 32, 3, 32, 1, 2, 2, 513, torch.float32),
    (200, 2, 96, 2, 32, 1, 1, 3, 300, torch.float32),
    (128, 3, 32, 3, 96, 1, 1, 1, 130, torch.bfloat16),    # keys with 4-bit high-group codes
    (128, 2, 64, 2, 64, 1, 2, 2, 513, torch.bfloat16),    # 3.5 / 2.5 bits: a last tile of one record
    (128, 2, 64, 2, 64, 1, 1, 2, 300, torch.bfloat16),    # odd capacity: rows not 16-byte aligned
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"d{s[0]}-k{s[1]}+{s[2]}-v{s[3]}+{s[4]}-B{s[5]}-H{s[6]}"
                                                       f"-G{s[7]}-T{s[8]}")
def test_mixed_rate_path_parity(shape):
    d, kb, km, vb, vm, B, H, G, T, dt = shape
    Pi, S = syn.rotation(d), syn.sketch(d)
    k = syn.gaussian((B, H, T, d), 71)
    k[0, 0, 5] = 0.0                                      # a zero vector: n = rho = 0, all signs 1
    k = k.to(dt)
    v = syn.lognormal_sphere((B, H, T, d), 72, dtype=dt)
    q = syn.gaussian((B, H * G, d), 73)
    ck_lo, ck_hi, ck = _books(d, kb)
    cv_lo, cv_hi, cv = _books(d, vb)
    Pig, Sg = Pi.cuda(), S.cuda()
    SPiT = tqb.tq_sketch_rotation(Pig, Sg)
    cap = T + 5
    kc = tqb.PackedCache.empty(d, kb, True, B, H, cap, n_hi=km)
    vc = tqb.PackedCache.empty(d, vb, False, B, H, cap, n_hi=vm)
    # keys appended in two parts (slots [0, 100) then [100, T)), values in one
    kg = k.cuda()
    tqb.tq_quantize_append(kc, kg[:, :, :100].contiguous(), 0, Pig, SPiT, ck)
    tqb.tq_quantize_append(kc, kg[:, :, 100:].contiguous(), 100, Pig, SPiT, ck)
    tqb.tq_quantize_append(vc, v.cuda(), 0, Pig, None, cv)
    lg = tqb.tq_logits(kc, q.cuda(), T, Pig, Sg, ck)
    sc = 1.0 / math.sqrt(d)
    out = tqb.tq_attend_v(vc, lg, sc, T, Pig, cv)
    out_d = tqb.tq_decode_attend(kc, vc, q.cuda(), T, sc, Pig, Sg, ck, cv)
    torch.cuda.synchronize()
    assert torch.equal(out_d, out)
    Pn, Sn = Pi.numpy(), S.numpy()
    krec, vrec = par.as_u32(kc.records.cpu().numpy()), par.as_u32(vc.records.cpu().numpy())
    kn, kr, vn = kc.norm.cpu().numpy(), kc.rnorm.cpu().numpy(), vc.norm.cpu().numpy()
    lg_np, out_np, qn = lg.cpu().numpy(), out.cpu().numpy(), q.numpy().astype(np.float64)
    kx, vx = k.float().numpy().astype(np.float64), v.float().numpy().astype(np.float64)
    for s_ in range(B):
        for h in range(H):
            par.check_encoding_mixed(kx[s_, h], krec[s_, h, :T], kn[s_, h, :T], kr[s_, h, :T], Pn, Sn, ck_lo, ck_hi,
                                     d, kb, km, True)
            par.check_encoding_mixed(vx[s_, h], vrec[s_, h, :T], vn[s_, h, :T], None, Pn, None, cv_lo, cv_hi, d, vb,
                                     vm, False)
            rows = slice(h * G, (h + 1) * G)
            par.check_logits_mixed(lg_np[s_, rows], qn[s_, rows], Pn, Sn, ck_lo, ck_hi, krec[s_, h, :T],
                                   kn[s_, h, :T], kr[s_, h, :T], d, kb, km)
            par.check_attend_mixed(out_np[s_, rows], lg_np[s_, rows].astype(np.float64), sc, Pn, cv_lo, cv_hi,
                                   vrec[s_, h, :T], vn[s_, h, :T], d, vb, vm)
    # slots past T were never written
    assert not kc.records[:, :, T:].any() and not vc.records[:, :, T:].any()


def test_mixed_rate_bsweep_full_size_sampled():
    # the b-sweep shape at 3.5 bits per channel (keys 2.5 code bits + QJL, values 3.5 code
    # bits): 8 x 8 KV heads x 131072 tokens, bf16 lognormal norms; sampled rows and heads
    B, H, T, d = 8, 8, 131072, 128
    k, v, q = syn.sweep_inputs(device="cuda")
    Pi, S = syn.rotation(d), syn.sketch(d)
    ck_lo, ck_hi, ck = _books(d, 2)
    cv_lo, cv_hi, cv = _books(d, 3)
    Pig, Sg = Pi.cuda(), S.cuda()
    SPiT = tqb.tq_sketch_rotation(Pig, Sg)
    kc = tqb.PackedCache.empty(d, 2, True, B, H, T, n_hi=64)
    vc = tqb.PackedCache.empty(d, 3, False, B, H, T, n_hi=64)
    tqb.tq_quantize_append(kc, k, 0, Pig, SPiT, ck)
    tqb.tq_quantize_append(vc, v, 0, Pig, None, cv)
    ws_l = torch.empty(tqb.tq_logits_workspace_size(kc, H), dtype=torch.uint8, device="cuda")
    ws_a = torch.empty(tqb.tq_attend_workspace_size(vc, H, T), dtype=torch.uint8, device="cuda")
    lg = tqb.tq_logits(kc, q, T, Pig, Sg, ck, workspace=ws_l)
    sc = 1.0 / math.sqrt(d)
    out = tqb.tq_attend_v(vc, lg, sc, T, Pig, cv, workspace=ws_a)
    torch.cuda.synchronize()
    tqb.tq_workspace_status(ws_l)
    tqb.tq_workspace_status(ws_a)
    Pn, Sn = Pi.numpy(), S.numpy()
    rng = np.random.default_rng(135)
    for _ in range(3):
        s_, h = int(rng.integers(B)), int(rng.integers(H))
        rows = np.sort(rng.choice(T, size=512, replace=False))
        idx = torch.from_numpy(rows).cuda()
        krec = par.as_u32(kc.records[s_, h].index_select(0, idx).cpu().numpy())
        kn = kc.norm[s_, h].index_select(0, idx).cpu().numpy()
        kr = kc.rnorm[s_, h].index_select(0, idx).cpu().numpy()
        par.check_encoding_mixed(k[s_, h].index_select(0, idx).float().cpu().numpy(), krec, kn, kr, Pn, Sn, ck_lo,
                                 ck_hi, d, 2, 64, True)
        par.check_encoding_mixed(v[s_, h].index_select(0, idx).float().cpu().numpy(),
                                 par.as_u32(vc.records[s_, h].index_select(0, idx).cpu().numpy()),
                                 vc.norm[s_, h].index_select(0, idx).cpu().numpy(), None, Pn, None, cv_lo, cv_hi, d,
                                 3, 64, False)
        par.check_logits_mixed(lg[s_, h].index_select(0, idx).cpu().numpy()[None, :],
                               q[s_, h].cpu().numpy()[None, :].astype(np.float64), Pn, Sn, ck_lo, ck_hi, krec, kn, kr,
                               d, 2, 64)
        par.check_attend_mixed(out[s_, h:h + 1].cpu().numpy(), lg[s_, h:h + 1].cpu().numpy().astype(np.float64), sc,
                               Pn, cv_lo, cv_hi, par.as_u32(vc.records[s_, h].cpu().numpy()),
                               vc.norm[s_, h].cpu().numpy(), d, 3, 64)
    assert torch.isfinite(lg).all() and torch.isfinite(out).all()
