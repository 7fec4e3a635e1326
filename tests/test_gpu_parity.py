"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small and ragged shapes are compared element by element; the full-size
workloads (the Llama-3-8B-shaped decode that bench.py times, and the b-sweep
caches) are compared on sampled rows and keys plus properties that hold at
any size. Every call goes through kv_cache_vector_quantize_b200 -> libtq.so.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import tq_synth as syn
from oracle import codebook as ocb
from oracle import turboquant as otq
from tests import _parity as par

pytestmark = pytest.mark.gpu

cuda_ok = torch.cuda.is_available()
if cuda_ok:
    import kv_cache_vector_quantize_b200 as tqb


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok:
        pytest.skip("needs a CUDA device")


def _codebook(d, bits):
    return ocb.fit_codebook(d, bits)[0]          # float32 centroids the oracle also uses


def _setup(d, k_idx_bits, v_bits):
    Pi = syn.rotation(d)
    S = syn.sketch(d)
    ck = _codebook(d, k_idx_bits)
    cv = _codebook(d, v_bits)
    dev = torch.device("cuda")
    g = dict(Pi=Pi.to(dev), S=S.to(dev), ck=torch.from_numpy(ck).to(dev), cv=torch.from_numpy(cv).to(dev))
    g["SPiT"] = tqb.tq_sketch_rotation(g["Pi"], g["S"])
    return Pi.numpy(), S.numpy(), ck, cv, g


def _run_path(k, v, q, d, k_idx_bits, v_bits, g, capacity=None, scale=None):
    """Quantize K and V, then logits and softmax.V. Returns GPU tensors."""
    n_seq, hkv, T, _ = k.shape
    cap = T if capacity is None else capacity
    kc = tqb.PackedCache.empty(d, k_idx_bits, True, n_seq, hkv, cap)
    vc = tqb.PackedCache.empty(d, v_bits, False, n_seq, hkv, cap)
    tqb.tq_quantize_append(kc, k.cuda(), 0, g["Pi"], g["SPiT"], g["ck"])
    tqb.tq_quantize_append(vc, v.cuda(), 0, g["Pi"], None, g["cv"])
    ws_l = torch.empty(max(256, tqb.tq_logits_workspace_size(kc, q.shape[1])), dtype=torch.uint8, device="cuda")
    ws_a = torch.empty(max(256, tqb.tq_attend_workspace_size(vc, q.shape[1], T)), dtype=torch.uint8, device="cuda")
    lg = tqb.tq_logits(kc, q.cuda(), T, g["Pi"], g["S"], g["ck"], workspace=ws_l)
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    out = tqb.tq_attend_v(vc, lg, sc, T, g["Pi"], g["cv"], workspace=ws_a)
    torch.cuda.synchronize()
    if T > 0:
        tqb.tq_workspace_status(ws_l)
        tqb.tq_workspace_status(ws_a)
    return kc, vc, lg, out, sc


def _check_all(k, v, q, d, k_idx_bits, v_bits, Pi, S, ck, cv, kc, vc, lg, out, sc, rows=None):
    n_seq, hkv, T, _ = k.shape
    hq = q.shape[1]
    G = hq // hkv
    kx = k.float().numpy().astype(np.float64)
    vx = v.float().numpy().astype(np.float64)
    krec = par.as_u32(kc.records.cpu().numpy())
    vrec = par.as_u32(vc.records.cpu().numpy())
    kn, kr, vn = kc.norm.cpu().numpy(), kc.rnorm.cpu().numpy(), vc.norm.cpu().numpy()
    lg_np, out_np, qn = lg.cpu().numpy(), out.cpu().numpy(), q.numpy().astype(np.float64)
    stats = {"index_flips": 0, "sign_flips": 0, "coords": 0}
    for s in range(n_seq):
        for h in range(hkv):
            sel = slice(None) if rows is None else rows
            ek = par.check_encoding(kx[s, h, :T][sel], krec[s, h, :T][sel], kn[s, h, :T][sel], kr[s, h, :T][sel],
                                    Pi, S, ck, d, k_idx_bits, True)
            ev = par.check_encoding(vx[s, h, :T][sel], vrec[s, h, :T][sel], vn[s, h, :T][sel], None,
                                    Pi, None, cv, d, v_bits, False)
            for e in (ek, ev):
                for key in stats:
                    stats[key] += e[key]
            qs = qn[s, h * G:(h + 1) * G]
            par.check_logits(lg_np[s, h * G:(h + 1) * G], qs, Pi, S, ck, krec[s, h, :T], kn[s, h, :T],
                             kr[s, h, :T], d, k_idx_bits)
            par.check_attend(out_np[s, h * G:(h + 1) * G], lg_np[s, h * G:(h + 1) * G].astype(np.float64), sc, Pi,
                             cv, vrec[s, h, :T], vn[s, h, :T], d, v_bits)
    return stats


def test_sketch_rotation_matches_float64_product():
    d = 128
    Pi, S = syn.rotation(d), syn.sketch(d)
    got = tqb.tq_sketch_rotation(Pi.cuda(), S.cuda()).cpu().numpy()
    want = S.double().numpy() @ Pi.double().numpy().T
    assert np.allclose(got, want, rtol=0, atol=2e-6 * np.abs(want).max())


def test_pr1_parity():
    # d=128, 4096 keys fp32 N(0,1) seed 0, 16 queries; b=3 keys (2-bit codebook + QJL);
    # values of the same law at 3 bits MSE-only.
    k, v, q = syn.pr1_inputs()
    Pi, S, ck, cv, g = _setup(128, 2, 3)
    kc, vc, lg, out, sc = _run_path(k, v, q, 128, 2, 3, g)
    stats = _check_all(k, v, q, 128, 2, 3, Pi, S, ck, cv, kc, vc, lg, out, sc)
    assert stats["index_flips"] + stats["sign_flips"] <= 1e-4 * stats["coords"]


SHAPES = [
    # d, k index bits, v bits, n_seq, kv heads, group, tokens, dtype
    (8, 1, 2, 2, 3, 2, 301, torch.float32),
    (200, 2, 3, 1, 2, 4, 1037, torch.bfloat16),
    (128, 3, 4, 2, 2, 1, 777, torch.float16),
    (64, 2, 1, 1, 1, 8, 129, torch.bfloat16),
    (256, 3, 4, 1, 1, 2, 300, torch.bfloat16),
    (128, 1, 2, 1, 2, 4, 1, torch.float32),
    (96, 2, 2, 3, 1, 3, 513, torch.float32),
    # bf16 heads of 128 take the tensor-core quantizer: ragged tails, all code widths
    (128, 3, 4, 2, 2, 1, 901, torch.bfloat16),
    (128, 1, 2, 1, 3, 2, 130, torch.bfloat16),
    (128, 2, 1, 1, 1, 4, 257, torch.bfloat16),
    # grouped queries on 1-/2-bit codes take the float16-table scan: 2, 4 and 8 heads per KV head,
    # several 512-key tiles with a ragged tail, more units than one CTA each
    (128, 2, 3, 2, 1, 8, 1100, torch.bfloat16),
    (128, 2, 2, 3, 2, 2, 1537, torch.bfloat16),
    (128, 1, 3, 1, 4, 4, 2049, torch.float16),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"d{s[0]}-kb{s[1]}-vb{s[2]}-B{s[3]}-H{s[4]}-G{s[5]}-T{s[6]}")
def test_shapes_parity(shape):
    d, kb, vb, B, H, G, T, dt = shape
    k = syn.gaussian((B, H, T, d), 10 + d).to(dt)
    v = syn.lognormal_sphere((B, H, T, d), 20 + d, dtype=dt)
    q = syn.gaussian((B, H * G, d), 30 + d)
    Pi, S, ck, cv, g = _setup(d, kb, vb)
    kc, vc, lg, out, sc = _run_path(k, v, q, d, kb, vb, g, capacity=T + 5)
    _check_all(k, v, q, d, kb, vb, Pi, S, ck, cv, kc, vc, lg, out, sc)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_structured_rotation_full_path(dt):
    # a randomized Hadamard rotation H diag(s) / sqrt(d) as the rotation input: quantize (tensor-core
    # path for bf16, FP32 path for fp32), logits, softmax.V and the one-call decode step against the
    # oracle on the same matrix
    d, kb, vb, B, H, G, T = 128, 2, 3, 1, 2, 4, 777
    k = syn.gaussian((B, H, T, d), 51).to(dt)
    v = syn.lognormal_sphere((B, H, T, d), 52, dtype=dt)
    q = syn.gaussian((B, H * G, d), 53)
    Pi_t, S_t = syn.randomized_hadamard(d), syn.sketch(d)
    ck, cv = _codebook(d, kb), _codebook(d, vb)
    dev = torch.device("cuda")
    g = dict(Pi=Pi_t.to(dev), S=S_t.to(dev), ck=torch.from_numpy(ck).to(dev), cv=torch.from_numpy(cv).to(dev))
    g["SPiT"] = tqb.tq_sketch_rotation(g["Pi"], g["S"])
    kc, vc, lg, out, sc = _run_path(k, v, q, d, kb, vb, g)
    _check_all(k, v, q, d, kb, vb, Pi_t.numpy(), S_t.numpy(), ck, cv, kc, vc, lg, out, sc)
    out_d = tqb.tq_decode_attend(kc, vc, q.cuda(), T, sc, g["Pi"], g["S"], g["ck"], g["cv"])
    torch.cuda.synchronize()
    assert torch.equal(out_d, out)


def test_append_in_parts_equals_one_call():
    d, kb, T = 128, 2, 700
    k = syn.gaussian((2, 2, T, d), 41).to(torch.bfloat16).cuda()
    _, _, _, _, g = _setup(d, kb, 3)
    one = tqb.PackedCache.empty(d, kb, True, 2, 2, T)
    parts = tqb.PackedCache.empty(d, kb, True, 2, 2, T)
    tqb.tq_quantize_append(one, k, 0, g["Pi"], g["SPiT"], g["ck"])
    for a, b in ((0, 65), (65, 66), (66, 640), (640, 700)):
        tqb.tq_quantize_append(parts, k[:, :, a:b].contiguous(), a, g["Pi"], g["SPiT"], g["ck"])
    torch.cuda.synchronize()
    assert torch.equal(one.records, parts.records)
    assert torch.equal(one.norm, parts.norm) and torch.equal(one.rnorm, parts.rnorm)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_special_vectors(dtype):
    # zero vectors, codeword directions, tiny and huge norms (bf16 and fp16: the tensor-core path;
    # fp16 keeps its tiny and huge rows inside its own range)
    d, kb = 128, 2
    tiny, huge = (1e-3, 1e3) if dtype == torch.float16 else (1e-20, 1e20)
    Pi, S, ck, cv, g = _setup(d, kb, 3)
    rng = np.random.default_rng(5)
    rows = [np.zeros(d)]
    c = ck.astype(np.float64)
    for a in range(5):
        w = c[rng.integers(0, 4, size=d)]
        rows.append(3.0 * (w @ Pi.astype(np.float64)) / np.linalg.norm(w))
    rows += [tiny * rng.standard_normal(d), huge * rng.standard_normal(d), np.ones(d), -np.ones(d)]
    x = torch.tensor(np.array(rows), dtype=torch.float32).reshape(1, 1, -1, d).to(dtype)
    kc = tqb.PackedCache.empty(d, kb, True, 1, 1, x.shape[2])
    tqb.tq_quantize_append(kc, x.cuda(), 0, g["Pi"], g["SPiT"], g["ck"])
    torch.cuda.synchronize()
    rec = par.as_u32(kc.records.cpu().numpy())[0, 0]
    par.check_encoding(x[0, 0].double().numpy(), rec, kc.norm.cpu().numpy()[0, 0], kc.rnorm.cpu().numpy()[0, 0],
                       Pi, S, ck, d, kb, True)
    gi, gs = otq.unpack(rec, d, kb, True)
    assert kc.norm[0, 0, 0].item() == 0 and kc.rnorm[0, 0, 0].item() == 0 and gs[0].all()


def test_empty_inputs():
    d = 64
    _, _, _, _, g = _setup(d, 2, 2)
    kc = tqb.PackedCache.empty(d, 2, True, 1, 2, 16)
    vc = tqb.PackedCache.empty(d, 2, False, 1, 2, 16)
    tqb.tq_quantize_append(kc, torch.empty((1, 2, 0, d), device="cuda"), 3, g["Pi"], g["SPiT"], g["ck"])
    lg = tqb.tq_logits(kc, torch.randn(1, 4, d, device="cuda"), 0, g["Pi"], g["S"], g["ck"])
    out = torch.full((1, 4, d), 7.0, device="cuda")
    tqb.tq_attend_v(vc, lg, 0.125, 0, g["Pi"], g["cv"], out=out)
    torch.cuda.synchronize()
    assert lg.numel() == 0 and torch.all(out == 0)
    assert torch.all(kc.records == 0)


def test_errors_reported_without_launch():
    d = 64
    _, _, _, _, g = _setup(d, 2, 2)
    kc = tqb.PackedCache.empty(d, 2, True, 1, 1, 8)
    with pytest.raises(tqb.TQError) as e:
        tqb.tq_quantize_append(kc, torch.zeros((1, 1, 9, d), device="cuda"), 0, g["Pi"], g["SPiT"], g["ck"])
    assert e.value.status == tqb.TQ_ERR_CAPACITY
    with pytest.raises(tqb.TQError) as e:
        tqb.tq_logits(kc, torch.zeros((1, 1, d), device="cuda"), 9, g["Pi"], g["S"], g["ck"])
    assert e.value.status == tqb.TQ_ERR_CAPACITY
    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(tqb.TQError) as e:
        tqb.tq_logits(kc, torch.zeros((1, 1, d), device="cuda"), 4, g["Pi"], g["S"], g["ck"], workspace=ws)
    assert e.value.status == tqb.TQ_ERR_WORKSPACE
    assert torch.all(kc.records == 0)


def test_workspace_status_clean_after_calls():
    d = 128
    _, _, _, _, g = _setup(d, 2, 3)
    kc = tqb.PackedCache.empty(d, 2, True, 1, 1, 256)
    tqb.tq_quantize_append(kc, torch.randn(1, 1, 256, d, device="cuda"), 0, g["Pi"], g["SPiT"], g["ck"])
    ws = torch.empty(tqb.tq_logits_workspace_size(kc, 2), dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)   # the call must clear the status word itself
    tqb.tq_logits(kc, torch.randn(1, 2, d, device="cuda"), 256, g["Pi"], g["S"], g["ck"], workspace=ws)
    tqb.tq_workspace_status(ws)


@pytest.mark.parametrize("kb,G", [(3, 1), (2, 1), (3, 2), (2, 2), (1, 4)])
def test_logits_unaligned_query_and_matrices(kb, G):
    # q, Pi and S 4 bytes off a 16-byte boundary: the scans that read them as float4 (the
    # single-head scan projecting its own queries, the float16-table scan) leave the projection
    # to a kernel of its own; both layouts must give the oracle's logits
    d, T, H = 128, 1100, 2
    Pi, S, ck, cv, g = _setup(d, kb, 3)
    k = syn.gaussian((1, H, T, d), 51).to(torch.bfloat16)
    q = syn.gaussian((1, H * G, d), 52)
    kc = tqb.PackedCache.empty(d, kb, True, 1, H, T)
    tqb.tq_quantize_append(kc, k.cuda(), 0, g["Pi"], g["SPiT"], g["ck"])

    def shifted(t):
        buf = torch.empty(t.numel() + 1, dtype=t.dtype, device="cuda")
        buf[1:] = t.reshape(-1)
        return buf[1:].view(t.shape)

    qd = q.cuda()
    runs = [(qd, g["Pi"], g["S"]), (shifted(qd), shifted(g["Pi"]), shifted(g["S"]))]
    assert runs[1][0].data_ptr() % 16 == 4
    krec = par.as_u32(kc.records.cpu().numpy())
    kn, kr = kc.norm.cpu().numpy(), kc.rnorm.cpu().numpy()
    qn = q.numpy().astype(np.float64)
    for qq, pi, sk in runs:
        ws = torch.empty(max(256, tqb.tq_logits_workspace_size(kc, H * G)), dtype=torch.uint8, device="cuda")
        ws.fill_(0xFF)
        lg = tqb.tq_logits(kc, qq, T, pi, sk, g["ck"], workspace=ws)
        torch.cuda.synchronize()
        tqb.tq_workspace_status(ws)
        lg_np = lg.cpu().numpy()
        for h in range(H):
            par.check_logits(lg_np[0, h * G:(h + 1) * G], qn[0, h * G:(h + 1) * G], Pi, S, ck, krec[0, h],
                             kn[0, h], kr[0, h], d, kb)


DECODE_SHAPES = [
    # k index bits, v bits, n_seq, kv heads, group, tokens: one query head per KV head takes the fused
    # pass (1- or 2-bit key codes), 2 / 4 / 8 query heads per KV head the fused grouped-query pass
    # (1- or 2-bit key codes, 1..3-bit value codes), every other shape the two calls inside the same
    # entry point
    (2, 3, 2, 3, 1, 1537),
    (1, 2, 1, 2, 1, 777),
    (2, 4, 1, 1, 1, 4096),
    (2, 1, 3, 1, 1, 130),
    (3, 3, 1, 2, 1, 901),
    (2, 3, 1, 2, 4, 1100),
    (1, 2, 2, 2, 2, 777),
    (2, 3, 1, 2, 8, 1537),
    (2, 1, 1, 3, 4, 130),
    (2, 2, 2, 1, 4, 5000),
    (1, 3, 1, 1, 2, 257),
    (2, 4, 1, 1, 4, 600),
]


@pytest.mark.parametrize("shape", DECODE_SHAPES, ids=lambda s: f"kb{s[0]}-vb{s[1]}-B{s[2]}-H{s[3]}-G{s[4]}-T{s[5]}")
def test_decode_attend_parity(shape):
    # the one-call decode step equals tq_logits followed by tq_attend_v bit for bit (same tables,
    # chunks and accumulation order), and that output matches the oracle's softmax.V of those logits
    kb, vb, B, H, G, T = shape
    d = 128
    k = syn.gaussian((B, H, T, d), 61).to(torch.bfloat16)
    v = syn.lognormal_sphere((B, H, T, d), 62, dtype=torch.bfloat16)
    q = syn.gaussian((B, H * G, d), 63)
    Pi, S, ck, cv, g = _setup(d, kb, vb)
    kc, vc, lg, out2, sc = _run_path(k, v, q, d, kb, vb, g, capacity=T + 3)
    ws = torch.empty(max(256, tqb.tq_decode_workspace_size(kc, vc, H * G, T)), dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)   # the call must clear the status word itself
    out1 = tqb.tq_decode_attend(kc, vc, q.cuda(), T, sc, g["Pi"], g["S"], g["ck"], g["cv"], workspace=ws)
    torch.cuda.synchronize()
    tqb.tq_workspace_status(ws)
    assert torch.equal(out1, out2)
    vrec = par.as_u32(vc.records.cpu().numpy())
    vn = vc.norm.cpu().numpy()
    lg_np, o1 = lg.cpu().numpy().astype(np.float64), out1.cpu().numpy()
    for s_ in range(B):
        for h in range(H):
            par.check_attend(o1[s_, h * G:(h + 1) * G], lg_np[s_, h * G:(h + 1) * G], sc, Pi, cv, vrec[s_, h, :T],
                             vn[s_, h, :T], d, vb)


def test_decode_attend_caches_of_different_capacity():
    # key and value caches sized differently (each indexed with its own capacity); the step equals
    # the two calls on the same caches
    d, B, H, T = 128, 2, 2, 1000
    k = syn.gaussian((B, H, T, d), 71).to(torch.bfloat16).cuda()
    v = syn.lognormal_sphere((B, H, T, d), 72, dtype=torch.bfloat16).cuda()
    q = syn.gaussian((B, H, d), 73).cuda()
    _, _, _, _, g = _setup(d, 2, 3)
    kc = tqb.PackedCache.empty(d, 2, True, B, H, T + 37)
    vc = tqb.PackedCache.empty(d, 3, False, B, H, T + 1029)
    tqb.tq_quantize_append(kc, k, 0, g["Pi"], g["SPiT"], g["ck"])
    tqb.tq_quantize_append(vc, v, 0, g["Pi"], None, g["cv"])
    sc = 1.0 / math.sqrt(d)
    for G in (1, 4):   # the single-head and the grouped-query fused passes
        qg = syn.gaussian((B, H * G, d), 74 + G).cuda()
        lg = tqb.tq_logits(kc, qg, T, g["Pi"], g["S"], g["ck"])
        out2 = tqb.tq_attend_v(vc, lg, sc, T, g["Pi"], g["cv"])
        ws = torch.empty(max(256, tqb.tq_decode_workspace_size(kc, vc, H * G, T)), dtype=torch.uint8, device="cuda")
        out1 = tqb.tq_decode_attend(kc, vc, qg, T, sc, g["Pi"], g["S"], g["ck"], g["cv"], workspace=ws)
        torch.cuda.synchronize()
        tqb.tq_workspace_status(ws)
        assert torch.equal(out1, out2), G
    del q


# ---------------------------------------------------------------------------
# nearest-neighbour search (top-k of the key estimator over one database stream)
# ---------------------------------------------------------------------------

def _nn_case(d, bits, n_db, n_q, k, capacity=None):
    db, qs = syn.nn_inputs(n_db, n_q, d)
    Pi, S, ck, _, g = _setup(d, bits, 1)
    cache = tqb.PackedCache.empty(d, bits, True, 1, 1, capacity or max(n_db, 1))
    if n_db:
        tqb.tq_quantize_append(cache, db.reshape(1, 1, n_db, d).cuda(), 0, g["Pi"], g["SPiT"], g["ck"])
    ws = torch.empty(max(256, tqb.tq_nn_workspace_size(cache, n_q, n_db)), dtype=torch.uint8, device="cuda")
    sc, ids = tqb.tq_nn_search(cache, qs.cuda(), n_db, g["Pi"], g["S"], g["ck"], k, workspace=ws)
    torch.cuda.synchronize()
    tqb.tq_workspace_status(ws)
    rec = par.as_u32(cache.records[0, 0, :n_db].cpu().numpy())
    norm = cache.norm[0, 0, :n_db].cpu().numpy()
    rnorm = cache.rnorm[0, 0, :n_db].cpu().numpy()
    return db, qs, Pi, S, ck, rec, norm, rnorm, sc.cpu().numpy(), ids.cpu().numpy()


@pytest.mark.parametrize("d,bits,n_db,n_q,k", [
    (200, 1, 5000, 300, 10),     # 40 tiles (ragged 8), 3 query blocks (ragged 44): one unit per CTA
    (200, 3, 5000, 300, 10),
    (200, 1, 40000, 300, 10),    # 313 tiles x 3 blocks over the SMs: CTA ranges cross query blocks
    (200, 3, 40000, 130, 16),
    (200, 2, 20000, 257, 1),
    (128, 2, 9000, 200, 7),
    (128, 1, 3000, 1, 16),
])
def test_nn_search_parity(d, bits, n_db, n_q, k):
    db, qs, Pi, S, ck, rec, norm, rnorm, sc, ids = _nn_case(d, bits, n_db, n_q, k)
    par.check_encoding(db.numpy(), rec, norm, rnorm, Pi, S, ck, d, bits, True)
    par.check_nn(sc, ids, qs.numpy(), Pi, S, ck, rec, norm, rnorm, d, bits, k)


@pytest.mark.parametrize("bits", [1, 3])
def test_nn_search_full_size_sampled(bits):
    # the nearest-neighbour workload bench.py times (10^6 x d = 200 database, 10^4 queries, top-10):
    # the encoding on 20000 sampled database rows, the top-10 of 12 sampled queries over all rows
    d, N, Q, k = 200, 1_000_000, 10_000, 10
    db, qs = syn.nn_inputs(N, Q, d, device="cuda")
    Pi, S, ck, _, g = _setup(d, bits, 1)
    cache = tqb.PackedCache.empty(d, bits, True, 1, 1, N)
    tqb.tq_quantize_append(cache, db.reshape(1, 1, N, d), 0, g["Pi"], g["SPiT"], g["ck"])
    ws = torch.empty(tqb.tq_nn_workspace_size(cache, Q, N), dtype=torch.uint8, device="cuda")
    sc, ids = tqb.tq_nn_search(cache, qs, N, g["Pi"], g["S"], g["ck"], k, workspace=ws)
    torch.cuda.synchronize()
    tqb.tq_workspace_status(ws)
    rec = par.as_u32(cache.records[0, 0].cpu().numpy())
    norm = cache.norm[0, 0].cpu().numpy()
    rnorm = cache.rnorm[0, 0].cpu().numpy()
    rows = np.random.default_rng(3).choice(N, 20000, replace=False)
    par.check_encoding(db[rows].cpu().numpy(), rec[rows], norm[rows], rnorm[rows], Pi, S, ck, d, bits, True)
    qi = np.random.default_rng(4).choice(Q, 12, replace=False)
    par.check_nn(sc[qi].cpu().numpy(), ids[qi].cpu().numpy(), qs[qi].cpu().numpy(), Pi, S, ck, rec, norm, rnorm,
                 d, bits, k)


def test_nn_search_query_scales_and_database_norms():
    # queries of norm 1e-4 .. 1e4 and zero (the per-query power-of-two scaling of the fp16 operand),
    # database rows with norms spread over two decades (the norm multiply of the epilogue)
    d, bits, n_db, k = 200, 2, 3000, 10
    db, qs = syn.nn_inputs(n_db, 8, d)
    db = db * torch.exp(torch.linspace(-2.3, 2.3, n_db))[:, None]
    qs = qs * torch.tensor([1e-4, 1e-2, 1.0, 1.0, 1e2, 1e4, 3e4, 0.0])[:, None]
    Pi, S, ck, _, g = _setup(d, bits, 1)
    cache = tqb.PackedCache.empty(d, bits, True, 1, 1, n_db)
    tqb.tq_quantize_append(cache, db.reshape(1, 1, n_db, d).cuda(), 0, g["Pi"], g["SPiT"], g["ck"])
    sc, ids = tqb.tq_nn_search(cache, qs.cuda(), n_db, g["Pi"], g["S"], g["ck"], k)
    torch.cuda.synchronize()
    rec = par.as_u32(cache.records[0, 0].cpu().numpy())
    norm, rnorm = cache.norm[0, 0].cpu().numpy(), cache.rnorm[0, 0].cpu().numpy()
    par.check_nn(sc.cpu().numpy(), ids.cpu().numpy(), qs.double().numpy(), Pi, S, ck, rec, norm, rnorm, d, bits, k)
    # the zero query scores every vector 0: the k lowest indices, in order
    assert np.array_equal(ids[7].cpu().numpy(), np.arange(k)) and torch.all(sc[7] == 0).item()


@pytest.mark.parametrize("n_db", [0, 1, 5])
def test_nn_search_fewer_vectors_than_k(n_db):
    db, qs, Pi, S, ck, rec, norm, rnorm, sc, ids = _nn_case(200, 1, n_db, 130, 10, capacity=64)
    assert np.all(ids[:, n_db:] == -1) and np.all(np.isneginf(sc[:, n_db:]))
    if n_db:
        par.check_nn(sc, ids, qs.numpy(), Pi, S, ck, rec, norm, rnorm, 200, 1, 10)


def test_nn_search_equal_vectors_rank_by_index():
    # the same vector stored 300 times: every score ties, so the top-k are the k lowest indices
    d, bits, n, k = 200, 1, 300, 16
    _, qs = syn.nn_inputs(1, 40, d)
    x = syn.nn_inputs(1, 1, d)[0].repeat(n, 1)
    _, _, _, _, g = _setup(d, bits, 1)
    cache = tqb.PackedCache.empty(d, bits, True, 1, 1, n)
    tqb.tq_quantize_append(cache, x.reshape(1, 1, n, d).cuda(), 0, g["Pi"], g["SPiT"], g["ck"])
    sc, ids = tqb.tq_nn_search(cache, qs.cuda(), n, g["Pi"], g["S"], g["ck"], k)
    ids = ids.cpu().numpy()
    assert np.all(ids == np.arange(k)[None, :]), ids[:3]
    assert torch.all(sc == sc[:, :1]).item()


@pytest.mark.parametrize("k", [1, 3, 5, 10])
def test_nn_search_duplicates_pushed_down_keep_index_order(k):
    # vectors 0..119 stored again at 150..269: identical records tie exactly. When a later, higher
    # score pushes a tied pair down the running list, the lower index must stay and the higher fall
    # off (the case of a duplicate at the k-th place with a better vector after both)
    d, bits, n = 128, 2, 300
    db, qs = syn.nn_inputs(n, 200, d)
    db[150:270] = db[0:120]
    _, _, _, _, g = _setup(d, bits, 1)
    Pi, S, ck = g["Pi"].cpu().numpy(), g["S"].cpu().numpy(), g["ck"].cpu().numpy()
    cache = tqb.PackedCache.empty(d, bits, True, 1, 1, n)
    tqb.tq_quantize_append(cache, db.reshape(1, 1, n, d).cuda(), 0, g["Pi"], g["SPiT"], g["ck"])
    sc, ids = tqb.tq_nn_search(cache, qs.cuda(), n, g["Pi"], g["S"], g["ck"], k)
    rec = par.as_u32(cache.records[0, 0].cpu().numpy())
    par.check_nn(sc.cpu().numpy(), ids.cpu().numpy(), qs.numpy().astype(np.float64), Pi, S, ck, rec,
                 cache.norm[0, 0].cpu().numpy(), cache.rnorm[0, 0].cpu().numpy(), d, bits, k)


def test_decode_attend_empty():
    d = 128
    _, _, _, _, g = _setup(d, 2, 3)
    kc = tqb.PackedCache.empty(d, 2, True, 1, 2, 16)
    vc = tqb.PackedCache.empty(d, 3, False, 1, 2, 16)
    out = torch.full((1, 2, d), 7.0, device="cuda")
    tqb.tq_decode_attend(kc, vc, torch.randn(1, 2, d, device="cuda"), 0, 0.1, g["Pi"], g["S"], g["ck"], g["cv"],
                         out=out)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


# ---------------------------------------------------------------------------
# full-size workloads, sampled
# ---------------------------------------------------------------------------

def test_llama_decode_full_size():
    # 1 x 8 KV heads x 32768 tokens x 128, bf16 with outlier channels; 32 query heads;
    # K at 3 bits (2-bit codes + QJL), V at 3 bits MSE-only; the bench's launch shapes.
    k, v, q = syn.llama_inputs(device="cuda")
    Pi, S, ck, cv, g = _setup(128, 2, 3)
    kc, vc, lg, out, sc = _run_path(k, v, q, 128, 2, 3, g)
    _decode_full_size(kc, vc, q.cuda(), 32768, sc, g, out)   # the fused grouped-query pass, bit-equal
    rng = np.random.default_rng(17)
    rows = np.sort(rng.choice(32768, size=1024, replace=False))
    kx = k[0].float().cpu().numpy()
    vx = v[0].float().cpu().numpy()
    krec = par.as_u32(kc.records.cpu().numpy())[0]
    vrec = par.as_u32(vc.records.cpu().numpy())[0]
    kn, kr, vn = kc.norm.cpu().numpy()[0], kc.rnorm.cpu().numpy()[0], vc.norm.cpu().numpy()[0]
    lg_np, out_np, qn = lg.cpu().numpy()[0], out.cpu().numpy()[0], q.cpu().numpy()[0].astype(np.float64)
    for h in range(8):
        par.check_encoding(kx[h][rows], krec[h][rows], kn[h][rows], kr[h][rows], Pi, S, ck, 128, 2, True)
        par.check_encoding(vx[h][rows], vrec[h][rows], vn[h][rows], None, Pi, None, cv, 128, 3, False)
        # logits and outputs: every key and every query head of this KV head
        par.check_logits(lg_np[4 * h:4 * h + 4], qn[4 * h:4 * h + 4], Pi, S, ck, krec[h], kn[h], kr[h], 128, 2)
        par.check_attend(out_np[4 * h:4 * h + 4], lg_np[4 * h:4 * h + 4].astype(np.float64), sc, Pi, cv,
                         vrec[h], vn[h], 128, 3)
    assert np.isfinite(lg_np).all() and np.isfinite(out_np).all()


def _decode_full_size(kc, vc, q, T, sc, g, out_two_calls):
    """The one-call decode step on a full-size cache: equal bit for bit to tq_logits +
    tq_attend_v (same tables, chunks and accumulation order), status clean."""
    hq = q.shape[1]
    ws = torch.empty(max(256, tqb.tq_decode_workspace_size(kc, vc, hq, T)), dtype=torch.uint8, device="cuda")
    ws[:256].fill_(0xFF)   # the call must clear the status word itself
    out1 = tqb.tq_decode_attend(kc, vc, q, T, sc, g["Pi"], g["S"], g["ck"], g["cv"], workspace=ws)
    torch.cuda.synchronize()
    tqb.tq_workspace_status(ws)
    assert torch.equal(out1, out_two_calls), float((out1 - out_two_calls).abs().max())
    return out1


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_bsweep_full_size_sampled(bits):
    # 8 x 8 KV heads x 131072 tokens x 128, bf16, lognormal norms; K at b bits (b-1 codes + QJL),
    # V at b bits (MSE only); the bench's launch shapes.
    B, H, T, d = 8, 8, 131072, 128
    k, v, q = syn.sweep_inputs(device="cuda")
    Pi, S, ck, cv, g = _setup(d, bits - 1, bits)
    kc = tqb.PackedCache.empty(d, bits - 1, True, B, H, T)
    vc = tqb.PackedCache.empty(d, bits, False, B, H, T)
    tqb.tq_quantize_append(kc, k, 0, g["Pi"], g["SPiT"], g["ck"])
    tqb.tq_quantize_append(vc, v, 0, g["Pi"], None, g["cv"])
    ws = torch.empty(tqb.tq_logits_workspace_size(kc, H), dtype=torch.uint8, device="cuda")
    ws_a = torch.empty(tqb.tq_attend_workspace_size(vc, H, T), dtype=torch.uint8, device="cuda")
    lg = tqb.tq_logits(kc, q, T, g["Pi"], g["S"], g["ck"], workspace=ws)
    sc = 1.0 / math.sqrt(d)
    out = tqb.tq_attend_v(vc, lg, sc, T, g["Pi"], g["cv"], workspace=ws_a)
    torch.cuda.synchronize()
    tqb.tq_workspace_status(ws)
    tqb.tq_workspace_status(ws_a)
    out_d = _decode_full_size(kc, vc, q, T, sc, g, out)
    rng = np.random.default_rng(100 + bits)
    for _ in range(4):
        s, h = int(rng.integers(B)), int(rng.integers(H))
        rows = np.sort(rng.choice(T, size=512, replace=False))
        idx = torch.from_numpy(rows).cuda()
        kx = k[s, h].index_select(0, idx).float().cpu().numpy()
        krec = par.as_u32(kc.records[s, h].index_select(0, idx).cpu().numpy())
        kn = kc.norm[s, h].index_select(0, idx).cpu().numpy()
        kr = kc.rnorm[s, h].index_select(0, idx).cpu().numpy()
        par.check_encoding(kx, krec, kn, kr, Pi, S, ck, d, bits - 1, True)
        par.check_logits(lg[s, h].index_select(0, idx).cpu().numpy()[None, :],
                         q[s, h].cpu().numpy()[None, :].astype(np.float64), Pi, S, ck, krec, kn, kr, d, bits - 1)
        vx = v[s, h].index_select(0, idx).float().cpu().numpy()
        par.check_encoding(vx, par.as_u32(vc.records[s, h].index_select(0, idx).cpu().numpy()),
                           vc.norm[s, h].index_select(0, idx).cpu().numpy(), None, Pi, None, cv, d, bits, False)
        # softmax.V (two calls and the one-call step) over all of this head's tokens, oracle on the
        # GPU's cache and logits
        for o in (out, out_d):
            par.check_attend(o[s, h:h + 1].cpu().numpy(), lg[s, h:h + 1].cpu().numpy().astype(np.float64), sc, Pi,
                             cv, par.as_u32(vc.records[s, h].cpu().numpy()), vc.norm[s, h].cpu().numpy(), d, bits)
    # properties at full size: the packed norms are finite and positive, logits and outputs finite
    assert torch.isfinite(lg).all() and torch.isfinite(out).all()
    assert bool((kc.norm > 0).all()) and bool(torch.isfinite(kc.rnorm).all()) and bool((vc.norm > 0).all())


@pytest.mark.parametrize("bits", [3, 4])
def test_large_model_layer_sampled(bits):
    # one layer of the large-model cache: 128 KV heads x 131072 tokens x 128, fp16 N(0,1) with
    # outlier channels, one query head per KV head; K at b bits (b-1 codes + QJL), V at b bits.
    H, T, d = 128, 131072, 128
    k, v, q = syn.large_layer_inputs(0, device="cuda")
    Pi, S, ck, cv, g = _setup(d, bits - 1, bits)
    kc = tqb.PackedCache.empty(d, bits - 1, True, 1, H, T)
    vc = tqb.PackedCache.empty(d, bits, False, 1, H, T)
    tqb.tq_quantize_append(kc, k, 0, g["Pi"], g["SPiT"], g["ck"])
    tqb.tq_quantize_append(vc, v, 0, g["Pi"], None, g["cv"])
    ws_l = torch.empty(tqb.tq_logits_workspace_size(kc, H), dtype=torch.uint8, device="cuda")
    ws_a = torch.empty(tqb.tq_attend_workspace_size(vc, H, T), dtype=torch.uint8, device="cuda")
    lg = tqb.tq_logits(kc, q, T, g["Pi"], g["S"], g["ck"], workspace=ws_l)
    sc = 1.0 / math.sqrt(d)
    out = tqb.tq_attend_v(vc, lg, sc, T, g["Pi"], g["cv"], workspace=ws_a)
    torch.cuda.synchronize()
    tqb.tq_workspace_status(ws_l)
    tqb.tq_workspace_status(ws_a)
    out_d = _decode_full_size(kc, vc, q, T, sc, g, out)
    rng = np.random.default_rng(300 + bits)
    for h in [int(x) for x in rng.choice(H, size=3, replace=False)]:
        rows = np.sort(rng.choice(T, size=512, replace=False))
        idx = torch.from_numpy(rows).cuda()
        kx = k[0, h].index_select(0, idx).float().cpu().numpy()
        vx = v[0, h].index_select(0, idx).float().cpu().numpy()
        krec = par.as_u32(kc.records[0, h].index_select(0, idx).cpu().numpy())
        kn = kc.norm[0, h].index_select(0, idx).cpu().numpy()
        kr = kc.rnorm[0, h].index_select(0, idx).cpu().numpy()
        par.check_encoding(kx, krec, kn, kr, Pi, S, ck, d, bits - 1, True)
        par.check_encoding(vx, par.as_u32(vc.records[0, h].index_select(0, idx).cpu().numpy()),
                           vc.norm[0, h].index_select(0, idx).cpu().numpy(), None, Pi, None, cv, d, bits, False)
        par.check_logits(lg[0, h].index_select(0, idx).cpu().numpy()[None, :],
                         q[0, h].cpu().numpy()[None, :].astype(np.float64), Pi, S, ck, krec, kn, kr, d, bits - 1)
        # softmax.V (two calls and the one-call step) over all of this head's tokens, oracle on the
        # GPU's cache and logits
        for o in (out, out_d):
            par.check_attend(o[0, h:h + 1].cpu().numpy(), lg[0, h:h + 1].cpu().numpy().astype(np.float64), sc, Pi,
                             cv, par.as_u32(vc.records[0, h].cpu().numpy()), vc.norm[0, h].cpu().numpy(), d, bits)
    assert torch.isfinite(lg).all() and torch.isfinite(out).all()
    assert bool((kc.norm > 0).all()) and bool(torch.isfinite(kc.rnorm).all())
