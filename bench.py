#!/usr/bin/env python
"""Benchmark of the TurboQuant hot path on B200: one JSON line on stdout.

A step is one pass of the whole path over one batch of synthetic input:
  quantize-append of all keys and values into the packed caches
  -> L2 flush (the decode reads a cache written long before, from HBM)
  -> tq_logits (query projection + logit scan) -> tq_attend_v (softmax.V).

Default workload (N = 1): the large-model cache -- 80 layers x 128 KV heads x
d = 128 x 131072 tokens, fp16 K/V N(0,1) with outlier channels, keys at 3 bits
(2-bit codes + 1 QJL bit), values at 3 bits MSE-only, one query head per KV
head. It does not fit in HBM at once (687 GB of fp16), so it is streamed: one
step is one layer, `--steps` layers are timed after `--warmup` warm-up layers,
and the layer seeds cycle over the 80 layers. `--workload llama` runs the
Llama-3-8B-shaped decode (32 query heads on 8 KV heads, 32768 tokens, bf16),
`--workload sweep-b{2,3,4}` the b-sweep caches (8 x 8 x 131072 tokens),
`--workload large-b4` the large-model cache at 4 bits and `--workload nn-b{2,4}`
the nearest-neighbour search.

Metric: packed-KV logit-scan GB/s = packed key bytes (records + norms) read
by one tq_logits call / its device time; quantize tokens/s is reported beside
it. Times are CUDA events on the launching stream; with N ranks (torchrun)
every rank runs its own copy of the workload (weak scaling, no collective on
the data path) and the slowest rank's time is used.

`--impl reference` times the float64 CPU oracle on a bounded sample of the
same workload (the reference arm of this benchmark).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import tq_synth as syn  # noqa: E402

METRIC = "packed-KV logit-scan GB/s (% of HBM peak); K/V quantize tokens/s at 1 B200"
UNIT = "GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}

# DRAM bytes (read + write) per launch from one ncu capture of the kernel as it
# stands (profiles/), keyed by (kernel, workload); a key is removed when its
# kernel changes, and the bench then reports traffic as null.
NCU_TRAFFIC = {
    ("quantize_k", "llama"): 67_317_760 + 1_836_544,   # quantize_tc_kernel<1, 2, 0, 0> (tile schedule, sign warps)
    # (the value launch has changed since its last capture: no traffic figure)
    # the large-model layer's key launch, too large to capture: the Llama capture scaled by the head-vectors
    # processed (16 777 216 / 262 144 = 64; the traffic is the 256 B input and the record per head-vector)
    ("quantize_k", "large-b3"): 64 * (67_317_760 + 1_836_544),
    ("logits", "sweep-b3"): 2 * (234_967_296 + 16_118_528),   # logits_fast_kernel<2, 1>, 4-sequence capture x 2
    ("attend_v", "sweep-b3"): 2 * (234_991_616 + 3_727_616),  # attend_fast_kernel<3, 1, 0>, 4-sequence capture x 2
    # the large-model layer's scan and softmax.V: the 4-sequence b-sweep captures (4 194 304 keys, one query
    # head per KV head, the same kernels) scaled by the keys processed (x 4)
    ("logits", "large-b3"): 4 * (234_967_296 + 16_118_528),
    ("attend_v", "large-b3"): 4 * (234_991_616 + 3_727_616),
    ("logits", "llama"): 15_756_288 + 0,               # logits_gqa_kernel<2, 4> (the scan; tables read from L2)
    ("decode_attend", "sweep-b3"): 2 * (453_062_656 + 5_392_640),   # decode_fused_kernel<2, 3>, 4-sequence capture x 2
    ("decode_attend", "large-b3"): 4 * (453_062_656 + 5_392_640),   # the same capture scaled by the tokens (x 4)
}


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", default="large-b3",
                    choices=["llama"] + [f"sweep-b{b}{s}" for b in (2, 3, 4, 2.5, 3.5) for s in ("", "-s4")]
                    + ["sweep-b3-had"]
                    + ["large-b3", "large-b4", "nn-b2", "nn-b4", "nn-b2-s", "nn-b4-s"])
    ap.add_argument("--split", choices=["layers", "heads"], default="layers",
                    help="large-model cache on N GPUs: every rank streams its own layers (weak scaling), or "
                         "every layer's KV heads are split over the ranks (strong scaling); no exchange either way")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

def workload(name: str):
    if name.startswith("nn"):
        # "nn-b2" is the full search; "nn-b2-s" keeps 10^5 of the 10^6 database vectors (a profiling size)
        b = int(name.split("-")[1][1:])
        n_db = 100_000 if name.endswith("-s") else 1_000_000
        return dict(kind="nn", name=f"nn-search-b{b}: {n_db:,} database vectors d=200 (unit-normalised anisotropic "
                                    f"Gaussian, per-dimension std U[0.2, 2]), 10,000 queries of the same law, b={b} "
                                    f"({b - 1}-bit codes + QJL), top-10 by the key estimator; a synthetic stand-in "
                                    f"for the GloVe-200 benchmark",
                    n_db=n_db, n_q=10_000, d=200, k_idx=b - 1, k=10)
    if name == "llama":
        return dict(name="llama3-8b-decode: B=1 Hq=32 Hkv=8 d=128 T=32768 bf16 K b=3 (2-bit codes+QJL) V b=3 MSE",
                    n_seq=1, hq=32, hkv=8, d=128, T=32768, k_idx=2, v_idx=3, dtype=torch.bfloat16,
                    gen=lambda dev, seed: syn.llama_inputs(device=dev, seed=seed))
    if name.startswith("large"):
        b = int(name.split("-")[1][1:])
        return dict(name=f"large-model-b{b}: L layers x 128 KV heads x d=128 x 131072 tokens fp16 N(0,1) with outlier "
                         f"channels, streamed layer by layer, K b={b} V b={b}, one query head per KV head",
                    n_seq=1, hq=128, hkv=128, d=128, T=131072, k_idx=b - 1, v_idx=b, dtype=torch.float16,
                    gen=lambda dev, seed: syn.large_layer_inputs(seed, device=dev))
    # "sweep-b3-had": the b-sweep at b = 3 with the structured rotation Pi = H diag(s) / sqrt(d), the
    # quantizer applying it by the fast Walsh-Hadamard transform (tq_quantize_append_hadamard)
    if name == "sweep-b3-had":
        w = workload("sweep-b3")
        w.update(name=w["name"] + "; rotation H diag(s)/sqrt(d) by the fast Walsh-Hadamard transform", hadamard=True)
        return w
    # "sweep-b3" is the full b-sweep cache; "sweep-b3-s4" keeps 4 of its 8 sequences
    # (a profiling size: still larger than L2, half the device memory). "sweep-b3.5" and
    # "sweep-b2.5": fractional bits per channel, half of the rotated coordinates at one more
    # code bit (keys: b - 1 code bits on average + QJL; values: b code bits on average)
    b = float(name.split("-")[1][1:])
    B = 4 if name.endswith("-s4") else 8
    d = 128
    kb, vb = b - 1, b
    k_idx, v_idx = int(math.floor(kb)), int(math.floor(vb))
    k_nhi, v_nhi = int(round((kb - k_idx) * d)), int(round((vb - v_idx) * d))
    btxt = f"{b:g}"
    rate = (f" (keys: {k_idx + 1}-bit codes on {k_nhi} and {k_idx}-bit on {d - k_nhi} rotated coordinates + QJL; "
            f"values: {v_idx + 1}-bit on {v_nhi} and {v_idx}-bit on {d - v_nhi})") if k_nhi or v_nhi else ""
    return dict(name=f"bsweep-b{btxt}: B={B} Hq=8 Hkv=8 d=128 T=131072 bf16 lognormal norms, K b={btxt} V b={btxt}"
                     + rate,
                n_seq=B, hq=8, hkv=8, d=d, T=131072, k_idx=k_idx, v_idx=v_idx, k_nhi=k_nhi, v_nhi=v_nhi,
                dtype=torch.bfloat16, gen=lambda dev, seed: syn.sweep_inputs(n_seq=B, device=dev, seed=seed))


def _code_words(d, idx, n_hi) -> int:
    return ((idx + 1) * n_hi + idx * (d - n_hi) + 31) // 32


def key_bytes(w) -> int:
    rec = 4 * (_code_words(w["d"], w["k_idx"], w.get("k_nhi", 0)) + (w["d"] + 31) // 32)
    return w["n_seq"] * w["hkv"] * w["T"] * (rec + 8)


def value_bytes(w) -> int:
    rec = 4 * _code_words(w["d"], w["v_idx"], w.get("v_nhi", 0))
    return w["n_seq"] * w["hkv"] * w["T"] * (rec + 4)


def fit_codebooks(tqb, d, idx, n_hi):
    """The codebook argument of a cache: 2^idx centroids, followed for a mixed-rate cache by
    the 2^(idx+1) centroids of its wider group (tq_codebook_fit, host setup)."""
    c = tqb.tq_codebook_fit(d, idx)
    return torch.cat([c, tqb.tq_codebook_fit(d, idx + 1)]) if n_hi else c


def head_split(n_heads: int, world: int, rank: int) -> tuple[int, int]:
    """[first, end) of the KV heads rank owns when every layer's heads are split evenly over the ranks."""
    if world < 1 or not 0 <= rank < world or n_heads % world:
        raise ValueError(f"{n_heads} KV heads do not split evenly over {world} ranks")
    per = n_heads // world
    return rank * per, (rank + 1) * per


def tensor_executed(products: int, d: int, head_vectors: int, ms: float, bf16: float) -> dict:
    """Tensor work the d = 128 quantizer actually issues: its d x d products run on split 16-bit
    operands (keys: Pi x as hi + lo, and the sketch as three split products; values: hi + lo),
    `products` of them per head-vector at 2 d^2 flop each, against the dense bf16 peak."""
    flop = products * 2 * d * d
    tfs = flop * head_vectors / (ms * 1e-3) / 1e12
    return {"products_per_head_vector": products, "flop_per_head_vector": flop, "tflops": round(tfs, 1),
            "frac": round(tfs / bf16, 4)}


def rank_seed(rank: int) -> int:
    """Seed of a rank's replica of the workload (ranks draw different data)."""
    return syn.SEED_DATA + 7919 * rank


def max_over_ranks(values, device, world: int):
    """Element-wise maximum of per-rank timings (the slowest rank decides)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.t0 = self.t1 = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # the whole sampling window brackets the timed region; prefer samples under load
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        loaded = [v for v in sm if v > 500] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows
                                                                          if r[3].replace(".", "").isdigit())}


# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------

def run_tq(args, rank, world, local_rank):
    import kv_cache_vector_quantize_b200 as tqb

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workload(args.workload)
    d = w["d"]
    k, v, q = w["gen"](dev, rank_seed(rank))
    had = w.get("hadamard", False)
    Pi = (syn.randomized_hadamard(d) if had else syn.rotation(d)).to(dev)
    signs = syn.hadamard_signs(d).to(dev) if had else None
    S = syn.sketch(d).to(dev)
    ck = fit_codebooks(tqb, d, w["k_idx"], w.get("k_nhi", 0)).to(dev)
    cv = fit_codebooks(tqb, d, w["v_idx"], w.get("v_nhi", 0)).to(dev)
    SPiT = tqb.tq_sketch_rotation(Pi, S)
    kc = tqb.PackedCache.empty(d, w["k_idx"], True, w["n_seq"], w["hkv"], w["T"], device=dev, n_hi=w.get("k_nhi", 0))
    vc = tqb.PackedCache.empty(d, w["v_idx"], False, w["n_seq"], w["hkv"], w["T"], device=dev,
                               n_hi=w.get("v_nhi", 0))
    logits = torch.empty((w["n_seq"], w["hq"], w["T"]), dtype=torch.float32, device=dev)
    out = torch.empty((w["n_seq"], w["hq"], d), dtype=torch.float32, device=dev)
    ws_l = torch.empty(tqb.tq_logits_workspace_size(kc, w["hq"]), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(tqb.tq_attend_workspace_size(vc, w["hq"], w["T"]), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream(dev)

    def quantize(cache, x, spit, cb):
        if had:
            tqb.tq_quantize_append_hadamard(cache, x, 0, signs, spit, cb)
        else:
            tqb.tq_quantize_append(cache, x, 0, Pi, spit, cb)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        quantize(kc, k, SPiT, ck)
        if ev is not None:
            ev[1].record(stream)
        quantize(vc, v, None, cv)
        if ev is not None:
            ev[2].record(stream)
        flush.fill_(1.0)
        if ev is not None:
            ev[3].record(stream)
        tqb.tq_logits(kc, q, w["T"], Pi, S, ck, logits=logits, workspace=ws_l)
        if ev is not None:
            ev[4].record(stream)
        tqb.tq_attend_v(vc, logits, scale, w["T"], Pi, cv, out=out, workspace=ws_a)
        if ev is not None:
            ev[5].record(stream)

    kernels_per_step = 6   # quantize K, quantize V, query projection, logit scan, V chunks, V merge
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    tqb.tq_workspace_status(ws_l)
    tqb.tq_workspace_status(ws_a)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    tqb.tq_workspace_status(ws_l)   # raises if a kernel of the timed region reported a failure
    tqb.tq_workspace_status(ws_a)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    per = {name: [] for name in ("quantize_k", "quantize_v", "l2_flush", "logits", "attend_v")}
    for e in evs:
        per["quantize_k"].append(e[0].elapsed_time(e[1]))
        per["quantize_v"].append(e[1].elapsed_time(e[2]))
        per["l2_flush"].append(e[2].elapsed_time(e[3]))
        per["logits"].append(e[3].elapsed_time(e[4]))
        per["attend_v"].append(e[4].elapsed_time(e[5]))
    mean = {kk: sum(vv) / len(vv) for kk, vv in per.items()}

    # slowest rank decides
    total_ms, logits_ms, quant_ms = max_over_ranks(
        [total_ms, mean["logits"], mean["quantize_k"] + mean["quantize_v"]], dev, world)

    kb, vb = key_bytes(w), value_bytes(w)
    scan_gbs_rank = kb / (logits_ms * 1e-3) / 1e9
    value = world * scan_gbs_rank
    head_vectors = w["n_seq"] * w["hkv"] * w["T"]
    quant_tps = world * w["n_seq"] * w["T"] / (quant_ms * 1e-3)

    # ---- structured rotation: the dense-Pi quantizers on the same rotation and inputs, for comparison ----
    dense = None
    if had:
        dk = tqb.PackedCache.empty(d, w["k_idx"], True, w["n_seq"], w["hkv"], w["T"], device=dev)
        dv = tqb.PackedCache.empty(d, w["v_idx"], False, w["n_seq"], w["hkv"], w["T"], device=dev)
        kf, vf = k.float(), v.float()   # fp32 inputs take the FP32-core kernel on both rotations
        calls = {
            "tensor_core_dense_bf16": (lambda: tqb.tq_quantize_append(dk, k, 0, Pi, SPiT, ck),
                                       lambda: tqb.tq_quantize_append(dv, v, 0, Pi, None, cv)),
            "fp32_cores_dense_fp32": (lambda: tqb.tq_quantize_append(dk, kf, 0, Pi, SPiT, ck),
                                      lambda: tqb.tq_quantize_append(dv, vf, 0, Pi, None, cv)),
            "fp32_cores_hadamard_fp32": (lambda: tqb.tq_quantize_append_hadamard(dk, kf, 0, signs, SPiT, ck),
                                         lambda: tqb.tq_quantize_append_hadamard(dv, vf, 0, signs, None, cv)),
        }
        dense = {"note": "ms per call on the same rotation and inputs: the dense Pi on the tensor cores (bf16 "
                         "inputs, the step's default), and on the FP32 cores with fp32 inputs against the fast "
                         "Walsh-Hadamard transform on the FP32 cores (per_kernel_ms: the transform on bf16 inputs)"}
        for label, (fk, fv) in calls.items():
            tk = tv = 0.0
            for rep_ in range(2 + args.steps):
                for which, fn in (("k", fk), ("v", fv)):
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    fn()
                    b.record(stream)
                    torch.cuda.synchronize(dev)
                    if rep_ >= 2:
                        if which == "k":
                            tk += a.elapsed_time(b) / args.steps
                        else:
                            tv += a.elapsed_time(b) / args.steps
            dense[label] = {"quantize_k_ms": round(tk, 5), "quantize_v_ms": round(tv, 5)}
        del dk, dv, kf, vf
        # d = 256 (fp32, 1 x 8 heads x 131072 tokens): where the transform's d log d against d^2 matters more
        d2 = 256
        x2 = syn.gaussian((1, 8, w["T"], d2), 91, device=dev)
        Pi2, s2 = syn.randomized_hadamard(d2).to(dev), syn.hadamard_signs(d2).to(dev)
        SPiT2 = tqb.tq_sketch_rotation(Pi2, syn.sketch(d2).to(dev))
        ck2, cv2 = tqb.tq_codebook_fit(d2, w["k_idx"]).to(dev), tqb.tq_codebook_fit(d2, w["v_idx"]).to(dev)
        dk2 = tqb.PackedCache.empty(d2, w["k_idx"], True, 1, 8, w["T"], device=dev)
        dv2 = tqb.PackedCache.empty(d2, w["v_idx"], False, 1, 8, w["T"], device=dev)
        for label, fk, fv in (("d256_fp32_cores_dense_fp32", lambda: tqb.tq_quantize_append(dk2, x2, 0, Pi2, SPiT2, ck2),
                               lambda: tqb.tq_quantize_append(dv2, x2, 0, Pi2, None, cv2)),
                              ("d256_fp32_cores_hadamard_fp32",
                               lambda: tqb.tq_quantize_append_hadamard(dk2, x2, 0, s2, SPiT2, ck2),
                               lambda: tqb.tq_quantize_append_hadamard(dv2, x2, 0, s2, None, cv2))):
            tk = tv = 0.0
            for rep_ in range(2 + args.steps):
                for which, fn in (("k", fk), ("v", fv)):
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    fn()
                    b.record(stream)
                    torch.cuda.synchronize(dev)
                    if rep_ >= 2:
                        if which == "k":
                            tk += a.elapsed_time(b) / args.steps
                        else:
                            tv += a.elapsed_time(b) / args.steps
            dense[label] = {"quantize_k_ms": round(tk, 5), "quantize_v_ms": round(tv, 5),
                            "head_vectors": 8 * w["T"]}
        del x2, dk2, dv2

    # ---- the one-call decode step (tq_decode_attend) on the same caches, L2 flushed before each ----
    ws_d = torch.empty(max(256, tqb.tq_decode_workspace_size(kc, vc, w["hq"], w["T"])), dtype=torch.uint8, device=dev)
    out_d = torch.empty_like(out)

    def decode_step():
        tqb.tq_decode_attend(kc, vc, q, w["T"], scale, Pi, S, ck, cv, out=out_d, workspace=ws_d)

    for _ in range(3):
        flush.fill_(1.0)
        decode_step()
    torch.cuda.synchronize(dev)
    dec_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in dec_evs:
        flush.fill_(1.0)
        a.record(stream)
        decode_step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    tqb.tq_workspace_status(ws_d)
    dec_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in dec_evs) / len(dec_evs)], dev, world)[0]

    # ---- end to end: pinned host inputs in, result out, through the public API ----
    e2e = None
    if args.e2e_steps > 0:
        hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
        hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
        hq_ = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hk.copy_(k)
        hv.copy_(v)
        hq_.copy_(q)
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

        def step_e2e():
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            q.copy_(hq_, non_blocking=True)
            step()
            hout.copy_(out, non_blocking=True)

        for _ in range(2):
            step_e2e()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        a.record(stream)
        for _ in range(args.e2e_steps):
            step_e2e()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks([a.elapsed_time(b) / args.e2e_steps], dev, world)[0]
        h2d = (hk.numel() * hk.element_size() + hv.numel() * hv.element_size() + hq_.numel() * hq_.element_size())
        e2e = {"value": world * kb / (e2e_ms * 1e-3) / 1e9, "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hout.numel() * hout.element_size(),
               "note": "packed key bytes scanned per end-to-end step (pinned H2D of K, V, q; path; D2H of out)"}

    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    bf16 = float(peaks["bf16_tflops"])
    src_txt = f"hbm_gbs / bf16_tflops, {peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    # quantize: algorithmic bytes = bf16 input + record + norms; algorithmic flops = the d x d projections
    qk_bytes = head_vectors * (2 * d + kb // head_vectors)
    qv_bytes = head_vectors * (2 * d + vb // head_vectors)
    qk_flops, qv_flops = head_vectors * 4 * d * d, head_vectors * 2 * d * d

    def quant_roof(kernel, nbytes, nflops, ms, traffic):
        gbs = nbytes / (ms * 1e-3) / 1e9
        tfs = nflops / (ms * 1e-3) / 1e12
        # the roofline bound is the slower of bytes at HBM peak and flops at dense bf16 peak
        bound = "hbm" if nbytes / hbm > nflops / (bf16 * 1e3) else "tensor"
        ach, peak, unit = (gbs, hbm, "GB/s") if bound == "hbm" else (tfs, bf16, "TFLOP/s")
        return {"kernel": kernel, "bound": bound, "achieved": round(ach, 1), "peak": peak, "unit": unit,
                "frac": round(ach / peak, 4), "traffic": traffic, "peak_source": src_txt,
                "tensor_tflops": round(tfs, 1), "tensor_frac": round(tfs / bf16, 4),
                "algorithmic": f"{nbytes // head_vectors} B and {nflops // head_vectors} flop per head-vector"}

    roofline = quant_roof("quantize_tc_kernel, key launch (tq_quantize_append on the K cache)", qk_bytes, qk_flops,
                          mean["quantize_k"], NCU_TRAFFIC.get(("quantize_k", args.workload)))
    roof_qv = quant_roof("quantize_tc_kernel, value launch (tq_quantize_append on the V cache)", qv_bytes, qv_flops,
                         mean["quantize_v"], NCU_TRAFFIC.get(("quantize_v", args.workload)))
    if w["d"] == 128:
        roofline["tensor_executed"] = tensor_executed(5, w["d"], head_vectors, mean["quantize_k"], bf16)
        roof_qv["tensor_executed"] = tensor_executed(2, w["d"], head_vectors, mean["quantize_v"], bf16)
    roof_scan = {"kernel": "tq_logits (query projection + logit scan)", "bound": "hbm",
                 "achieved": round(scan_gbs_rank, 1), "peak": hbm, "unit": "GB/s",
                 "frac": round(scan_gbs_rank / hbm, 4), "traffic": NCU_TRAFFIC.get(("logits", args.workload)),
                 "peak_source": src_txt,
                 "algorithmic": f"{kb // head_vectors} B per key (record + norm + rnorm)"}
    att_gbs = vb / (mean["attend_v"] * 1e-3) / 1e9
    roof_att = {"kernel": "tq_attend_v (chunk softmax.V + merge)", "bound": "hbm", "achieved": round(att_gbs, 1),
                "peak": hbm, "unit": "GB/s", "frac": round(att_gbs / hbm, 4),
                "traffic": NCU_TRAFFIC.get(("attend_v", args.workload)), "peak_source": src_txt,
                "algorithmic": f"{vb // head_vectors} B per value (record + norm)"}
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w["name"], "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed (2 x L2 write) between quantize and decode inside every step; the flush is in "
                         "ms_per_step, not in the kernel times",
                   "value_definition": "packed K bytes per tq_logits call / its mean device time (CUDA events), "
                                       "summed over ranks"},
        "quantize_tokens_per_s": round(quant_tps, 1),
        "quantize_head_vectors_per_s": round(world * head_vectors / (quant_ms * 1e-3), 1),
        "per_kernel_ms": {kk: round(vv, 5) for kk, vv in mean.items()},
        **({"dense_rotation_quantize": dense} if dense is not None else {}),
        "packed_bytes": {"keys": kb, "values": vb},
        "roofline": roofline, "roofline_logit_scan": roof_scan, "roofline_quantize_v": roof_qv,
        "roofline_attend_v": roof_att,
        "roofline_decode_attend": decode_roof(dec_ms, mean["logits"] + mean["attend_v"], kb + vb, w, hbm, src_txt,
                                              NCU_TRAFFIC.get(("decode_attend", args.workload))),
        "gpu_launches": kernels_per_step * args.steps,
        "clocks": clk, "e2e": e2e,
    }
    return result, w


def decode_roof(ms, two_call_ms, nbytes, w, hbm, src_txt, traffic=None):
    """The one-call decode step against HBM: packed key + value bytes per call / its time."""
    one_pass = (w["hq"] == w["hkv"] and w["d"] == 128 and w["k_idx"] in (1, 2) and not w.get("k_nhi")
                and not w.get("v_nhi"))
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "tq_decode_attend (" + ("query projection + fused logits/softmax.V pass + merge" if one_pass
                                              else "tq_logits + tq_attend_v") + ")",
            "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
            "traffic": traffic, "peak_source": src_txt, "ms": round(ms, 5),
            "two_calls_ms": round(two_call_ms, 5), "algorithmic": "packed key and value records + norms per call"}


def run_large(args, rank, world, local_rank):
    """Large-model cache streamed layer by layer. A step is one layer: quantize its K and V
    into the packed caches, flush L2, then one decode step on them (tq_logits, tq_attend_v).
    The layer's fp16 inputs are generated on the device between steps (the 80 layers do not
    fit in HBM at once: 687 GB), so every step starts with its inputs resident; steps cycle
    through the 80 layer seeds. The packed buffers are reused by every layer."""
    import kv_cache_vector_quantize_b200 as tqb

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workload(args.workload)
    by_heads = args.split == "heads" and world > 1
    if by_heads:
        # this rank's slice of every layer: KV heads [h0, h1) and their query heads
        h0, h1 = head_split(w["hkv"], world, rank)
        w = dict(w, hkv=h1 - h0, hq=(h1 - h0) * (w["hq"] // w["hkv"]))
    d, H, T = w["d"], w["hkv"], w["T"]
    n_layers = 80
    Pi = syn.rotation(d).to(dev)
    S = syn.sketch(d).to(dev)
    ck = tqb.tq_codebook_fit(d, w["k_idx"]).to(dev)
    cv = tqb.tq_codebook_fit(d, w["v_idx"]).to(dev)
    SPiT = tqb.tq_sketch_rotation(Pi, S)
    kc = tqb.PackedCache.empty(d, w["k_idx"], True, 1, H, T, device=dev)
    vc = tqb.PackedCache.empty(d, w["v_idx"], False, 1, H, T, device=dev)
    logits = torch.empty((1, w["hq"], T), dtype=torch.float32, device=dev)
    out = torch.empty((1, w["hq"], d), dtype=torch.float32, device=dev)
    ws_l = torch.empty(tqb.tq_logits_workspace_size(kc, w["hq"]), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(tqb.tq_attend_workspace_size(vc, w["hq"], T), dtype=torch.uint8, device=dev)
    ws_d = torch.empty(max(256, tqb.tq_decode_workspace_size(kc, vc, w["hq"], T)), dtype=torch.uint8, device=dev)
    out_d = torch.empty_like(out)
    flush = torch.empty((2 * torch.cuda.get_device_properties(dev).L2_cache_size) // 4, dtype=torch.float32,
                        device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(d)
    names = ("quantize_k", "quantize_v", "l2_flush", "logits", "attend_v")

    def path(k, v, q, ev=None):
        calls = (lambda: tqb.tq_quantize_append(kc, k, 0, Pi, SPiT, ck),
                 lambda: tqb.tq_quantize_append(vc, v, 0, Pi, None, cv),
                 lambda: flush.fill_(1.0),
                 lambda: tqb.tq_logits(kc, q, T, Pi, S, ck, logits=logits, workspace=ws_l),
                 lambda: tqb.tq_attend_v(vc, logits, scale, T, Pi, cv, out=out, workspace=ws_a))
        for i, call in enumerate(calls):
            if ev is not None:
                ev[i].record(stream)
            call()
        if ev is not None:
            ev[len(calls)].record(stream)

    def layer_inputs(step):
        if by_heads:   # the same layer on every rank, each generating its own heads
            return syn.large_layer_inputs(step % n_layers + 1000 * rank, n_heads=H, device=dev)
        return w["gen"](dev, step % n_layers + rank_seed(rank))

    for i in range(args.warmup):
        k, v, q = layer_inputs(i)
        path(k, v, q)
        del k, v
    torch.cuda.synchronize(dev)
    tqb.tq_workspace_status(ws_l)
    tqb.tq_workspace_status(ws_a)
    per = {n: 0.0 for n in names}
    clocks = ClockSampler(dev.index)
    time.sleep(0.3)
    clocks.mark_start()
    for step in range(args.steps):
        k, v, q = layer_inputs(step)   # generated on the device, outside the timed calls
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        path(k, v, q, ev)
        torch.cuda.synchronize(dev)
        for i, n in enumerate(names):
            per[n] += ev[i].elapsed_time(ev[i + 1])
        if step + 1 < args.steps:
            del k, v
    clocks.mark_end()
    tqb.tq_workspace_status(ws_l)   # raises if a kernel of the timed region reported a failure
    tqb.tq_workspace_status(ws_a)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = {n: per[n] / args.steps for n in names}
    path_ms = sum(step_ms[n] for n in names if n != "l2_flush")
    logits_ms, quant_ms, path_ms, qk_ms, qv_ms, att_ms = max_over_ranks(
        [step_ms["logits"], step_ms["quantize_k"] + step_ms["quantize_v"], path_ms, step_ms["quantize_k"],
         step_ms["quantize_v"], step_ms["attend_v"]], dev, world)

    # ---- the one-call decode step (tq_decode_attend) on the last layer's caches, L2 flushed before each ----
    def decode_step():
        tqb.tq_decode_attend(kc, vc, q, T, scale, Pi, S, ck, cv, out=out_d, workspace=ws_d)

    for _ in range(3):
        flush.fill_(1.0)
        decode_step()
    torch.cuda.synchronize(dev)
    dec_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
    for a, b in dec_evs:
        flush.fill_(1.0)
        a.record(stream)
        decode_step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    tqb.tq_workspace_status(ws_d)
    dec_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in dec_evs) / len(dec_evs)], dev, world)[0]

    # ---- end to end: one layer's pinned host K, V, q in, the path, out back, through the public API ----
    e2e = None
    if args.e2e_steps > 0:
        hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
        hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
        hq_ = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hk.copy_(k)
        hv.copy_(v)
        hq_.copy_(q)
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

        def step_e2e():
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            q.copy_(hq_, non_blocking=True)
            path(k, v, q)
            hout.copy_(out, non_blocking=True)

        step_e2e()
        torch.cuda.synchronize(dev)
        n_e2e = min(args.e2e_steps, 5)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        a.record(stream)
        for _ in range(n_e2e):
            step_e2e()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks([a.elapsed_time(b) / n_e2e], dev, world)[0]
        h2d = hk.numel() * hk.element_size() + hv.numel() * hv.element_size() + hq_.numel() * hq_.element_size()
        e2e = {"value": round(world * key_bytes(w) / (e2e_ms * 1e-3) / 1e9, 3), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 4), "steps": n_e2e, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": hout.numel() * hout.element_size(),
               "note": "packed key bytes scanned per end-to-end layer step (pinned H2D of the layer's fp16 K and V "
                       "and its queries, quantize, flush, logits, softmax.V, D2H of out); bound by the H2D copy"}
        del hk, hv

    kb, vb = key_bytes(w), value_bytes(w)
    fp16_bytes = 2 * H * T * d * 2
    lw = world if by_heads else 1   # ranks holding parts of one layer
    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    bf16 = float(peaks["bf16_tflops"])
    src_txt = f"hbm_gbs / bf16_tflops, {peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    scan_gbs = kb / (logits_ms * 1e-3) / 1e9
    hv_layer = H * T
    qk_bytes, qv_bytes = hv_layer * 2 * d + kb, hv_layer * 2 * d + vb
    qk_flops, qv_flops = hv_layer * 4 * d * d, hv_layer * 2 * d * d

    def quant_roof(kernel, nbytes, nflops, ms, traffic):
        gbs = nbytes / (ms * 1e-3) / 1e9
        tfs = nflops / (ms * 1e-3) / 1e12
        bound = "hbm" if nbytes / hbm > nflops / (bf16 * 1e3) else "tensor"
        ach, peak, unit = (gbs, hbm, "GB/s") if bound == "hbm" else (tfs, bf16, "TFLOP/s")
        return {"kernel": kernel, "bound": bound, "achieved": round(ach, 1), "peak": peak, "unit": unit,
                "frac": round(ach / peak, 4), "traffic": traffic, "peak_source": src_txt,
                "tensor_tflops": round(tfs, 1), "tensor_frac": round(tfs / bf16, 4), "ms": round(ms, 4),
                "algorithmic": f"{nbytes // hv_layer} B and {nflops // hv_layer} flop per head-vector, "
                               f"{hv_layer} head-vectors per launch"}

    roofline = quant_roof("quantize_tc_kernel, key launch (tq_quantize_append on the layer's K cache)", qk_bytes,
                          qk_flops, qk_ms, NCU_TRAFFIC.get(("quantize_k", args.workload)))
    roof_qv = quant_roof("quantize_tc_kernel, value launch (tq_quantize_append on the layer's V cache)", qv_bytes,
                         qv_flops, qv_ms, NCU_TRAFFIC.get(("quantize_v", args.workload)))
    roofline["tensor_executed"] = tensor_executed(5, d, hv_layer, qk_ms, bf16)
    roof_qv["tensor_executed"] = tensor_executed(2, d, hv_layer, qv_ms, bf16)
    att_gbs = vb / (att_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": round(world * scan_gbs, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(path_ms, 4), "higher_is_better": True,
        "scaling": "strong" if by_heads else "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": w["name"].replace("L layers", f"{n_layers} layers"),
                   "parallelism": "single" if world == 1 else (f"heads{world}: {H} KV heads of every layer per rank"
                                                               if by_heads else f"replicas{world}"),
                   "step": "one layer (layer seeds cycled over the 80 layers; its fp16 K/V generated on the device "
                           "before the step, outside the timed calls): quantize K and V, L2 flush, tq_logits, "
                           "tq_attend_v; ms_per_step = the four calls' device time, the flush excluded",
                   "l2": "flushed (2 x L2 write) between quantize and the decode of every layer; every layer's "
                         "inputs (8.6 GB) are also larger than L2",
                   "value_definition": "packed K bytes of one layer per tq_logits call / its mean device time "
                                       "(CUDA events), summed over ranks",
                   "dtype_note": "narrowest arithmetic on the path: fp16 tensor-core products with split operands "
                                 "and float32 accumulation in the quantizer; the single-head scan and softmax.V "
                                 "accumulate in float32"},
        "quantize_tokens_per_s": round((1 if by_heads else world) * T / (quant_ms * 1e-3), 1),
        "quantize_head_vectors_per_s": round(world * 2 * hv_layer / (quant_ms * 1e-3), 1),
        "per_kernel_ms_per_layer": {n: round(x, 5) for n, x in step_ms.items()},
        # a whole layer (all ranks' heads when they are split)
        "compressed_bytes": {"per_layer": lw * (kb + vb), "timed_layers": args.steps * lw * (kb + vb),
                             "all_80_layers": n_layers * lw * (kb + vb)},
        "uncompressed_fp16_bytes": {"per_layer": lw * fp16_bytes, "all_80_layers": n_layers * lw * fp16_bytes},
        "compression_ratio_vs_fp16": round(fp16_bytes / (kb + vb), 4),
        "packed_bytes": {"keys": kb, "values": vb},
        "roofline": roofline, "roofline_quantize_v": roof_qv,
        "roofline_logit_scan": {"kernel": "tq_logits (query projection + logit scan)", "bound": "hbm",
                                "achieved": round(scan_gbs, 1), "peak": hbm, "unit": "GB/s",
                                "frac": round(scan_gbs / hbm, 4),
                                "traffic": NCU_TRAFFIC.get(("logits", args.workload)), "peak_source": src_txt,
                                "ms": round(logits_ms, 5),
                                "algorithmic": f"{kb // hv_layer} B per key (record + norm + rnorm)"},
        "roofline_attend_v": {"kernel": "tq_attend_v (chunk softmax.V + merge)", "bound": "hbm",
                              "achieved": round(att_gbs, 1), "peak": hbm, "unit": "GB/s",
                              "frac": round(att_gbs / hbm, 4),
                              "traffic": NCU_TRAFFIC.get(("attend_v", args.workload)), "peak_source": src_txt,
                              "ms": round(att_ms, 5), "algorithmic": f"{vb // hv_layer} B per value (record + norm)"},
        "roofline_decode_attend": decode_roof(dec_ms, logits_ms + att_ms, kb + vb, w, hbm, src_txt,
                                              NCU_TRAFFIC.get(("decode_attend", args.workload))),
        # per step: quantize K, quantize V; projection + scan; V chunks + merge
        "gpu_launches": 6 * args.steps, "clocks": clk, "e2e": e2e,
    }
    return result, w


def nn_record_bytes(w) -> int:
    return 4 * ((w["k_idx"] * w["d"] + 31) // 32 + (w["d"] + 31) // 32) + 8


def run_nn(args, rank, world, local_rank):
    """Nearest-neighbour search: per step, quantize the database into a packed key stream, flush
    L2, then the top-10 search of every query (tq_nn_search). Recall@10 against the exact float64
    inner products is measured after the timed region."""
    import kv_cache_vector_quantize_b200 as tqb

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workload(args.workload)
    d, N, Q, k = w["d"], w["n_db"], w["n_q"], w["k"]
    db, qs = syn.nn_inputs(N, Q, d, device=dev)
    Pi = syn.rotation(d).to(dev)
    S = syn.sketch(d).to(dev)
    cb = tqb.tq_codebook_fit(d, w["k_idx"]).to(dev)
    SPiT = tqb.tq_sketch_rotation(Pi, S)
    cache = tqb.PackedCache.empty(d, w["k_idx"], True, 1, 1, N, device=dev)
    x = db.reshape(1, 1, N, d)
    scores = torch.empty((Q, k), dtype=torch.float32, device=dev)
    ids = torch.empty((Q, k), dtype=torch.int64, device=dev)
    ws = torch.empty(tqb.tq_nn_workspace_size(cache, Q, N), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        tqb.tq_quantize_append(cache, x, 0, Pi, SPiT, cb)
        if ev is not None:
            ev[1].record(stream)
        flush.fill_(1.0)
        if ev is not None:
            ev[2].record(stream)
        tqb.tq_nn_search(cache, qs, N, Pi, S, cb, k, scores, ids, ws)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    tqb.tq_workspace_status(ws)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    tqb.tq_workspace_status(ws)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    per = {n: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / len(evs)
           for i, n in enumerate(("quantize", "l2_flush", "nn_search"))}
    total_ms = t_start.elapsed_time(t_end)
    total_ms, search_ms, quant_ms = max_over_ranks([total_ms, per["nn_search"], per["quantize"]], dev, world)

    # recall@10 of the returned ids against the exact top-10 of the float64 inner products
    hits = 0
    dbd = db.double()
    for a in range(0, Q, 500):
        exact = (qs[a:a + 500].double() @ dbd.T).topk(k, dim=1).indices
        hits += int((exact[:, :, None] == ids[a:a + 500, None, :]).any(dim=2).sum().item())
    del dbd
    recall = hits / (Q * k)

    e2e = None
    if args.e2e_steps > 0:
        hx = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        hq = torch.empty(qs.shape, dtype=qs.dtype, pin_memory=True)
        hx.copy_(x)
        hq.copy_(qs)
        hs = torch.empty(scores.shape, dtype=scores.dtype, pin_memory=True)
        hi = torch.empty(ids.shape, dtype=ids.dtype, pin_memory=True)

        def step_e2e():
            x.copy_(hx, non_blocking=True)
            qs.copy_(hq, non_blocking=True)
            tqb.tq_quantize_append(cache, x, 0, Pi, SPiT, cb)
            tqb.tq_nn_search(cache, qs, N, Pi, S, cb, k, scores, ids, ws)
            hs.copy_(scores, non_blocking=True)
            hi.copy_(ids, non_blocking=True)

        for _ in range(2):
            step_e2e()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        a.record(stream)
        for _ in range(args.e2e_steps):
            step_e2e()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks([a.elapsed_time(b) / args.e2e_steps], dev, world)[0]
        e2e = {"value": round(world * N * nn_record_bytes(w) / (e2e_ms * 1e-3) / 1e9, 3), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 4),
               "h2d_bytes_per_step": hx.numel() * hx.element_size() + hq.numel() * hq.element_size(),
               "d2h_bytes_per_step": hs.numel() * hs.element_size() + hi.numel() * hi.element_size(),
               "note": "packed database bytes per end-to-end step (pinned H2D of the database and the queries, "
                       "quantize, search, D2H of the top-10 scores and ids)"}

    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    tf_burst = float(peaks["bf16_tflops"])
    tf_sust = float(peaks.get("bf16_tflops_sustained", tf_burst))
    src_txt = (f"bf16_tflops (burst; fp16 has the same nominal dense rate), {peak_src} (MEASURED_PEAKS.json)"
               if peak_src == "measured" else "fallback")
    nb = N * nn_record_bytes(w)
    scan_gbs = nb / (search_ms * 1e-3) / 1e9
    flops = 2.0 * Q * N * 2 * d
    tfs = flops / (search_ms * 1e-3) / 1e12
    kp = 64 * ((2 * d + 63) // 64)
    padded = 2.0 * ((Q + 127) // 128 * 128) * ((N + 127) // 128 * 128) * kp
    q_bytes, q_flops = N * (4 * d + nn_record_bytes(w)), N * 4 * d * d
    q_gbs, q_tfs = q_bytes / (quant_ms * 1e-3) / 1e9, q_flops / (quant_ms * 1e-3) / 1e12
    result = {
        "metric": METRIC, "value": round(world * scan_gbs, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": w["name"], "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed (2 x L2 write) between quantize and search inside every step",
                   "value_definition": "packed database bytes (records + norms) per tq_nn_search call / its mean "
                                       "device time; the call is bound by the tensor core (roofline)"},
        "recall_at_10": round(recall, 4),
        "quantize_tokens_per_s": round(world * N / (quant_ms * 1e-3), 1),
        "per_kernel_ms": {n: round(v, 4) for n, v in per.items()},
        "packed_bytes": {"database": nb},
        "roofline": {"kernel": "tq_nn_search (query projection + nn_scan_kernel tensor-core scan + merge)",
                     "bound": "tensor", "achieved": round(tfs, 1), "peak": tf_burst, "unit": "TFLOP/s",
                     "frac": round(tfs / tf_burst, 4), "frac_vs_sustained": round(tfs / tf_sust, 4),
                     "traffic": NCU_TRAFFIC.get(("nn_search", args.workload)), "peak_source": src_txt,
                     "algorithmic": f"{4 * d} flop per (query, database vector) pair (two length-{d} dot "
                                    f"products); the kernel issues {padded / flops:.3f}x that with the padding of "
                                    f"K to {kp} and of queries and vectors to 128"},
        "roofline_nn_scan_hbm": {"bound": "hbm", "achieved": round(scan_gbs, 2), "peak": hbm, "unit": "GB/s",
                                 "frac": round(scan_gbs / hbm, 5)},
        "roofline_quantize": {"kernel": "quantize_kernel (tq_quantize_append, d = 200 fp32 database)",
                              "bound": "hbm" if q_bytes / hbm > q_flops / (tf_burst * 1e3) else "tensor",
                              "achieved_gbs": round(q_gbs, 1), "hbm_frac": round(q_gbs / hbm, 4),
                              "achieved_tflops": round(q_tfs, 2),
                              "algorithmic": f"{4 * d + nn_record_bytes(w)} B and {4 * d * d} flop per vector"},
        # per step: the quantize kernel; projection, scan and merge of the search
        "gpu_launches": 4 * args.steps, "clocks": clk, "e2e": e2e,
    }
    return result, w


# ----------------------------------------------------------------------------
# the oracle on a bounded sample (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------

def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return 1


def oracle_sample_step(w, state):
    """One bounded sample of the workload through the oracle: quantize 2048 keys and
    2048 values of one KV head; unpack + logits of that head's query group over
    all T keys of the head (pre-packed); softmax.V over the same head.
    Returns (packed key bytes scanned, logit seconds, quantize seconds, head-vectors quantized)."""
    d = w["d"]
    o = state["ops"]
    t0 = time.perf_counter()
    ek = o["enc_k"](state["k_rows"])
    ev = o["enc_v"](state["v_rows"])
    o["pack_k"](ek)
    o["pack_v"](ev)
    t1 = time.perf_counter()
    gi, gs = o["unpack_k"](state["krec"])
    lg = o["logits"](state["q"], state["kn"], state["kr"], gi, gs)
    t2 = time.perf_counter()
    vi, _ = o["unpack_v"](state["vrec"])
    o["attend"](lg, 1.0 / math.sqrt(d), state["vn"], vi)
    return key_bytes(w) // (w["n_seq"] * w["hkv"]), t2 - t1, t1 - t0, 2 * state["k_rows"].shape[0]


def oracle_nn_step(w, state):
    """One bounded sample of the search through the oracle: quantize 2048 database vectors;
    unpack + estimator scores of 32 queries over 20000 packed vectors + top-10. Returns (the
    workload's packed database bytes prorated to the (query, vector) pairs scored, scoring
    seconds, quantize seconds, vectors quantized)."""
    from oracle import turboquant as otq

    d = w["d"]
    t0 = time.perf_counter()
    e = otq.quantize(state["rows"], state["Pi"], state["c"], state["S"])
    otq.pack(e["idx"], e["sign"], d, w["k_idx"], True)
    t1 = time.perf_counter()
    gi, gs = otq.unpack(state["rec"], d, w["k_idx"], True)
    lg = otq.logits(state["q"], state["Pi"], state["S"], state["c"], state["n"], state["r"], gi, gs)
    otq.topk(lg, w["k"])
    t2 = time.perf_counter()
    pairs = state["q"].shape[0] * state["rec"].shape[0]
    return nn_record_bytes(w) * pairs / w["n_q"], t2 - t1, t1 - t0, state["rows"].shape[0]


def oracle_nn_state(w):
    from oracle import codebook as ocb
    from oracle import turboquant as otq

    d = w["d"]
    Pi = syn.rotation(d).double().numpy()
    S = syn.sketch(d).double().numpy()
    c = ocb.fit_codebook(d, w["k_idx"])[0]
    db, qs = syn.nn_inputs(20000, 32, d)
    dbn = db.double().numpy()
    e = otq.quantize(dbn, Pi, c, S)
    return {"Pi": Pi, "S": S, "c": c, "rows": dbn[:2048], "n": e["norm"], "r": e["rnorm"],
            "rec": otq.pack(e["idx"], e["sign"], d, w["k_idx"], True), "q": qs.double().numpy()}


def oracle_state(w):
    import numpy as np
    from oracle import codebook as ocb
    from oracle import turboquant as otq

    d = w["d"]
    T = w["T"]
    G = w["hq"] // w["hkv"]
    Pi = (syn.randomized_hadamard(d) if w.get("hadamard") else syn.rotation(d)).double().numpy()
    S = syn.sketch(d).double().numpy()
    from oracle import mixed_rate as omr

    ki, vi, km, vm = w["k_idx"], w["v_idx"], w.get("k_nhi", 0), w.get("v_nhi", 0)
    ck = ocb.fit_codebook(d, ki)[0]
    cv = ocb.fit_codebook(d, vi)[0]
    if km or vm:   # mixed rate: the codebooks of both widths
        ckh, cvh = ocb.fit_codebook(d, ki + 1)[0], ocb.fit_codebook(d, vi + 1)[0]
        ops = {"enc_k": lambda x: omr.quantize(x, Pi, ck, ckh, km, S), "enc_v": lambda x: omr.quantize(x, Pi, cv, cvh, vm),
               "pack_k": lambda e: omr.pack(e["idx"], e["sign"], d, ki, km, True),
               "pack_v": lambda e: omr.pack(e["idx"], None, d, vi, vm, False),
               "unpack_k": lambda r: omr.unpack(r, d, ki, km, True), "unpack_v": lambda r: omr.unpack(r, d, vi, vm, False),
               "logits": lambda q, n, r, i, sg: omr.logits(q, Pi, S, ck, ckh, km, n, r, i, sg),
               "attend": lambda lg, sc, n, i: omr.attend_v(lg, sc, n, i, Pi, cv, cvh, vm)}
    else:
        ops = {"enc_k": lambda x: otq.quantize(x, Pi, ck, S), "enc_v": lambda x: otq.quantize(x, Pi, cv),
               "pack_k": lambda e: otq.pack(e["idx"], e["sign"], d, ki, True),
               "pack_v": lambda e: otq.pack(e["idx"], None, d, vi, False),
               "unpack_k": lambda r: otq.unpack(r, d, ki, True), "unpack_v": lambda r: otq.unpack(r, d, vi, False),
               "logits": lambda q, n, r, i, sg: otq.logits(q, Pi, S, ck, n, r, i, sg),
               "attend": lambda lg, sc, n, i: otq.attend_v(lg, sc, n, i, Pi, cv)}
    g = torch.Generator().manual_seed(5)
    # one KV head of T keys/values of the workload's law, packed once by the oracle
    kfull = torch.randn(T, d, generator=g).to(w["dtype"]).double().numpy()
    vfull = torch.randn(T, d, generator=g).to(w["dtype"]).double().numpy()
    ek = ops["enc_k"](kfull)
    ev = ops["enc_v"](vfull)
    return {"Pi": Pi, "S": S, "ops": ops, "k_rows": kfull[:2048], "v_rows": vfull[:2048],
            "krec": ops["pack_k"](ek), "kn": ek["norm"], "kr": ek["rnorm"],
            "vrec": ops["pack_v"](ev), "vn": ev["norm"],
            "q": torch.randn(G, d, generator=g).double().numpy()}


def run_oracle(w, n_steps, n_warmup, budget_s=None):
    """Returns (logit-scan GB/s, mean step seconds, steps, quantize head-vectors/s)."""
    nn = w.get("kind") == "nn"
    state = oracle_nn_state(w) if nn else oracle_state(w)
    sample_step = oracle_nn_step if nn else oracle_sample_step
    for _ in range(n_warmup):
        sample_step(w, state)
    steps, lg_s, q_s, nbytes, nvec = [], 0.0, 0.0, 0, 0
    t_all = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        b, tl, tq_, nv = sample_step(w, state)
        steps.append(time.perf_counter() - t0)
        lg_s += tl
        q_s += tq_
        nbytes += b
        nvec += nv
        if budget_s is None:
            if len(steps) >= n_steps:
                break
        elif time.perf_counter() - t_all >= budget_s:
            break
    return nbytes / lg_s / 1e9, sum(steps) / len(steps), len(steps), nvec / q_s


def sample_text(w):
    if w.get("kind") == "nn":
        return (f"per step: oracle quantize of 2048 database vectors, unpack + estimator scores of 32 queries over "
                f"20000 packed vectors + top-{w['k']}; value = the workload's packed database bytes x (pairs "
                f"scored / {w['n_q']} queries x {w['n_db']} vectors) / oracle scoring time, i.e. the GB/s of one "
                f"pass of all {w['n_q']} queries at the sampled rate")
    G = w["hq"] // w["hkv"]
    return (f"per step: oracle quantize of 2048 keys + 2048 values, unpack + logits of {G} query heads over one "
            f"KV head's {w['T']} packed keys, softmax.V over that head (1/{w['n_seq'] * w['hkv']} of the "
            f"workload's decode); value = that head's packed key bytes / oracle logit time (unpack + estimator)")


# ----------------------------------------------------------------------------

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = workload(args.workload)

    if args.impl == "reference":
        if rank != 0:
            return
        val, step_s, n, qvps = run_oracle(w, args.steps, args.warmup)
        cores = _threads()
        val = float(f"{val:.4g}")
        line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus, "steps": n,
                "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 2), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": w["name"], "parallelism": "single"},
                "quantize_head_vectors_per_s": round(qvps, 1),
                "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle",
                                 "sample": sample_text(w)},
                "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.workload.startswith("large"):
        result, w = run_large(args, rank, world, local_rank)
    elif args.workload.startswith("nn"):
        result, w = run_nn(args, rank, world, local_rank)
    else:
        result, w = run_tq(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, step_s, n, qvps = run_oracle(w, 0, 1, budget_s=12.0)
        result["cpu_baseline"] = {"value": float(f"{val:.4g}"), "unit": UNIT, "cores": _threads(), "kind": "oracle",
                                  "quantize_head_vectors_per_s": round(qvps, 1),
                                  "sample": sample_text(w) + f"; {n} steps of {step_s:.2f} s"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
