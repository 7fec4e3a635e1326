// Softmax-weighted value accumulation for d = 128 value caches, streamed
// through shared memory by bulk copies, with a running (online) softmax.
//
// Estimator (zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to
// 3.5 bits per channel", paragraph 1: values are stored MSE-only, norm + codes).
// With p = softmax(scale * logits):  out = Pi^T sum_t p_t n_t c[code_t].
// This kernel produces, per (query head, token chunk), the partial
// (m, l, acc) with m = max_t scale l_t, l = sum_t e^{scale l_t - m} and
// acc = sum_t e^{scale l_t - m} n_t c[code_t] (rotated domain); the merge
// kernel of attend.cu combines the chunks and applies Pi^T.
//
// Work split. One CTA per (token chunk, sequence, KV head, block of <= 4 query
// heads). One producer thread streams 512-token tiles of records with
// cp.async.bulk into a ring of shared-memory stages guarded by mbarriers; 16
// consumer warps take 32 tokens of each tile. Each warp keeps its own running
// maximum per query head (warp-uniform) and rescales its accumulators when it
// grows, so the tiles need no block-wide barrier; the 16 warps' states are
// merged once at the end. The logits and norms of the next tile are loaded
// while the current one is accumulated. In the accumulation loop each
// half-warp takes one token and a lane owns 8 consecutive coordinates: per
// token it reads its code bits once (an 8 * BITS-bit field), the token's
// weights for all query heads with one 16-byte load (two addresses per warp),
// and one centroid per coordinate, shared by the query heads. Tokens past the
// end of a tile carry weight 0, so both half-warps run the same iterations.
#include "common.cuh"

namespace tq {

namespace {

constexpr int kVD = 128;                       // head dimension of this kernel
constexpr int kVWarps = 16;                    // consumer warps
constexpr int kVThreads = 32 * (kVWarps + 1);
constexpr int kVTile = 32 * kVWarps;           // tokens per stage
constexpr int kVStages = 4;
constexpr int kVMaxQ = 4;
constexpr uint32_t kVBarBytes = 128;           // full[kVStages], empty[kVStages], padded

template <int BITS>
struct VTile {
  static constexpr int RW = BITS * kVD / 32;                    // record words (no sign field)
  static constexpr uint32_t kStageBytes = kVTile * RW * 4;      // 8 .. 32 KB
  static constexpr uint32_t kStages = kVStages * kStageBytes;
  static constexpr uint32_t kMerge = kVWarps * kVMaxQ * kVD * 4;   // 32 KB, aliases the stages
  static constexpr uint32_t kScratch = kVWarps * 32 * 16;          // per-warp token weights (float4)
  static constexpr uint32_t kBytes = kVBarBytes + (kStages > kMerge ? kStages : kMerge) + kScratch;
  static_assert((RW * 4) % 16 == 0, "bulk copies of whole records need 16-byte multiples");
  static_assert(kVBarBytes >= 2 * kVStages * 8, "barrier area");
};

struct VFastParams {
  AttendParams p;
  int tiles_per_chunk;
};

template <int BITS, int QMAX>
__global__ void __launch_bounds__(kVThreads, 1) attend_fast_kernel(const VFastParams fp) {
  using T = VTile<BITS>;
  constexpr int RW = T::RW;
  constexpr int L = 1 << BITS;
  constexpr int CPL = 8;          // coordinates per lane (16 lanes per token)
  constexpr int FB = CPL * BITS;  // code bits of a lane's coordinates
  const AttendParams &p = fp.p;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float cbs[16];
  __shared__ float mst[kVWarps][kVMaxQ], lst[kVWarps][kVMaxQ];

  const uint32_t sb = smem_u32(smem);
  auto full_bar = [&](int s) { return sb + 8u * s; };
  auto empty_bar = [&](int s) { return sb + 8u * (kVStages + s); };
  unsigned char *stages = smem + kVBarBytes;
  float4 *wscr = reinterpret_cast<float4 *>(smem + T::kBytes - T::kScratch);   // [kVWarps][32]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, unit = blockIdx.y;
  const int qb = unit % p.qblocks, sk = unit / p.qblocks;
  const int seq = sk / p.n_kv_heads, kvh = sk - seq * p.n_kv_heads;
  const int h0 = kvh * p.group + qb * p.q_per_cta;
  const int nq = min(p.q_per_cta, p.group - qb * p.q_per_cta);
  const int64_t t_begin = (int64_t)chunk * fp.tiles_per_chunk * kVTile;
  const int64_t t_end = min(p.n_tokens, t_begin + (int64_t)fp.tiles_per_chunk * kVTile);
  const int n_tiles = t_begin < t_end ? (int)((t_end - t_begin + kVTile - 1) / kVTile) : 0;
  const size_t slot0 = (size_t)sk * p.capacity;

  pdl_launch_dependents();   // the merge may become resident and stage its matrix meanwhile
  if (tid == 0) {
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kVWarps);
    }
    mbar_fence_init();
  }
  if (tid < L) cbs[tid] = p.codebook[tid];
  __syncthreads();

  if (warp == kVWarps) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kVStages;
        if (i >= kVStages && !mbar_wait(empty_bar(s), ((i / kVStages) - 1) & 1)) {
          atomicOr(p.status, kDevTimeout);
          break;
        }
        const int64_t t0 = t_begin + (int64_t)i * kVTile;
        const uint32_t bytes = (uint32_t)min((int64_t)kVTile, t_end - t0) * RW * 4;
        mbar_arrive_expect_tx(full_bar(s), bytes);
        bulk_g2s(sb + kVBarBytes + (uint32_t)s * T::kStageBytes, p.records + (slot0 + t0) * RW, bytes, full_bar(s));
        ++issued;
      }
      // drain: every issued copy must land before the CTA exits
      for (int i = max(0, issued - kVStages); i < issued; ++i)
        if (!mbar_wait(full_bar(i % kVStages), (i / kVStages) & 1)) {
          atomicOr(p.status, kDevTimeout);
          break;
        }
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  // running max (warp-uniform), this lane's share of l, coordinates 8 (lane mod 16) + a
  float m[QMAX], l[QMAX], acc[CPL][QMAX];
#pragma unroll
  for (int qq = 0; qq < QMAX; ++qq) {
    m[qq] = -INFINITY;
    l[qq] = 0.f;
#pragma unroll
    for (int a = 0; a < CPL; ++a) acc[a][qq] = 0.f;
  }
  const float *lrow[QMAX];
#pragma unroll
  for (int qq = 0; qq < QMAX; ++qq) lrow[qq] = p.logits + ((size_t)seq * p.n_q_heads + h0 + min(qq, nq - 1)) * p.n_tokens;
  const int half = lane >> 4, sub = lane & 15;
  const int bit0 = FB * sub, wd = bit0 >> 5, sh = bit0 & 31;
  const bool two = sh + FB > 32;   // the field crosses into word wd + 1 (< RW)
  const int tw = 32 * warp;        // this warp's first token in a tile
  const int k = tw + lane;         // this lane's token for the weights
  // logits (times scale) and norm of this lane's token in tile i
  auto fetch = [&](int i, float (&z)[QMAX], float &nrm) {
    const int64_t t0 = t_begin + (int64_t)i * kVTile;
    const bool valid = t0 + k < t_end;
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) z[qq] = (valid && qq < nq) ? p.scale * __ldg(lrow[qq] + t0 + k) : -INFINITY;
    nrm = valid ? __ldg(p.norm + slot0 + t0 + k) : 0.f;
  };
  float zn[QMAX], nn = 0.f;
  if (n_tiles > 0) fetch(0, zn, nn);
  bool ok = true;

  for (int i = 0; i < n_tiles && ok; ++i) {
    const int s = i % kVStages;
    const int n = (int)min((int64_t)kVTile, t_end - (t_begin + (int64_t)i * kVTile));
    float z[QMAX];
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) z[qq] = zn[qq];
    const float nrm = nn;
    if (i + 1 < n_tiles) fetch(i + 1, zn, nn);   // in flight during this tile
    float wq[QMAX];
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) {
      const float mx = fmaxf(m[qq], warp_max(z[qq]));
      // mx is -inf only while every logit seen is -inf: nothing has weight yet
      const float f = mx == -INFINITY ? 0.f : expf(m[qq] - mx);
      const float e = mx == -INFINITY ? 0.f : expf(z[qq] - mx);
      m[qq] = mx;
      l[qq] = fmaf(l[qq], f, e);
#pragma unroll
      for (int a = 0; a < CPL; ++a) acc[a][qq] *= f;
      wq[qq] = e * nrm;   // 0 for a token past the end
    }
    wscr[tw + lane] = make_float4(wq[0], QMAX > 1 ? wq[1 % QMAX] : 0.f, QMAX > 2 ? wq[2 % QMAX] : 0.f,
                                  QMAX > 3 ? wq[3 % QMAX] : 0.f);
    __syncwarp();
    if (!mbar_wait(full_bar(s), (i / kVStages) & 1)) {
      atomicOr(p.status, kDevTimeout);
      ok = false;
      break;
    }
    // token tw + 2 j + half of the tile for this half-warp (records past n hold stale codes, weight 0)
    const uint32_t *rs = reinterpret_cast<const uint32_t *>(stages + (size_t)s * T::kStageBytes) + (size_t)(tw + half) * RW;
    const int np = (min(32, n - tw) + 1) >> 1;   // token pairs of this warp (warp-uniform, may be <= 0)
#pragma unroll 2
    for (int j = 0; j < np; ++j) {
      const uint32_t *rec = rs + 2 * j * RW;
      const uint32_t lo = rec[wd];
      const uint32_t hi = two ? rec[wd + 1] : 0u;
      const uint32_t bits = __funnelshift_r(lo, hi, sh);
      const float4 w4 = wscr[tw + 2 * j + half];
      const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int a = 0; a < CPL; ++a) {
        // byte offset of code a in the centroid table: one shift and one mask
        constexpr uint32_t kMask = 4u * (L - 1);
        const int shr = BITS * a - 2;
        const uint32_t off = (shr >= 0 ? bits >> (shr & 31) : bits << ((-shr) & 31)) & kMask;
        const float cv = *reinterpret_cast<const float *>(reinterpret_cast<const unsigned char *>(cbs) + off);
#pragma unroll
        for (int qq = 0; qq < QMAX; ++qq) acc[a][qq] = fmaf(wv[qq], cv, acc[a][qq]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));   // this warp is done with the stage and its weights
  }
  // the two half-warps accumulated different tokens of the same coordinates
#pragma unroll
  for (int a = 0; a < CPL; ++a)
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) acc[a][qq] += __shfl_xor_sync(0xffffffffu, acc[a][qq], 16);

  // ---- merge the warps: M = max_w m_w, each warp scaled by e^{m_w - M} ----
#pragma unroll
  for (int qq = 0; qq < QMAX; ++qq) l[qq] = warp_sum(l[qq]);
  if (lane == 0) {
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) {
      mst[warp][qq] = m[qq];
      lst[warp][qq] = l[qq];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kVWarps) : "memory");   // also: every stage has been consumed
  float *mg = reinterpret_cast<float *>(stages);   // [kVWarps][kVMaxQ][kVD], over the stages
#pragma unroll
  for (int qq = 0; qq < QMAX; ++qq) {
    float mc = -INFINITY;
    for (int w = 0; w < kVWarps; ++w) mc = fmaxf(mc, mst[w][qq]);
    const float sc = mc == -INFINITY ? 0.f : expf(m[qq] - mc);
    if (half == 0) {
      float4 *dst = reinterpret_cast<float4 *>(mg + (warp * kVMaxQ + qq) * kVD + CPL * sub);
      dst[0] = make_float4(acc[0][qq] * sc, acc[1][qq] * sc, acc[2][qq] * sc, acc[3][qq] * sc);
      dst[1] = make_float4(acc[4][qq] * sc, acc[5][qq] * sc, acc[6][qq] * sc, acc[7][qq] * sc);
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kVWarps) : "memory");
  if (!ok) return;
  for (int e = tid; e < nq * kVD; e += 32 * kVWarps) {
    const int qq = e / kVD, ii = e - qq * kVD;
    float v = 0.f;
    for (int w = 0; w < kVWarps; ++w) v += mg[(w * kVMaxQ + qq) * kVD + ii];
    const size_t hrow = (size_t)seq * p.n_q_heads + h0 + qq;
    p.partial[(hrow * p.n_chunks + chunk) * (size_t)(kVD + 2) + 2 + ii] = v;
  }
  if (tid < nq) {
    float mc = -INFINITY;
    for (int w = 0; w < kVWarps; ++w) mc = fmaxf(mc, mst[w][tid]);
    float lc = 0.f;
    for (int w = 0; w < kVWarps; ++w) lc += mc == -INFINITY ? 0.f : lst[w][tid] * expf(mst[w][tid] - mc);
    const size_t hrow = (size_t)seq * p.n_q_heads + h0 + tid;
    float *part = p.partial + (hrow * p.n_chunks + chunk) * (size_t)(kVD + 2);
    part[0] = mc;
    part[1] = lc;
  }
}

template <int BITS, int QMAX>
cudaError_t launch_vf(const VFastParams &fp, int units, cudaStream_t st) {
  auto kern = attend_fast_kernel<BITS, QMAX>;
  const size_t smem = VTile<BITS>::kBytes;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)fp.p.n_chunks, (unsigned)units), kVThreads, smem, st>>>(fp);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_vf_q(const VFastParams &fp, int units, cudaStream_t st) {
  switch (fp.p.q_per_cta) {
    case 1: return launch_vf<BITS, 1>(fp, units, st);
    case 2: return launch_vf<BITS, 2>(fp, units, st);
    case 3: return launch_vf<BITS, 3>(fp, units, st);
    default: return launch_vf<BITS, 4>(fp, units, st);
  }
}

}  // namespace

bool attend_fast_supported(int d, int bits, int q_per_cta, const void *records) {
  return d == kVD && bits >= 1 && bits <= 4 && q_per_cta >= 1 && q_per_cta <= kVMaxQ &&
         (reinterpret_cast<uintptr_t>(records) & 15) == 0;
}

// Tokens per chunk (a multiple of the 512-token tile): the split of every
// unit's tiles into equal chunks that minimises the busiest SM's tile count
// (whole waves of one CTA per SM times tiles per chunk).
int64_t attend_fast_chunk(int64_t n_tokens, int units) {
  const int64_t tpu = (n_tokens + kVTile - 1) / kVTile;
  const int64_t slots = device_sm_count();
  int64_t best_tpc = tpu, best_cost = INT64_MAX;
  const int64_t max_nc = tpu < 8 * slots ? tpu : 8 * slots;
  for (int64_t nc = 1; nc <= max_nc; ++nc) {
    const int64_t tpc = (tpu + nc - 1) / nc;
    const int64_t ctas = (int64_t)units * ((tpu + tpc - 1) / tpc);
    const int64_t cost = ((ctas + slots - 1) / slots) * tpc;
    if (cost < best_cost) {
      best_cost = cost;
      best_tpc = tpc;
    }
  }
  return best_tpc * kVTile;
}

cudaError_t launch_attend_fast(const AttendParams &p, int bits, int n_seq, cudaStream_t st) {
  VFastParams fp{};
  fp.p = p;
  fp.tiles_per_chunk = (int)(p.chunk / kVTile);
  const int units = n_seq * p.n_kv_heads * p.qblocks;
  switch (bits) {
    case 1: return launch_vf_q<1>(fp, units, st);
    case 2: return launch_vf_q<2>(fp, units, st);
    case 3: return launch_vf_q<3>(fp, units, st);
    default: return launch_vf_q<4>(fp, units, st);
  }
}

}  // namespace tq
