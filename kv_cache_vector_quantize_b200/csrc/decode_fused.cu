// Fused decode attention for d = 128 caches with one query head per KV head:
// the logit of every key, the running softmax and the softmax-weighted sum of
// the values in one pass over the tokens; the logits never leave the SM.
//
// Method: the logit estimator of the key cache (usedby.ai, "TurboQuant:
// Compresion de KV Cache a 3 bits y aceleracion de inferencia en H100",
// "El Pitch"; winningdata.io, "TurboQuant: Google comprime KV cache para 3 bits
// sem perder acuracia", "2. QJL Residual") and the value accumulation
// (zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5 bits per
// channel", paragraph 1):
//   l_t = n_t ( <Pi q, c_K[code_t]> + rho_t sqrt(pi/2)/d <S q, 2 sign_t - 1> ),
//   out = Pi^T sum_t softmax_t(scale l_t) nV_t c_V[codeV_t].
// The kernel writes, per (query head, token chunk), the partial (m, l, acc) of
// the softmax.V chunk kernel (acc in the rotated domain); the merge kernel of
// attend.cu combines the chunks and applies Pi^T.
//
// Work split. One CTA per (token chunk, sequence, KV head). The CTA builds its
// head's lookup tables once (scan_core.cuh) from the query projection, which a
// previous grid computes (this grid is its programmatic dependent). One
// producer thread streams 512-token tiles of key records and of value records
// by bulk copies into two rings of shared-memory stages. Consumer warp w owns
// tokens [32 w, 32 w + 32) of every tile in both phases: lane l computes the
// logit of key 32 w + l from the tables (one key per lane), the warp updates
// its running maximum and turns the logits into softmax weights, and then the
// warp accumulates the values of the same 32 tokens (a half-warp per token,
// 8 coordinates per lane), so no logit or weight crosses warps. The 16 warps'
// (m, l, acc) merge once at the end. Every wait is bounded and reports a
// timeout through the workspace status word. Value codes of 1-3 bits are read
// two coordinates at a time from a table of centroid pairs stored once per
// lane of a 16-lane phase and accumulated with packed two-lane FMAs
// (fma.rn.f32x2), as the softmax.V kernel does, so the sums are bit-equal to
// its; 4-bit codes (a 32 KB pair table would cost a value stage) take one
// centroid and one FMA per coordinate, the same operations.
//
// Shared memory: barriers | key stages (below the 64 KB-aligned table base) |
// staged Pi q, S q | tables (64 KB) | value stages | token weights | pair table.
#include "scan_core.cuh"

namespace tq {

namespace {

using scan::kFD;
using scan::kTabStride;
constexpr int kDWarps = 16;                    // consumer warps
constexpr int kDThreads = 32 * (kDWarps + 1);
constexpr int kDTile = 32 * kDWarps;           // tokens per stage
constexpr int kDMaxStages = 4;                 // per ring
constexpr uint32_t kDBarBytes = 4 * kDMaxStages * 8;   // key full/empty, value full/empty
constexpr uint32_t kDQStage = 1024;            // staged Pi q and S q of the head
constexpr uint32_t kDScratch = kDWarps * 32 * 4;       // token weights
static_assert(kDBarBytes <= 128, "barrier area");

template <int BETA, int VBITS>
struct DLayout {
  static constexpr int KRW = scan::FastKeys<BETA>::RW;         // key record words
  static constexpr int VRW = VBITS * kFD / 32;                  // value record words
  // centroid pairs (c[k & (2^VBITS - 1)], c[k >> VBITS]) at entry 16 k + lane copy, 1-3-bit codes
  static constexpr int kPairs = VBITS <= 3 ? (1 << (2 * VBITS)) * 16 : 0;
  static constexpr uint32_t kPairBytes = kPairs * 8;
  static constexpr uint32_t kKStage = kDTile * (KRW + 2) * 4;   // records, norm, rnorm
  static constexpr uint32_t kVStage = kDTile * (VRW + 1) * 4;   // records, norm
  static constexpr uint32_t kMerge = kDWarps * kFD * 4;         // warp accumulators at the end
  static_assert((KRW * 4) % 16 == 0 && (VRW * 4) % 16 == 0, "bulk copies of whole records");
};

struct DecodeParams {
  const uint32_t *krec;
  const float *knorm, *krnorm;
  const uint32_t *vrec;
  const float *vnorm;
  const float *qrot, *qsk;    // [n_seq][n_heads][128]: Pi q, S q
  const float *cbk, *cbv;     // key and value codebooks
  float *partial;             // [n_seq][n_heads][n_chunks][130]
  uint32_t *status;
  int64_t n_tokens, cap_k, cap_v;
  int n_heads;                // query heads = KV heads
  int n_chunks, tiles_per_chunk;
  float scale;
  uint32_t dyn_bytes;
};

// Shared-memory plan of a launch with dynamic memory starting at dyn0.
template <int BETA, int VBITS>
struct DPlan {
  uint32_t T0, ka, vb, nk, nv, wscr, ptab, end;
  __host__ __device__ DPlan(uint32_t dyn0, uint32_t limit) {
    using L = DLayout<BETA, VBITS>;
    T0 = (dyn0 + kDBarBytes + kTabStride - 1) & ~(kTabStride - 1);
    ka = dyn0 + kDBarBytes;
    const uint32_t below = T0 - kDQStage - ka;
    nk = below / L::kKStage;
    if (nk > (uint32_t)kDMaxStages) nk = kDMaxStages;
    vb = T0 + kTabStride;
    const uint32_t dyn_end = dyn0 + limit;
    const uint32_t tail = kDScratch + L::kPairBytes;
    const uint32_t above = dyn_end > vb + tail ? dyn_end - vb - tail : 0;
    nv = above / L::kVStage;
    if (nv > (uint32_t)kDMaxStages) nv = kDMaxStages;
    uint32_t vend = vb + nv * L::kVStage;
    if (vend < vb + L::kMerge) vend = vb + L::kMerge;   // the merge reuses the value stages
    wscr = vend;
    ptab = wscr + kDScratch;
    end = ptab + L::kPairBytes;
  }
};

template <int BETA, int VBITS>
__global__ void __launch_bounds__(kDThreads, 1) decode_fused_kernel(const DecodeParams p) {
  using L = DLayout<BETA, VBITS>;
  constexpr int KRW = L::KRW, VRW = L::VRW;
  constexpr int LV = 1 << VBITS;
  constexpr int CPL = 8;              // value coordinates per lane (16 lanes per token)
  constexpr int FB = CPL * VBITS;     // value code bits of a lane's coordinates
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float cbk[8], cbv[16];
  __shared__ float mst[kDWarps], lst[kDWarps];

  const uint32_t dyn0 = smem_u32(smem);
  const DPlan<BETA, VBITS> plan(dyn0, p.dyn_bytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk = (int)plan.nk, nv = (int)plan.nv;
  auto kfull = [&](int s) { return dyn0 + 8u * s; };
  auto kempty = [&](int s) { return dyn0 + 8u * (kDMaxStages + s); };
  auto vfull = [&](int s) { return dyn0 + 8u * (2 * kDMaxStages + s); };
  auto vempty = [&](int s) { return dyn0 + 8u * (3 * kDMaxStages + s); };
  if (nk < 2 || nv < 2 || plan.end > dyn0 + p.dyn_bytes) {
    if (tid == 0) {
      pdl_wait();   // a clean status word comes from the previous grid
      atomicOr(p.status, kDevBadShape);   // the launch's shared memory cannot hold this layout
    }
    return;
  }
  const int chunk = blockIdx.x, sk = blockIdx.y;   // sk = seq * n_heads + head (one query head per KV head)
  const int64_t t_begin = (int64_t)chunk * p.tiles_per_chunk * kDTile;
  const int64_t t_end = min(p.n_tokens, t_begin + (int64_t)p.tiles_per_chunk * kDTile);
  const int n_tiles = t_begin < t_end ? (int)((t_end - t_begin + kDTile - 1) / kDTile) : 0;
  const size_t kslot0 = (size_t)sk * p.cap_k, vslot0 = (size_t)sk * p.cap_v;
  // norms arrive with the tiles when their arrays are 16-byte aligned for this head (tiles start
  // 512 tokens apart) and the tile's length is a multiple of 4
  const bool knc = (reinterpret_cast<uintptr_t>(p.knorm + kslot0) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(p.krnorm + kslot0) % 16 == 0);
  const bool vnc = reinterpret_cast<uintptr_t>(p.vnorm + vslot0) % 16 == 0;

  if (tid == 0) {
    for (int s = 0; s < kDMaxStages; ++s) {
      mbar_init(kfull(s), 1);
      mbar_init(kempty(s), kDWarps);
      mbar_init(vfull(s), 1);
      mbar_init(vempty(s), kDWarps);
    }
    mbar_fence_init();
  }
  if (tid < (1 << BETA)) cbk[tid] = p.cbk[tid];
  if (tid < LV) cbv[tid] = p.cbv[tid];
  __syncthreads();

  if (warp == kDWarps) {
    // ------------------------------ producer ------------------------------
    // records are written by earlier grids (not the projection this grid depends on)
    if (lane == 0) {
      int ik = 0, iv = 0, sk_ = 0, sv = 0;
      uint32_t kph = 1u, vph = 1u;   // parities of the empty-barrier phases a stage's reuse waits for
      bool ok = true;
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int64_t t0 = t_begin + (int64_t)i * kDTile;
        const int n = (int)min((int64_t)kDTile, t_end - t0);
        const bool n4 = (n & 3) == 0;
        // key tile
        if (i >= nk && !mbar_wait(kempty(sk_), kph)) {
          ok = false;
          break;
        }
        {
          const uint32_t rb = (uint32_t)n * KRW * 4, st = plan.ka + (uint32_t)sk_ * L::kKStage;
          mbar_arrive_expect_tx(kfull(sk_), rb + (knc && n4 ? 8u * n : 0u));
          bulk_g2s(st, p.krec + (kslot0 + t0) * KRW, rb, kfull(sk_));
          if (knc && n4) {
            bulk_g2s(st + kDTile * KRW * 4, p.knorm + kslot0 + t0, 4u * n, kfull(sk_));
            bulk_g2s(st + kDTile * KRW * 4 + kDTile * 4, p.krnorm + kslot0 + t0, 4u * n, kfull(sk_));
          }
        }
        ++ik;
        if (++sk_ == nk) {
          sk_ = 0;
          kph ^= 1u;
        }
        // value tile
        if (i >= nv && !mbar_wait(vempty(sv), vph)) {
          ok = false;
          break;
        }
        {
          const uint32_t rb = (uint32_t)n * VRW * 4, st = plan.vb + (uint32_t)sv * L::kVStage;
          mbar_arrive_expect_tx(vfull(sv), rb + (vnc && n4 ? 4u * n : 0u));
          bulk_g2s(st, p.vrec + (vslot0 + t0) * VRW, rb, vfull(sv));
          if (vnc && n4) bulk_g2s(st + kDTile * VRW * 4, p.vnorm + vslot0 + t0, 4u * n, vfull(sv));
        }
        ++iv;
        if (++sv == nv) {
          sv = 0;
          vph ^= 1u;
        }
      }
      if (!ok) {
        pdl_wait();
        atomicOr(p.status, kDevTimeout);
      }
      // drain: every issued copy must land before the CTA exits
      for (int i = max(0, ik - nk); i < ik; ++i)
        if (!mbar_wait(kfull(i % nk), (i / nk) & 1)) {
          pdl_wait();
          atomicOr(p.status, kDevTimeout);
          break;
        }
      for (int i = max(0, iv - nv); i < iv; ++i)
        if (!mbar_wait(vfull(i % nv), (i / nv) & 1)) {
          pdl_wait();
          atomicOr(p.status, kDevTimeout);
          break;
        }
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  pdl_wait();   // the query projection (and a clean status word) come from the previous grid
  const float kappa = 1.2533141373155003f / (float)kFD;   // sqrt(pi/2)/d
  float *qv = reinterpret_cast<float *>(smem + (plan.T0 - kDQStage - dyn0));   // [Pi q | S q]
  float *tables = reinterpret_cast<float *>(smem + (plan.T0 - dyn0));
  for (int e = tid; e < 2 * kFD; e += 32 * kDWarps)
    qv[e] = e < kFD ? p.qrot[(size_t)sk * kFD + e] : p.qsk[(size_t)sk * kFD + e - kFD];
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDWarps) : "memory");
  scan::build_tables<BETA, 32 * kDWarps>(qv, qv + kFD, tables, cbk, tid, kappa);
  uint64_t *ptab = reinterpret_cast<uint64_t *>(smem + (plan.ptab - dyn0));
  for (int e2 = tid; e2 < L::kPairs; e2 += 32 * kDWarps) {
    const int key = e2 >> 4;
    ptab[e2] = f2_pack(cbv[key & (LV - 1)], cbv[key >> VBITS]);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDWarps) : "memory");

  float m = -INFINITY, lsum = 0.f, acc[CPL];   // running max (warp-uniform), this lane's share of l
  uint64_t acc2[CPL / 2];                       // coordinate pairs (2 pp, 2 pp + 1), the 1-3-bit codes
#pragma unroll
  for (int a = 0; a < CPL; ++a) acc[a] = 0.f;
#pragma unroll
  for (int pp = 0; pp < CPL / 2; ++pp) acc2[pp] = 0ull;   // (+0, +0)
  const uint32_t lane8 = 8u * (uint32_t)(lane & 15);     // this lane's copy of the pair table
  float *wscr = reinterpret_cast<float *>(smem + (plan.wscr - dyn0));   // [kDWarps][32]
  const int half = lane >> 4, sub = lane & 15;
  const int bit0 = FB * sub, wd = bit0 >> 5, sh = bit0 & 31;
  const bool two = sh + FB > 32;   // the field crosses into word wd + 1 (< VRW)
  const int tw = 32 * warp, k = tw + lane;
  int sk_ = 0, sv = 0;
  uint32_t kph = 0u, vph = 0u;
  bool ok = true;

  for (int i = 0; i < n_tiles && ok; ++i) {
    const int64_t t0 = t_begin + (int64_t)i * kDTile;
    const int n = (int)min((int64_t)kDTile, t_end - t0);
    const bool valid = k < n, n4 = (n & 3) == 0;
    // ---- logit of key k ----
    if (!mbar_wait(kfull(sk_), kph)) {
      atomicOr(p.status, kDevTimeout);
      ok = false;
      break;
    }
    const unsigned char *kst = smem + (plan.ka + (uint32_t)sk_ * L::kKStage - dyn0);
    uint32_t w[KRW];
    float nrm = 0.f, rho = 0.f;
    if (valid) {
      const uint4 *src = reinterpret_cast<const uint4 *>(kst + (size_t)k * KRW * 4);
#pragma unroll
      for (int j = 0; j < KRW / 4; ++j) {
        const uint4 v4 = src[j];
        w[4 * j] = v4.x;
        w[4 * j + 1] = v4.y;
        w[4 * j + 2] = v4.z;
        w[4 * j + 3] = v4.w;
      }
      if (knc && n4) {
        nrm = reinterpret_cast<const float *>(kst + kDTile * KRW * 4)[k];
        rho = reinterpret_cast<const float *>(kst + kDTile * KRW * 4 + kDTile * 4)[k];
      } else {
        nrm = __ldg(p.knorm + kslot0 + t0 + k);
        rho = __ldg(p.krnorm + kslot0 + t0 + k);
      }
    } else {
#pragma unroll
      for (int j = 0; j < KRW; ++j) w[j] = 0u;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(kempty(sk_));   // this warp is done with the key stage
    if (++sk_ == nk) {
      sk_ = 0;
      kph ^= 1u;
    }
    float lg[1];
    scan::key_logits<BETA, 1>(w, lane, plan.T0, 1, nrm, rho, lg);
    // ---- running softmax over the warp's tokens ----
    const float z = valid ? p.scale * lg[0] : -INFINITY;
    const float mx = fmaxf(m, warp_max(z));
    // mx is -inf only while every logit seen is -inf: nothing has weight yet
    const float f = mx == -INFINITY ? 0.f : expf(m - mx);
    const float e = mx == -INFINITY ? 0.f : expf(z - mx);
    m = mx;
    lsum = fmaf(lsum, f, e);
    if constexpr (L::kPairs > 0) {
      const uint64_t f2 = f2_pack(f, f);
#pragma unroll
      for (int pp = 0; pp < CPL / 2; ++pp) acc2[pp] = f2_mul(acc2[pp], f2);
    } else {
#pragma unroll
      for (int a = 0; a < CPL; ++a) acc[a] *= f;
    }
    // ---- values of the warp's 32 tokens ----
    if (!mbar_wait(vfull(sv), vph)) {
      atomicOr(p.status, kDevTimeout);
      ok = false;
      break;
    }
    const unsigned char *vst = smem + (plan.vb + (uint32_t)sv * L::kVStage - dyn0);
    float vn = 0.f;
    if (valid) vn = (vnc && n4) ? reinterpret_cast<const float *>(vst + kDTile * VRW * 4)[k] : __ldg(p.vnorm + vslot0 + t0 + k);
    wscr[k] = e * vn;   // 0 for a token past the end
    __syncwarp();
    const uint32_t *rs = reinterpret_cast<const uint32_t *>(vst) + (size_t)(tw + half) * VRW;
    const int np = (min(32, n - tw) + 1) >> 1;   // token pairs of this warp (warp-uniform, may be <= 0)
    // token pair j of this warp: two tokens, one per half-warp
    auto pair_step = [&](int j) {
      const uint32_t *rec = rs + 2 * j * VRW;
      const uint32_t lo = rec[wd];
      const uint32_t hi = two ? rec[wd + 1] : 0u;
      const uint32_t bits = __funnelshift_r(lo, hi, sh);
      const float wt = wscr[tw + 2 * j + half];
      if constexpr (L::kPairs > 0) {
        const uint64_t w2 = f2_pack(wt, wt);
#pragma unroll
        for (int pp = 0; pp < CPL / 2; ++pp) {
          // byte offset of the pair (codes 2 pp, 2 pp + 1) in the table: key * 128 (+ the lane copy)
          constexpr uint32_t kMask = 128u * (LV * LV - 1);
          const int shr = 2 * VBITS * pp - 7;
          const uint32_t off = ((shr >= 0 ? bits >> (shr & 31) : bits << ((-shr) & 31)) & kMask) | lane8;
          const uint64_t cv = *reinterpret_cast<const uint64_t *>(reinterpret_cast<const unsigned char *>(ptab) + off);
          acc2[pp] = f2_fma(w2, cv, acc2[pp]);
        }
      } else {
#pragma unroll
        for (int a = 0; a < CPL; ++a) acc[a] = fmaf(wt, cbv[(bits >> (VBITS * a)) & (LV - 1)], acc[a]);
      }
    };
    if (np == 16) {
      // a whole warp's 32 tokens: fully unrolled (immediate addresses, no loop counter)
#pragma unroll
      for (int j = 0; j < 16; ++j) pair_step(j);
    } else {
#pragma unroll 2
      for (int j = 0; j < np; ++j) pair_step(j);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(vempty(sv));   // this warp is done with the value stage and its weights
    if (++sv == nv) {
      sv = 0;
      vph ^= 1u;
    }
  }
  if constexpr (L::kPairs > 0) {
#pragma unroll
    for (int pp = 0; pp < CPL / 2; ++pp) f2_unpack(acc2[pp], acc[2 * pp], acc[2 * pp + 1]);
  }
  // the two half-warps accumulated different tokens of the same coordinates
#pragma unroll
  for (int a = 0; a < CPL; ++a) acc[a] += __shfl_xor_sync(0xffffffffu, acc[a], 16);

  // Only now may the merge grid become resident (it stages its matrix while the last CTAs finish):
  // its CTAs wait for this whole grid, and resident earlier they would hold registers and shared
  // memory on SMs that this grid's later waves need.
  pdl_launch_dependents();
  // ---- merge the warps: M = max_w m_w, each warp scaled by e^{m_w - M} ----
  lsum = warp_sum(lsum);
  if (lane == 0) {
    mst[warp] = m;
    lst[warp] = lsum;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDWarps) : "memory");   // also: every value stage has been consumed
  float *mg = reinterpret_cast<float *>(smem + (plan.vb - dyn0));    // [kDWarps][128], over the value stages
  float mc = -INFINITY;
  for (int w2 = 0; w2 < kDWarps; ++w2) mc = fmaxf(mc, mst[w2]);
  const float sc = mc == -INFINITY ? 0.f : expf(m - mc);
  if (half == 0) {
    float4 *dst = reinterpret_cast<float4 *>(mg + warp * kFD + CPL * sub);
    dst[0] = make_float4(acc[0] * sc, acc[1] * sc, acc[2] * sc, acc[3] * sc);
    dst[1] = make_float4(acc[4] * sc, acc[5] * sc, acc[6] * sc, acc[7] * sc);
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDWarps) : "memory");
  if (!ok) return;
  float *part = p.partial + ((size_t)sk * p.n_chunks + chunk) * (size_t)(kFD + 2);
  if (tid < kFD) {
    float v = 0.f;
    for (int w2 = 0; w2 < kDWarps; ++w2) v += mg[w2 * kFD + tid];
    part[2 + tid] = v;
  }
  if (tid == 0) {
    float lc = 0.f;
    for (int w2 = 0; w2 < kDWarps; ++w2) lc += mc == -INFINITY ? 0.f : lst[w2] * expf(mst[w2] - mc);
    part[0] = mc;
    part[1] = lc;
  }
}

constexpr uint32_t kDDyn0 = 1024;   // reserved shared memory below the dynamic window on sm_100

template <int BETA, int VBITS>
bool fits(uint32_t limit) {
  const DPlan<BETA, VBITS> pl(kDDyn0, limit);
  return pl.nk >= 2 && pl.nv >= 2 && pl.end <= kDDyn0 + limit;
}

template <int BETA, int VBITS>
cudaError_t launch_d(DecodeParams p, int n_seq, uint32_t limit, cudaStream_t st) {
  const DPlan<BETA, VBITS> pl(kDDyn0, limit);
  p.dyn_bytes = pl.end - kDDyn0;
  auto kern = decode_fused_kernel<BETA, VBITS>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), p.dyn_bytes);
  if (e != cudaSuccess) return e;
  // a programmatic dependent of the query projection: the producer streams tiles meanwhile
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)p.n_chunks, (unsigned)(n_seq * p.n_heads));
  cfg.blockDim = dim3(kDThreads);
  cfg.dynamicSmemBytes = p.dyn_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int BETA>
cudaError_t launch_d_v(const DecodeParams &p, int vbits, int n_seq, uint32_t limit, cudaStream_t st) {
  switch (vbits) {
    case 1: return launch_d<BETA, 1>(p, n_seq, limit, st);
    case 2: return launch_d<BETA, 2>(p, n_seq, limit, st);
    case 3: return launch_d<BETA, 3>(p, n_seq, limit, st);
    default: return launch_d<BETA, 4>(p, n_seq, limit, st);
  }
}

template <int BETA>
bool fits_v(int vbits, uint32_t limit) {
  switch (vbits) {
    case 1: return fits<BETA, 1>(limit);
    case 2: return fits<BETA, 2>(limit);
    case 3: return fits<BETA, 3>(limit);
    default: return fits<BETA, 4>(limit);
  }
}

}  // namespace

namespace {
__global__ void status_or_kernel(uint32_t *dst, const uint32_t *a, const uint32_t *b) { *dst = *a | *b; }
}  // namespace

// dst = *a | *b on the device (one thread), in stream order.
cudaError_t launch_status_or(uint32_t *dst, const uint32_t *a, const uint32_t *b, cudaStream_t st) {
  status_or_kernel<<<1, 1, 0, st>>>(dst, a, b);
  return cudaGetLastError();
}

bool decode_fused_supported(int d, int kbits, int vbits, int n_q_heads, int n_kv_heads, const void *krec,
                            const void *vrec, size_t limit) {
  if (d != kFD || n_q_heads != n_kv_heads || vbits < 1 || vbits > 4) return false;
  if ((reinterpret_cast<uintptr_t>(krec) | reinterpret_cast<uintptr_t>(vrec)) & 15) return false;
  const uint32_t lim = (uint32_t)limit;
  switch (kbits) {
    case 1: return fits_v<1>(vbits, lim);
    case 2: return fits_v<2>(vbits, lim);
    default: return false;   // 3-bit key codes: the key ring does not fit twice below the tables
  }
}

cudaError_t launch_decode_fused(const DecodeFusedArgs &a, cudaStream_t st) {
  DecodeParams p{};
  p.krec = a.krec;
  p.knorm = a.knorm;
  p.krnorm = a.krnorm;
  p.vrec = a.vrec;
  p.vnorm = a.vnorm;
  p.qrot = a.qrot;
  p.qsk = a.qsk;
  p.cbk = a.cbk;
  p.cbv = a.cbv;
  p.partial = a.partial;
  p.status = a.status;
  p.n_tokens = a.n_tokens;
  p.cap_k = a.cap_k;
  p.cap_v = a.cap_v;
  p.n_heads = a.n_heads;
  p.n_chunks = a.n_chunks;
  p.tiles_per_chunk = (int)(a.chunk / kDTile);
  p.scale = a.scale;
  const uint32_t lim = (uint32_t)a.smem_limit;
  return a.kbits == 1 ? launch_d_v<1>(p, a.vbits, a.n_seq, lim, st) : launch_d_v<2>(p, a.vbits, a.n_seq, lim, st);
}

}  // namespace tq
