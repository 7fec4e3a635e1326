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
// token it reads its code bits once (an 8 * BITS-bit field) and the token's
// weights for all query heads (stored as (w, w) pairs), then looks up its 8
// centroids two at a time in a table of centroid pairs indexed by two
// consecutive codes (2 * BITS bits) and accumulates them with packed
// two-lane float32 FMAs (fma.rn.f32x2: the same two round-to-nearest FMAs as
// two scalar FMAs, in the same order). The pair table is stored once per lane
// of a 16-lane shared-memory phase (entry (key, lane) at (16 key + lane) * 8
// bytes), so the half-warp's random lookups never conflict. Tokens past the
// end of a tile carry weight 0, so both half-warps run the same iterations.
//
// Mixed rate (MIXED, fractional bits per channel with the first 64 of the 128
// coordinates at BITS + 1 code bits): lanes 0..7 of a half-warp hold
// coordinates of the wider group (8 (BITS+1)-bit codes), lanes 8..15 of the
// narrower one; each lane has its own field position and width and reads its
// group's pair table (the wider group's first, then the narrower's), with the
// same instruction count per pair. A mixed record is not a multiple of 16
// bytes, so a tile with an odd number of tokens gets its last record by plain
// loads from the producer before the bulk copy of the others.
#include "common.cuh"

namespace tq {

namespace {

constexpr int kVD = 128;                       // head dimension of this kernel
constexpr int kVWarps = 16;                    // consumer warps
constexpr int kVThreads = 32 * (kVWarps + 1);
constexpr int kVTile = 32 * kVWarps;           // tokens per stage
constexpr int kVStages = 4;
constexpr int kVMaxQ = 4;
constexpr uint32_t kVBarBytes = 128;           // full[kVStages], empty[kVStages], the test hook's barrier

template <int BITS, bool MIXED = false>
struct VTile {
  // record words (no sign field); mixed: 64 coordinates at BITS + 1 bits, 64 at BITS
  static constexpr int RW = MIXED ? 2 * (2 * BITS + 1) : BITS * kVD / 32;
  static constexpr uint32_t kStageBytes = kVTile * RW * 4;      // 8 .. 32 KB
  static constexpr uint32_t kStages = kVStages * kStageBytes;
  static constexpr uint32_t kMerge = kVWarps * kVMaxQ * kVD * 4;   // 32 KB, aliases the stages
  static constexpr uint32_t kScratch = kVWarps * 32 * kVMaxQ * 8;  // per-warp token weights ((w, w) per head)
  // centroid-pair table entries, 16 lane copies (mixed: the wider group's table, then the narrower's)
  static constexpr int kPairsHi = MIXED ? (1 << (2 * (BITS + 1))) * 16 : 0;
  static constexpr int kPairs = kPairsHi + (1 << (2 * BITS)) * 16;
  static constexpr uint32_t kBytes = kVBarBytes + (kStages > kMerge ? kStages : kMerge) + kScratch;
  static_assert(MIXED || (RW * 4) % 16 == 0, "bulk copies of whole records need 16-byte multiples");
  static_assert(kStageBytes % 16 == 0, "stage slots 16-byte aligned");
  static_assert(kVBarBytes >= (2 * kVStages + 1) * 8, "barrier area");
};

struct VFastParams {
  AttendParams p;
  int tiles_per_chunk;
};

template <int BITS, int QMAX, bool MIXED = false>
__global__ void __launch_bounds__(kVThreads, 1) attend_fast_kernel(const VFastParams fp) {
  using T = VTile<BITS, MIXED>;
  constexpr int RW = T::RW;
  constexpr int L = 1 << BITS;
  constexpr int CPL = 8;          // coordinates per lane (16 lanes per token)
  constexpr int FB = CPL * BITS;  // code bits of a lane's coordinates (integer rate)
  const AttendParams &p = fp.p;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float cbs[48];       // the BITS codebook at 0, the BITS + 1 codebook (mixed) at 16
  __shared__ float mst[kVWarps][kVMaxQ], lst[kVWarps][kVMaxQ];
  // (c[k & (L-1)], c[k >> BITS]) at entry 16 k + lane copy; static, so a lookup's address is the
  // byte offset plus an immediate
  __shared__ __align__(128) uint64_t ptab[T::kPairs];

  const uint32_t sb = smem_u32(smem);
  auto full_bar = [&](int s) { return sb + 8u * s; };
  auto empty_bar = [&](int s) { return sb + 8u * (kVStages + s); };
  const uint32_t stall_bar = sb + 8u * (2 * kVStages);   // the failure-detection hook's: nothing completes it
  const uint32_t tries = p.stall_tries ? p.stall_tries : kSpinLimit;
  unsigned char *stages = smem + kVBarBytes;
  uint64_t *wscr = reinterpret_cast<uint64_t *>(smem + T::kBytes - T::kScratch);   // [kVWarps][32][kVMaxQ]

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

  if (tid == 0) {
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kVWarps);
    }
    mbar_init(stall_bar, 1);
    mbar_fence_init();
  }
  if (tid < L) cbs[tid] = p.codebook[tid];
  if (MIXED && tid < 2 * L) cbs[16 + tid] = p.codebook[L + tid];
  __syncthreads();
  for (int e = tid; e < T::kPairs; e += kVThreads) {
    if (e < T::kPairsHi) {   // the wider group's pairs (mixed only)
      const int key = e >> 4;
      ptab[e] = f2_pack(cbs[16 + (key & (2 * L - 1))], cbs[16 + (key >> (BITS + 1))]);
    } else {
      const int key = (e - T::kPairsHi) >> 4;
      ptab[e] = f2_pack(cbs[key & (L - 1)], cbs[key >> BITS]);
    }
  }
  __syncthreads();

  if (warp == kVWarps) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kVStages;
        if (i >= kVStages && !mbar_wait_n(empty_bar(s), ((i / kVStages) - 1) & 1, tries)) {
          atomicOr(p.status, kDevTimeout);
          break;
        }
        const int64_t t0 = t_begin + (int64_t)i * kVTile;
        int nrec = (int)min((int64_t)kVTile, t_end - t0);
        if (MIXED && (nrec * RW * 4) % 16 != 0) {
          // the last record by plain loads (before the arrival that releases the stage), the rest by copy
          --nrec;
          const uint32_t *src = p.records + (slot0 + t0 + nrec) * RW;
          uint32_t *dst = reinterpret_cast<uint32_t *>(stages + (size_t)s * T::kStageBytes) + (size_t)nrec * RW;
#pragma unroll
          for (int w = 0; w < RW; ++w) dst[w] = __ldg(src + w);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // ordered with the copy engine's writes
        }
        const uint32_t bytes = (uint32_t)nrec * RW * 4;
        mbar_arrive_expect_tx(full_bar(s), bytes);
        if (bytes > 0)
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
  // running max (warp-uniform), this lane's share of l, coordinates 8 (lane mod 16) + 2 pp + {0, 1}
  float m[QMAX], l[QMAX];
  uint64_t acc2[CPL / 2][QMAX];
#pragma unroll
  for (int qq = 0; qq < QMAX; ++qq) {
    m[qq] = -INFINITY;
    l[qq] = 0.f;
#pragma unroll
    for (int pp = 0; pp < CPL / 2; ++pp) acc2[pp][qq] = 0ull;   // (+0, +0)
  }
  const float *lrow[QMAX];
#pragma unroll
  for (int qq = 0; qq < QMAX; ++qq) lrow[qq] = p.logits + ((size_t)seq * p.n_q_heads + h0 + min(qq, nq - 1)) * p.n_tokens;
  const int half = lane >> 4, sub = lane & 15;
  // this lane's code field: integer rate FB bits at FB * sub; mixed: lanes 0..7 hold 8 codes of
  // BITS + 1 bits at 8 (BITS+1) sub, lanes 8..15 8 codes of BITS bits after the 64 wider codes
  const bool wide = MIXED && sub < 8;
  const int lb = wide ? BITS + 1 : BITS;
  const int bit0 = !MIXED ? FB * sub : wide ? 8 * (BITS + 1) * sub : 64 * (BITS + 1) + 8 * BITS * (sub - 8);
  const int wd = bit0 >> 5, sh = bit0 & 31;
  const bool two = sh + 8 * lb > 32;   // the field crosses into word wd + 1 (< RW)
  // mixed: per lane, the pair key mask (shifted to byte offset 128 key) and the table base (the
  // narrower group's table starts after the wider one's, a power of two of bytes)
  const uint32_t kmask_l = 128u * ((1u << (2 * lb)) - 1u);
  const uint32_t tbase_l = (MIXED && !wide ? 8u * (uint32_t)T::kPairsHi : 0u) | (8u * sub);
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
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) {
      const float mx = fmaxf(m[qq], warp_max(z[qq]));
      // mx is -inf only while every logit seen is -inf: nothing has weight yet
      const float f = mx == -INFINITY ? 0.f : expf(m[qq] - mx);
      const float e = mx == -INFINITY ? 0.f : expf(z[qq] - mx);
      m[qq] = mx;
      l[qq] = fmaf(l[qq], f, e);
      const uint64_t f2 = f2_pack(f, f);
#pragma unroll
      for (int pp = 0; pp < CPL / 2; ++pp) acc2[pp][qq] = f2_mul(acc2[pp][qq], f2);
      const float w = e * nrm;   // 0 for a token past the end
      wscr[(tw + lane) * kVMaxQ + qq] = f2_pack(w, w);
    }
    __syncwarp();
    // (with the test hook set, a barrier that nothing completes instead: the wait runs out)
    if (!(p.stall_tries ? mbar_wait_n(stall_bar, 0, tries) : mbar_wait(full_bar(s), (i / kVStages) & 1))) {
      atomicOr(p.status, kDevTimeout);
      ok = false;
      break;
    }
    // token tw + 2 j + half of the tile for this half-warp (records past n hold stale codes, weight 0)
    const uint32_t *rs = reinterpret_cast<const uint32_t *>(stages + (size_t)s * T::kStageBytes) + (size_t)(tw + half) * RW;
    const int np = (min(32, n - tw) + 1) >> 1;   // token pairs of this warp (warp-uniform, may be <= 0)
    const uint32_t lane8 = 8u * sub;   // this lane's copy of the pair table
    // token pair j of this warp: two tokens, one per half-warp
    auto pair_step = [&](int j) {
      const uint32_t *rec = rs + 2 * j * RW;
      const uint32_t lo = rec[wd];
      const uint32_t hi = two ? rec[wd + 1] : 0u;
      const uint32_t bits = __funnelshift_r(lo, hi, sh);
      const uint64_t *wt = wscr + (tw + 2 * j + half) * kVMaxQ;
      uint64_t w2[QMAX];
#pragma unroll
      for (int qq = 0; qq < QMAX; ++qq) w2[qq] = wt[qq];
      if constexpr (!MIXED) {
#pragma unroll
        for (int pp = 0; pp < CPL / 2; ++pp) {
          // byte offset of the pair (codes 2 pp, 2 pp + 1) in the table: key * 128 (+ the lane copy)
          constexpr uint32_t kMask = 128u * (L * L - 1);
          const int shr = 2 * BITS * pp - 7;
          const uint32_t off = ((shr >= 0 ? bits >> (shr & 31) : bits << ((-shr) & 31)) & kMask) | lane8;
          const uint64_t cv = *reinterpret_cast<const uint64_t *>(reinterpret_cast<const unsigned char *>(ptab) + off);
#pragma unroll
          for (int qq = 0; qq < QMAX; ++qq) acc2[pp][qq] = f2_fma(w2[qq], cv, acc2[pp][qq]);
        }
      } else {
        // bits << 7 as a 64-bit pair, so that a pair key of a runtime width is one funnel shift
        const uint32_t lo7 = bits << 7, hi7 = bits >> 25;
#pragma unroll
        for (int pp = 0; pp < CPL / 2; ++pp) {
          const uint32_t off = (__funnelshift_r(lo7, hi7, 2 * lb * pp) & kmask_l) | tbase_l;
          const uint64_t cv = *reinterpret_cast<const uint64_t *>(reinterpret_cast<const unsigned char *>(ptab) + off);
#pragma unroll
          for (int qq = 0; qq < QMAX; ++qq) acc2[pp][qq] = f2_fma(w2[qq], cv, acc2[pp][qq]);
        }
      }
    };
    if (QMAX == 1 && np == 16) {
      // a whole warp's 32 tokens (every tile but a chunk's ragged last one), one query head: fully unrolled,
      // so the record and weight addresses are immediates and no loop counter is kept (8-18% faster; with
      // four heads the unrolled loop measured 8% slower)
#pragma unroll
      for (int j = 0; j < 16; ++j) pair_step(j);
    } else {
#pragma unroll 2
      for (int j = 0; j < np; ++j) pair_step(j);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));   // this warp is done with the stage and its weights
  }
  // the two half-warps accumulated different tokens of the same coordinates
  float acc[CPL][QMAX];
#pragma unroll
  for (int pp = 0; pp < CPL / 2; ++pp)
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) f2_unpack(acc2[pp][qq], acc[2 * pp][qq], acc[2 * pp + 1][qq]);
#pragma unroll
  for (int a = 0; a < CPL; ++a)
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) acc[a][qq] += __shfl_xor_sync(0xffffffffu, acc[a][qq], 16);

  // Only now may the merge grid become resident (it stages its matrix while the last CTAs finish):
  // its CTAs wait for this whole grid, and resident earlier they would hold registers and shared
  // memory on SMs that this grid's later waves need.
  pdl_launch_dependents();
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

template <int BITS, int QMAX, bool MIXED>
cudaError_t launch_vf(const VFastParams &fp, int units, cudaStream_t st) {
  auto kern = attend_fast_kernel<BITS, QMAX, MIXED>;
  const size_t smem = VTile<BITS, MIXED>::kBytes;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)fp.p.n_chunks, (unsigned)units), kVThreads, smem, st>>>(fp);
  return cudaGetLastError();
}

template <int BITS, bool MIXED = false>
cudaError_t launch_vf_q(const VFastParams &fp, int units, cudaStream_t st) {
  switch (fp.p.q_per_cta) {
    case 1: return launch_vf<BITS, 1, MIXED>(fp, units, st);
    case 2: return launch_vf<BITS, 2, MIXED>(fp, units, st);
    case 3: return launch_vf<BITS, 3, MIXED>(fp, units, st);
    default: return launch_vf<BITS, 4, MIXED>(fp, units, st);
  }
}

}  // namespace

bool attend_fast_supported(int d, int bits, int q_per_cta, const void *records, int n_hi, int64_t capacity) {
  if (d != kVD || q_per_cta < 1 || q_per_cta > kVMaxQ || (reinterpret_cast<uintptr_t>(records) & 15) != 0)
    return false;
  if (n_hi == 0) return bits >= 1 && bits <= 4;
  // mixed rate with the first 64 coordinates wider; the rows of every (sequence, head) must start on
  // 16 bytes (a record is 40 or 56 bytes: an even capacity)
  return n_hi == 64 && bits >= 1 && bits <= 3 && capacity % 2 == 0;
}

// Tokens per chunk (a multiple of the 512-token tile): the split of every
// unit's tiles into equal chunks that minimises the busiest SM's time, counted
// as whole waves of one CTA per SM times (tiles per chunk + a CTA's fixed cost:
// set-up, the first copies' latency and the end-of-chunk merge, about two
// tiles' time). Without the fixed cost, many units would be split into
// one-tile chunks (16 384 CTAs on the 8 x 8 x 131072 cache), slower per token
// and with 256 partials per query head to merge.
int64_t attend_fast_chunk(int64_t n_tokens, int units) {
  constexpr int64_t kCtaCost = 2;
  const int64_t tpu = (n_tokens + kVTile - 1) / kVTile;
  const int64_t slots = device_sm_count();
  int64_t best_tpc = tpu, best_cost = INT64_MAX;
  const int64_t max_nc = tpu < 8 * slots ? tpu : 8 * slots;
  for (int64_t nc = 1; nc <= max_nc; ++nc) {
    const int64_t tpc = (tpu + nc - 1) / nc;
    const int64_t ctas = (int64_t)units * ((tpu + tpc - 1) / tpc);
    const int64_t cost = ((ctas + slots - 1) / slots) * (tpc + kCtaCost);
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
  if (p.n_hi == 64) {
    switch (bits) {
      case 1: return launch_vf_q<1, true>(fp, units, st);
      case 2: return launch_vf_q<2, true>(fp, units, st);
      default: return launch_vf_q<3, true>(fp, units, st);
    }
  }
  switch (bits) {
    case 1: return launch_vf_q<1>(fp, units, st);
    case 2: return launch_vf_q<2>(fp, units, st);
    case 3: return launch_vf_q<3>(fp, units, st);
    default: return launch_vf_q<4>(fp, units, st);
  }
}

}  // namespace tq
