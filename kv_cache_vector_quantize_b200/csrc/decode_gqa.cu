// One decode step for grouped queries in one pass over the tokens: the logits of
// several query heads on their shared packed keys, the running softmax and the
// packed values, without writing the logits to memory.
//
// Estimator (usedby.ai, "TurboQuant: Compresion de KV Cache a 3 bits y
// aceleracion de inferencia en H100", "El Pitch": attention computed on the
// compressed cache; zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache
// to 3.5 bits per channel", paragraph 1: the cache holds keys and values):
//   l_t = n_t ( <Pi q, c[code_t]> + rho_t sqrt(pi/2)/d <S q, 2 sign_t - 1> ),
//   out = Pi^T sum_t softmax_t(scale l_t) vnorm_t cV[vcode_t].
//
// It computes exactly what the grouped-query logit scan (logits_gqa.cu)
// followed by the softmax.V chunk kernel (attend_fast.cu) compute, bit for bit:
//   - the logits come from the same float16 four-head tables (gqa_tables_kernel,
//     built once per call), and key t of a 512-token tile is computed by lane
//     t mod 32, so its table reads are summed in the same order;
//   - the softmax.V kernel splits a 512-token tile over 16 warps of 32 tokens.
//     Here a tile arrives as two 256-token stages and each of the 8 consumer
//     warps plays two of those 16 warps (w on the first stage, w + 8 on the
//     second), with a separate running state (max, sum, accumulators) for each,
//     so every float operation happens on the same operands in the same order;
//   - chunks and the final merge of the 16 states are those of the softmax.V
//     kernel, and the same merge kernel (attend.cu) reduces the chunk partials.
//
// Shared memory (dynamic): barriers and merge statistics; stage slots of 256
// keys (records, norms, residual norms) and of 256 values (records, norms)
// below and above the 128 KB table block, which sits at a 64 KB-aligned base
// (the table addressing of the grouped-query scan); above it the table of
// value-centroid pairs (one copy per lane of a 16-lane phase) and the token
// weights. One producer thread streams the key and value stages by bulk
// copies; every wait is bounded.
#include "common.cuh"
#include "gqa_core.cuh"

namespace tq {

namespace {

using namespace gqa;

constexpr int kQWarps = 8;                     // consumer warps
constexpr int kQThreads = 32 * (kQWarps + 1);  // + one producer warp
constexpr int kQHalf = 256;                    // tokens per stage
constexpr int kQVW = 16;                       // the softmax.V kernel's warps per 512-token tile
constexpr int kQMaxK = 4, kQMaxV = 4;          // stage slots
constexpr uint32_t kQHdr = 1024;               // barriers, merge statistics, value codebook

template <int BETA, int VBITS, int QH>
struct QLay {
  static constexpr int RWK = GKeys<BETA>::RW;
  static constexpr int RWV = VBITS * kGD / 32;
  static constexpr uint32_t kKStage = kQHalf * (RWK + 2) * 4;   // records, norms, residual norms
  static constexpr uint32_t kVStage = kQHalf * (RWV + 1) * 4;   // records, norms
  static constexpr uint32_t kPairs = (1u << (2 * VBITS)) * 16 * 8;
  static constexpr uint32_t kScratch = kQWarps * 32 * QH * 8;
  static constexpr uint32_t kMerge = kQVW * QH * kGD * 4;
  static_assert((kQHalf * RWK * 4) % 16 == 0 && (kQHalf * RWV * 4) % 16 == 0, "bulk copy offsets");
};

// Placement of the stage slots: regions [a0, T0) and [b0, end), filled K, V, K, V, ...
// (first fit), at most kQMaxK and kQMaxV of each. The same on host and device.
template <int BETA, int VBITS, int QH>
struct QPlan {
  uint32_t T0, P0, W0, end;
  uint32_t kslot[kQMaxK], vslot[kQMaxV];
  int nk, nv;
  __host__ __device__ QPlan(uint32_t dyn0, uint32_t dyn_bytes) {
    using Q = QLay<BETA, VBITS, QH>;
    const uint32_t a0 = dyn0 + kQHdr;
    T0 = (a0 + kGHalf - 1) & ~(kGHalf - 1);
    P0 = T0 + 2 * kGHalf;
    W0 = P0 + Q::kPairs;
    end = dyn0 + dyn_bytes;
    uint32_t lo = a0, hi = W0 + Q::kScratch;
    nk = nv = 0;
    for (int r = 0; r < kQMaxK + kQMaxV; ++r) {
      const bool want_k = (r % 2 == 0) ? nk < kQMaxK : false;
      const bool want_v = (r % 2 == 1) ? nv < kQMaxV : false;
      const uint32_t sz = want_k ? Q::kKStage : Q::kVStage;
      if (!want_k && !want_v) continue;
      uint32_t at = 0;
      if (lo + sz <= T0) {
        at = lo;
        lo += sz;
      } else if (hi + sz <= end) {
        at = hi;
        hi += sz;
      } else {
        continue;
      }
      if (want_k) kslot[nk++] = at;
      else vslot[nv++] = at;
    }
  }
  __host__ __device__ bool ok(uint32_t dyn0) const {
    return nk >= 2 && nv >= 2 && W0 + QLay<BETA, VBITS, QH>::kScratch <= end &&
           dyn0 + kQHdr + QLay<BETA, VBITS, QH>::kMerge <= T0;
  }
};

struct DGParams {
  const uint32_t *krec;
  const float *knorm, *krnorm;
  const uint32_t *vrec;
  const float *vnorm;
  const unsigned char *tables;   // units x 128 KB
  const float *sigma;            // [n_seq][n_q_heads]
  const float *cbv;
  float *partial;                // [n_seq][n_q_heads][n_chunks][130]
  uint32_t *status;
  int64_t n_tokens, cap_k, cap_v;
  int n_kv_heads, n_q_heads, group, qblocks, tiles_per_chunk, n_chunks;
  float scale;
  uint32_t dyn_bytes;
};

template <int BETA, int VBITS, int QH>
__global__ void __launch_bounds__(kQThreads, 1) decode_gqa_kernel(const DGParams p) {
  using K = GKeys<BETA>;
  using Q = QLay<BETA, VBITS, QH>;
  constexpr int RWK = Q::RWK, RWV = Q::RWV, IW = K::IW;
  constexpr int LV = 1 << VBITS;
  constexpr int CPL = 8;              // value coordinates per lane (16 lanes per token)
  constexpr int FB = CPL * VBITS;     // value code bits of a lane's coordinates
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t dyn0 = smem_u32(smem);
  const QPlan<BETA, VBITS, QH> pl(dyn0, p.dyn_bytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto kfull = [&](int s) { return dyn0 + 8u * s; };
  auto kempty = [&](int s) { return dyn0 + 8u * (kQMaxK + s); };
  auto vfull = [&](int s) { return dyn0 + 8u * (2 * kQMaxK + s); };
  auto vempty = [&](int s) { return dyn0 + 8u * (2 * kQMaxK + kQMaxV + s); };
  const uint32_t tab_bar = dyn0 + 8u * (2 * kQMaxK + 2 * kQMaxV);
  float *mst = reinterpret_cast<float *>(smem + 256);          // [16][QH]
  float *lst = mst + kQVW * QH;                                // [16][QH]
  float *sig_s = lst + kQVW * QH;                              // [QH]
  float *cbs = sig_s + 4;                                      // [16]
  if (!pl.ok(dyn0)) {
    if (tid == 0) {
      pdl_wait();   // a clean status word comes from the table kernel
      atomicOr(p.status, kDevBadShape);
    }
    return;
  }
  const int chunk = blockIdx.x, unit = blockIdx.y;
  const int qb = unit % p.qblocks, sk = unit / p.qblocks;
  const int64_t t_begin = (int64_t)chunk * p.tiles_per_chunk * 512;
  const int64_t t_end = min(p.n_tokens, t_begin + (int64_t)p.tiles_per_chunk * 512);
  const int n_half = t_begin < t_end ? (int)((t_end - t_begin + kQHalf - 1) / kQHalf) : 0;
  const size_t kslot0 = (size_t)sk * p.cap_k, vslot0 = (size_t)sk * p.cap_v;
  const bool knc = (reinterpret_cast<uintptr_t>(p.knorm + kslot0) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(p.krnorm + kslot0) % 16 == 0);
  const bool vnc = reinterpret_cast<uintptr_t>(p.vnorm + vslot0) % 16 == 0;

  if (tid == 0) {
    for (int s = 0; s < kQMaxK; ++s) {
      mbar_init(kfull(s), 1);
      mbar_init(kempty(s), kQWarps);
    }
    for (int s = 0; s < kQMaxV; ++s) {
      mbar_init(vfull(s), 1);
      mbar_init(vempty(s), kQWarps);
    }
    mbar_init(tab_bar, 1);
    mbar_fence_init();
  }
  if (tid < LV) cbs[tid] = p.cbv[tid];
  __syncthreads();
  // value-centroid pairs (c[k & (LV-1)], c[k >> VBITS]) at entry 16 k + lane copy
  uint64_t *ptab = reinterpret_cast<uint64_t *>(smem + (pl.P0 - dyn0));
  for (int e = tid; e < (int)(Q::kPairs / 8); e += kQThreads) {
    const int key = e >> 4;
    ptab[e] = f2_pack(cbs[key & (LV - 1)], cbs[key >> VBITS]);
  }
  __syncthreads();

  if (warp == kQWarps) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      int kis = 0, vis = 0;
      bool good = true;
      for (int h = 0; h < n_half && good; ++h) {
        const int64_t t0 = t_begin + (int64_t)h * kQHalf;
        const int n = (int)min((int64_t)kQHalf, t_end - t0);
        {
          const int s = h % pl.nk;
          if (h >= pl.nk && !mbar_wait(kempty(s), ((h / pl.nk) - 1) & 1)) {
            good = false;
            break;
          }
          const bool nc = knc && (n % 4) == 0;
          const uint32_t rb = (uint32_t)n * RWK * 4;
          mbar_arrive_expect_tx(kfull(s), rb + (nc ? 8u * n : 0u));
          bulk_g2s(pl.kslot[s], p.krec + (kslot0 + t0) * RWK, rb, kfull(s));
          if (nc) {
            bulk_g2s(pl.kslot[s] + kQHalf * RWK * 4, p.knorm + kslot0 + t0, 4u * n, kfull(s));
            bulk_g2s(pl.kslot[s] + kQHalf * RWK * 4 + kQHalf * 4, p.krnorm + kslot0 + t0, 4u * n, kfull(s));
          }
          ++kis;
        }
        {
          const int s = h % pl.nv;
          if (h >= pl.nv && !mbar_wait(vempty(s), ((h / pl.nv) - 1) & 1)) {
            good = false;
            break;
          }
          const bool nc = vnc && (n % 4) == 0;
          const uint32_t rb = (uint32_t)n * RWV * 4;
          mbar_arrive_expect_tx(vfull(s), rb + (nc ? 4u * n : 0u));
          bulk_g2s(pl.vslot[s], p.vrec + (vslot0 + t0) * RWV, rb, vfull(s));
          if (nc) bulk_g2s(pl.vslot[s] + kQHalf * RWV * 4, p.vnorm + vslot0 + t0, 4u * n, vfull(s));
          ++vis;
        }
      }
      if (!good) {
        pdl_wait();
        atomicOr(p.status, kDevTimeout);
      }
      // every issued copy must land before the CTA exits
      for (int h = max(0, kis - pl.nk); h < kis; ++h)
        if (!mbar_wait(kfull(h % pl.nk), (h / pl.nk) & 1)) {
          pdl_wait();
          atomicOr(p.status, kDevTimeout);
          break;
        }
      for (int h = max(0, vis - pl.nv); h < vis; ++h)
        if (!mbar_wait(vfull(h % pl.nv), (h / pl.nv) & 1)) {
          pdl_wait();
          atomicOr(p.status, kDevTimeout);
          break;
        }
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  pdl_wait();   // the tables and scales (and a clean status word) come from the table kernel
  const int seq = sk / p.n_kv_heads, kvh = sk - seq * p.n_kv_heads;
  const int h0 = kvh * p.group + qb * QH;
  if (tid == 0) {
    constexpr uint32_t kChunk = 16384;
    mbar_arrive_expect_tx(tab_bar, 2 * kGHalf);
    const unsigned char *src = p.tables + (size_t)unit * (2 * kGHalf);
    for (uint32_t o = 0; o < 2 * kGHalf; o += kChunk) bulk_g2s(pl.T0 + o, src + o, kChunk, tab_bar);
  }
  if (tid < QH) sig_s[tid] = p.sigma[(size_t)seq * p.n_q_heads + h0 + tid];
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kQWarps) : "memory");
  float sg[QH];
#pragma unroll
  for (int h = 0; h < QH; ++h) sg[h] = sig_s[h];
  bool ok = mbar_wait(tab_bar, 0);
  if (!ok) atomicOr(p.status, kDevTimeout);

  // key-table address constants of this lane (as in the grouped-query scan)
  uint32_t sel[4];
  const uint32_t sel0 = 0x7604u | ((uint32_t)(lane & 3) << 4);
#pragma unroll
  for (int j = 0; j < 4; ++j) sel[j] = sel0 ^ ((uint32_t)(j & 1) | ((uint32_t)j << 4));
  constexpr int PSH = QH == 4 ? 3 : 2;
  const uint32_t x0 = (pl.T0 & 0xFFFF0000u) | ((uint32_t)lane << PSH) | ((uint32_t)(lane ^ 1) << (8 + PSH));
  uint32_t xv[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) xv[m] = x0 ^ ((uint32_t)m * (0x202u << PSH));
  // value-code field of this lane (8 coordinates, 16 lanes per token) and its pair-table copy
  const int half = lane >> 4, sub = lane & 15;
  const int bit0 = FB * sub, wd = bit0 >> 5, sh = bit0 & 31;
  const bool two = sh + FB > 32;
  const unsigned char *ptl = smem + (pl.P0 - dyn0) + 8 * sub;
  uint64_t *wscr = reinterpret_cast<uint64_t *>(smem + (pl.W0 - dyn0)) + (size_t)warp * 32 * QH;   // [32][QH]

  // running states of the two softmax.V warps this warp plays (w and w + 8)
  float m[2][QH], l[2][QH];
  uint64_t acc2[2][CPL / 2][QH];
#pragma unroll
  for (int v = 0; v < 2; ++v)
#pragma unroll
    for (int qq = 0; qq < QH; ++qq) {
      m[v][qq] = -INFINITY;
      l[v][qq] = 0.f;
#pragma unroll
      for (int pp = 0; pp < CPL / 2; ++pp) acc2[v][pp][qq] = 0ull;
    }
  const int k = warp * 32 + lane;   // this lane's key / token within a stage

  for (int h = 0; h < n_half && ok; ++h) {
    const int vwo = h & 1;   // 0: this stage holds tokens [0, 256) of its tile (softmax.V warp w), 1: w + 8
    const int64_t t0 = t_begin + (int64_t)h * kQHalf;
    const int n = (int)min((int64_t)kQHalf, t_end - t0);
    const bool valid = k < n;
    // ---- logits of this lane's key for the QH heads ----
    const int ks = h % pl.nk;
    if (!mbar_wait(kfull(ks), (h / pl.nk) & 1)) {
      atomicOr(p.status, kDevTimeout);
      ok = false;
      break;
    }
    const unsigned char *kst = smem + (pl.kslot[ks] - dyn0);
    uint32_t w[RWK];
    if (valid) {
      const uint4 *src = reinterpret_cast<const uint4 *>(kst + (size_t)k * RWK * 4);
#pragma unroll
      for (int j = 0; j < RWK / 4; ++j) {
        const uint4 v = src[j];
        w[4 * j] = v.x;
        w[4 * j + 1] = v.y;
        w[4 * j + 2] = v.z;
        w[4 * j + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < RWK; ++j) w[j] = 0u;
    }
    float nrm = 0.f, rho = 0.f;
    if (valid) {
      if (knc && (n & 3) == 0) {   // the producer's condition for this stage
        nrm = reinterpret_cast<const float *>(kst + kQHalf * RWK * 4)[k];
        rho = reinterpret_cast<const float *>(kst + kQHalf * RWK * 4 + kQHalf * 4)[k];
      } else {
        nrm = __ldg(p.knorm + kslot0 + t0 + k);
        rho = __ldg(p.krnorm + kslot0 + t0 + k);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(kempty(ks));
    uint32_t wi[IW], wsg[4];
#pragma unroll
    for (int j = 0; j < IW; ++j) wi[j] = w[j];
#pragma unroll
    for (int j = 0; j < 4; ++j) wsg[j] = w[IW + j];
    xor_perm<IW>(wi, (lane >> 2) & (IW - 1));
    xor_perm<4>(wsg, (lane >> 2) & 3);
    float fi[QH], fs[QH];
#pragma unroll
    for (int qq = 0; qq < QH; ++qq) fi[qq] = fs[qq] = 0.f;
    gqa_sum<QH, K::NI, 0u>(wi, sel, xv, fi);
    gqa_sum<QH, 16, kGHalf>(wsg, sel, xv, fs);
    float z[QH];
#pragma unroll
    for (int qq = 0; qq < QH; ++qq) {
      const float lg = nrm * sg[qq] * fmaf(rho, fs[qq], fi[qq]);   // the scan's stored logit
      z[qq] = valid ? p.scale * lg : -INFINITY;
    }
    // ---- values: wait for the stage, weights, accumulation (the softmax.V kernel's steps) ----
    const int vs = h % pl.nv;
    if (!mbar_wait(vfull(vs), (h / pl.nv) & 1)) {
      atomicOr(p.status, kDevTimeout);
      ok = false;
      break;
    }
    const unsigned char *vst = smem + (pl.vslot[vs] - dyn0);
    float vn = 0.f;
    if (valid) vn = (vnc && (n & 3) == 0) ? reinterpret_cast<const float *>(vst + kQHalf * RWV * 4)[k]
                                          : __ldg(p.vnorm + vslot0 + t0 + k);
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      if (v != vwo) continue;   // warp-uniform
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) {
        const float mx = fmaxf(m[v][qq], warp_max(z[qq]));
        const float f = mx == -INFINITY ? 0.f : expf(m[v][qq] - mx);
        const float e = mx == -INFINITY ? 0.f : expf(z[qq] - mx);
        m[v][qq] = mx;
        l[v][qq] = fmaf(l[v][qq], f, e);
        const uint64_t f2 = f2_pack(f, f);
#pragma unroll
        for (int pp = 0; pp < CPL / 2; ++pp) acc2[v][pp][qq] = f2_mul(acc2[v][pp][qq], f2);
        const float wt = e * vn;   // 0 for a token past the end
        wscr[lane * QH + qq] = f2_pack(wt, wt);
      }
      __syncwarp();
      const uint32_t *rs = reinterpret_cast<const uint32_t *>(vst) + (size_t)(32 * warp + half) * RWV;
      const int np = (min(32, n - 32 * warp) + 1) >> 1;   // token pairs of this warp (may be <= 0)
#pragma unroll 2
      for (int j = 0; j < np; ++j) {
        const uint32_t *rec = rs + 2 * j * RWV;
        const uint32_t lo = rec[wd];
        const uint32_t hi = two ? rec[wd + 1] : 0u;
        const uint32_t bits = __funnelshift_r(lo, hi, sh);
        const uint64_t *wt = wscr + (2 * j + half) * QH;
        uint64_t w2[QH];
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) w2[qq] = wt[qq];
#pragma unroll
        for (int pp = 0; pp < CPL / 2; ++pp) {
          constexpr uint32_t kMask = 128u * (LV * LV - 1);
          const int shr = 2 * VBITS * pp - 7;
          const uint32_t off = (shr >= 0 ? bits >> (shr & 31) : bits << ((-shr) & 31)) & kMask;
          const uint64_t cv = *reinterpret_cast<const uint64_t *>(ptl + off);
#pragma unroll
          for (int qq = 0; qq < QH; ++qq) acc2[v][pp][qq] = f2_fma(w2[qq], cv, acc2[v][pp][qq]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(vempty(vs));
  }
  pdl_launch_dependents();   // the merge grid may become resident now (see attend_fast.cu)

  // ---- merge the 16 states: M = max_w m_w, each scaled by e^{m_w - M}, summed in warp order ----
  float acc[2][CPL][QH];
#pragma unroll
  for (int v = 0; v < 2; ++v) {
#pragma unroll
    for (int pp = 0; pp < CPL / 2; ++pp)
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) f2_unpack(acc2[v][pp][qq], acc[v][2 * pp][qq], acc[v][2 * pp + 1][qq]);
#pragma unroll
    for (int a = 0; a < CPL; ++a)
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) acc[v][a][qq] += __shfl_xor_sync(0xffffffffu, acc[v][a][qq], 16);
#pragma unroll
    for (int qq = 0; qq < QH; ++qq) l[v][qq] = warp_sum(l[v][qq]);
    if (lane == 0) {
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) {
        mst[(warp + 8 * v) * QH + qq] = m[v][qq];
        lst[(warp + 8 * v) * QH + qq] = l[v][qq];
      }
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kQWarps) : "memory");   // also: every stage has been consumed
  float *mg = reinterpret_cast<float *>(smem + kQHdr);   // [16][QH][128], over the lower stages
#pragma unroll
  for (int qq = 0; qq < QH; ++qq) {
    float mc = -INFINITY;
    for (int w2 = 0; w2 < kQVW; ++w2) mc = fmaxf(mc, mst[w2 * QH + qq]);
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const float sc = mc == -INFINITY ? 0.f : expf(m[v][qq] - mc);
      if (half == 0) {
        float4 *dst = reinterpret_cast<float4 *>(mg + ((warp + 8 * v) * QH + qq) * kGD + CPL * sub);
        dst[0] = make_float4(acc[v][0][qq] * sc, acc[v][1][qq] * sc, acc[v][2][qq] * sc, acc[v][3][qq] * sc);
        dst[1] = make_float4(acc[v][4][qq] * sc, acc[v][5][qq] * sc, acc[v][6][qq] * sc, acc[v][7][qq] * sc);
      }
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kQWarps) : "memory");
  if (!ok) return;
  for (int e = tid; e < QH * kGD; e += 32 * kQWarps) {
    const int qq = e / kGD, ii = e - qq * kGD;
    float v = 0.f;
    for (int w2 = 0; w2 < kQVW; ++w2) v += mg[(w2 * QH + qq) * kGD + ii];
    const size_t hrow = (size_t)seq * p.n_q_heads + h0 + qq;
    p.partial[(hrow * p.n_chunks + chunk) * (size_t)(kGD + 2) + 2 + ii] = v;
  }
  if (tid < QH) {
    float mc = -INFINITY;
    for (int w2 = 0; w2 < kQVW; ++w2) mc = fmaxf(mc, mst[w2 * QH + tid]);
    float lc = 0.f;
    for (int w2 = 0; w2 < kQVW; ++w2) lc += mc == -INFINITY ? 0.f : lst[w2 * QH + tid] * expf(mst[w2 * QH + tid] - mc);
    const size_t hrow = (size_t)seq * p.n_q_heads + h0 + tid;
    float *part = p.partial + (hrow * p.n_chunks + chunk) * (size_t)(kGD + 2);
    part[0] = mc;
    part[1] = lc;
  }
}

constexpr uint32_t kQDyn0 = 1024;   // reserved shared memory below the dynamic window on sm_100

template <int BETA, int VBITS, int QH>
bool q_fits(uint32_t limit) {
  return QPlan<BETA, VBITS, QH>(kQDyn0, limit).ok(kQDyn0);
}

template <int BETA, int VBITS, int QH>
cudaError_t q_launch(DGParams p, int n_seq, uint32_t limit, cudaStream_t st) {
  const QPlan<BETA, VBITS, QH> pl(kQDyn0, limit);
  p.dyn_bytes = limit;
  auto kern = decode_gqa_kernel<BETA, VBITS, QH>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), limit);
  if (e != cudaSuccess) return e;
  const int units = n_seq * p.n_kv_heads * p.qblocks;
  return launch_after(kern, dim3((unsigned)p.n_chunks, (unsigned)units), dim3(kQThreads), (size_t)limit, st, p);
}

template <int BETA, int QH>
bool q_fits_v(int vbits, uint32_t limit) {
  switch (vbits) {
    case 1: return q_fits<BETA, 1, QH>(limit);
    case 2: return q_fits<BETA, 2, QH>(limit);
    case 3: return q_fits<BETA, 3, QH>(limit);
    default: return false;   // 4-bit value codes: the pair table (32 KB) leaves too little room
  }
}

template <int BETA, int QH>
cudaError_t q_launch_v(const DGParams &p, int vbits, int n_seq, uint32_t limit, cudaStream_t st) {
  switch (vbits) {
    case 1: return q_launch<BETA, 1, QH>(p, n_seq, limit, st);
    case 2: return q_launch<BETA, 2, QH>(p, n_seq, limit, st);
    default: return q_launch<BETA, 3, QH>(p, n_seq, limit, st);
  }
}

}  // namespace

bool decode_gqa_supported(int d, int kbits, int vbits, int group, size_t limit) {
  if (d != kGD || !gqa_supported(d, kbits, group)) return false;
  const int qh = group >= 4 ? 4 : 2;
  const uint32_t lim = (uint32_t)limit;
  if (kbits == 1) return qh == 4 ? q_fits_v<1, 4>(vbits, lim) : q_fits_v<1, 2>(vbits, lim);
  return qh == 4 ? q_fits_v<2, 4>(vbits, lim) : q_fits_v<2, 2>(vbits, lim);
}

cudaError_t launch_decode_gqa(const DecodeGqaArgs &a, cudaStream_t st) {
  DGParams p{};
  p.krec = a.krec;
  p.knorm = a.knorm;
  p.krnorm = a.krnorm;
  p.vrec = a.vrec;
  p.vnorm = a.vnorm;
  p.tables = a.tables;
  p.sigma = a.sigma;
  p.cbv = a.cbv;
  p.partial = a.partial;
  p.status = a.status;
  p.n_tokens = a.n_tokens;
  p.cap_k = a.cap_k;
  p.cap_v = a.cap_v;
  p.n_kv_heads = a.n_kv_heads;
  p.n_q_heads = a.n_q_heads;
  p.group = a.n_q_heads / a.n_kv_heads;
  p.qblocks = a.qblocks;
  p.tiles_per_chunk = (int)(a.chunk / 512);
  p.n_chunks = a.n_chunks;
  p.scale = a.scale;
  const uint32_t lim = (uint32_t)a.smem_limit;
  const int qh = p.group >= 4 ? 4 : 2;
  if (a.kbits == 1) return qh == 4 ? q_launch_v<1, 4>(p, a.vbits, a.n_seq, lim, st) : q_launch_v<1, 2>(p, a.vbits, a.n_seq, lim, st);
  return qh == 4 ? q_launch_v<2, 4>(p, a.vbits, a.n_seq, lim, st) : q_launch_v<2, 2>(p, a.vbits, a.n_seq, lim, st);
}

}  // namespace tq
