// Quantize-append on the tcgen05 tensor cores, for bf16 inputs with d = 128.
//
// The method is the encoder of zubnet.ai news, "Google's TurboQuant quantizes
// LLM KV cache to 3.5 bits per channel", paragraph 2, and winningdata.io,
// "TurboQuant: Google comprime KV cache para 3 bits sem perder acuracia",
// "Como o TurboQuant funciona": n = ||x||, y = Pi x / n, code_i = #{j : y_i > t_j},
// and for keys e = y - c[code], rho = ||e||, sign bits of (S Pi^T) e.
//
// Precision. The codes must agree with a float64 encoder except within 1e-5
// of a threshold, so the projections need about 1e-6 of the vectors' scale:
// more than one bf16 product gives. A bf16 input x is exact in bf16; each
// float32 matrix is split into two bf16 parts, P = P_hi + P_lo with
// |P - P_hi - P_lo| <= 2^-18 |P|, and Pi x = x P_hi^T + x P_lo^T accumulates in
// float32 in tensor memory: worst-case error 2^-18 ||Pi_i|| ||x||, below the
// 1e-5 band. The residual e (float32) is split the same way, and
// (S Pi^T) e = E_hi M_hi^T + E_hi M_lo^T + E_lo M_hi^T + E_lo M_lo^T (four
// products) keeps the sign decisions within the band as well.
//
// Tile flow (one CTA of 8 warps per SM, persistent over 128-token tiles):
//   load x rows into the A tile (and ||x|| in double) -> 16 MMAs (Pi parts)
//   -> epilogue: one token per tensor-memory lane, a warp pair splitting the
//      128 columns: codes, code-stream words, residual parts into the E tiles
//   -> 32 MMAs (S Pi^T parts) -> epilogue: sign words -> records and norms.
// Operand tiles use the no-swizzle K-major core-matrix layout of tc.cuh.
#include "common.cuh"
#include "tc.cuh"

namespace tq {

namespace {

constexpr int kTD = 128;                   // head dimension
constexpr int kTT = 128;                   // tokens per tile (MMA M)
// keys: 16 warps (4 threads per token, 32 columns each); values: 8 warps, two CTAs per SM
template <bool QJL>
__host__ __device__ constexpr int tc_threads() { return QJL ? 512 : 256; }
constexpr uint32_t kTile = kTT * kTD * 2;  // bytes of one bf16 operand tile (32 KB)
constexpr uint32_t kLBO = kTT * 16;        // K-direction core-matrix stride (2048 B)
constexpr uint32_t kSBO = 128;             // row-direction core-matrix stride

template <bool QJL>
struct TcLayout {
  // dynamic shared memory, byte offsets
  static constexpr uint32_t kPhi = 0, kPlo = kTile;
  static constexpr uint32_t kMhi = 2 * kTile, kMlo = 3 * kTile;              // keys only
  static constexpr uint32_t kX = QJL ? 4 * kTile : 2 * kTile;
  static constexpr uint32_t kEhi = kX + kTile, kElo = kX + 2 * kTile;        // keys only
  // record staging: inside the E tiles for keys (free once the sketch product is done),
  // a buffer of its own for values
  static constexpr uint32_t kRec = QJL ? kEhi : kX + kTile;                  // uint32[128][<= 21] records
  static constexpr uint32_t kRho = kRec + 11264;                             // float[4][128] residual partials
  static constexpr uint32_t kSlot = kRec + 13312;                            // int64[128] cache slots
  static constexpr uint32_t kSmall = QJL ? kX + 3 * kTile : kRec + 14336;
  static constexpr uint32_t kNrm = kSmall;                                   // float[2][128] (two tiles in flight)
  static constexpr uint32_t kCb = kNrm + 1024;                               // float[16] centroids, [16] thresholds
  static constexpr uint32_t kBar = kCb + 128;                                // 2 mbarriers
  static constexpr uint32_t kTslot = kBar + 16;                              // tensor-memory base address
  static constexpr uint32_t kBytes = kTslot + 16;
  static constexpr uint32_t kTmemCols = QJL ? 256 : 128;
};

// The x rows of one tile as this thread loads them: with NW warps, warp w owns
// rows [w R, w R + R) (R = 128 / NW, a multiple of 8), lane l row 8 g + (l & 7)
// and 16-byte chunks 4 i + (l >> 3), for g < R / 8, i < 4.
template <int NW>
struct XRegs {
  uint4 v[128 / NW / 8][4];
};

template <int NW>
__device__ __forceinline__ void load_x(XRegs<NW> &xr, const __nv_bfloat16 *__restrict__ x, int64_t row0,
                                       int64_t rows, int warp, int lane) {
  constexpr int R = 128 / NW;
#pragma unroll
  for (int g = 0; g < R / 8; ++g) {
    const int64_t row = row0 + R * warp + 8 * g + (lane & 7);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int kc = 4 * i + (lane >> 3);
      xr.v[g][i] = row < rows ? __ldg(reinterpret_cast<const uint4 *>(x + row * kTD + 8 * kc)) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// Registers -> A tile, and ||x|| (double accumulation) -> nrm[row].
template <int NW>
__device__ __forceinline__ void store_x(const XRegs<NW> &xr, unsigned char *xtile, float *nrm, int warp, int lane) {
  constexpr int R = 128 / NW;
#pragma unroll
  for (int g = 0; g < R / 8; ++g) {
    const int t = R * warp + 8 * g + (lane & 7);
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int kc = 4 * i + (lane >> 3);
      const uint4 v = xr.v[g][i];
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const double a = (double)__uint_as_float(wv[q] << 16), b = (double)__uint_as_float(wv[q] & 0xFFFF0000u);
        ss = fma(a, a, fma(b, b, ss));
      }
      *reinterpret_cast<uint4 *>(xtile + tc::tile_off(kTT, t, 8 * kc)) = v;
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 8);
    ss += __shfl_xor_sync(0xffffffffu, ss, 16);
    if ((lane >> 3) == 0) nrm[t] = (float)sqrt(ss);
  }
}

// Split float32 matrix rows into hi/lo bf16 operand tiles (rows = output coordinates).
__device__ __forceinline__ void load_split(unsigned char *hi, unsigned char *lo, const float *__restrict__ src) {
  for (int e = threadIdx.x; e < kTD * kTD; e += blockDim.x) {
    const int n = e >> 7, k = e & 127;
    const float v = __ldg(src + e);
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
    const uint32_t off = tc::tile_off(kTT, n, k);
    *reinterpret_cast<__nv_bfloat16 *>(hi + off) = h;
    *reinterpret_cast<__nv_bfloat16 *>(lo + off) = l;
  }
}

// Eight bf16 values -> one 16-byte chunk.
__device__ __forceinline__ uint4 pack8(const __nv_bfloat16 (&v)[8]) {
  uint4 r;
  r.x = (uint32_t)__bfloat16_as_ushort(v[0]) | ((uint32_t)__bfloat16_as_ushort(v[1]) << 16);
  r.y = (uint32_t)__bfloat16_as_ushort(v[2]) | ((uint32_t)__bfloat16_as_ushort(v[3]) << 16);
  r.z = (uint32_t)__bfloat16_as_ushort(v[4]) | ((uint32_t)__bfloat16_as_ushort(v[5]) << 16);
  r.w = (uint32_t)__bfloat16_as_ushort(v[6]) | ((uint32_t)__bfloat16_as_ushort(v[7]) << 16);
  return r;
}

template <bool QJL, int BITS>
__global__ void __launch_bounds__(tc_threads<QJL>(), QJL ? 1 : 2) quantize_tc_kernel(const QuantParams p) {
  using Lay = TcLayout<QJL>;
  constexpr int NT = tc_threads<QJL>(), NW = NT / 32;
  constexpr int NSPLIT = NT / 128;                    // threads per token in the epilogues
  constexpr int CPT = 128 / NSPLIT;                   // columns per thread (32 or 64)
  constexpr int WPT = CPT * BITS / 32;                // code-stream words per thread
  constexpr int IW = BITS * kTD / 32;                 // code-stream words
  constexpr int RW = IW + (QJL ? kTD / 32 : 0);       // record words
  constexpr int RS = RW | 1;                          // record row stride in shared memory (odd: no bank conflicts)
  constexpr int L = 1 << BITS;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  float *nrm_s = reinterpret_cast<float *>(smem + Lay::kNrm);
  float *cb = reinterpret_cast<float *>(smem + Lay::kCb);
  uint32_t *rec_s = reinterpret_cast<uint32_t *>(smem + Lay::kRec);
  float *rho_s = reinterpret_cast<float *>(smem + Lay::kRho);
  int64_t *slot_s = reinterpret_cast<int64_t *>(smem + Lay::kSlot);
  unsigned char *xtile = smem + Lay::kX;
  const uint32_t bar1 = sbase + Lay::kBar, bar2 = sbase + Lay::kBar + 8;
  const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(p.x);
  const int64_t n_tiles = (p.rows + kTT - 1) / kTT;
  const int n_my = n_tiles > blockIdx.x ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  auto row0_of = [&](int i) -> int64_t { return ((int64_t)blockIdx.x + (int64_t)i * gridDim.x) * kTT; };

  // ---- set-up: split matrices, codebook, barriers, tensor memory, first tile ----
  XRegs<NW> xr;
  if (n_my > 0) load_x<NW>(xr, x, row0_of(0), p.rows, warp, lane);
  load_split(smem + Lay::kPhi, smem + Lay::kPlo, p.Pi);
  if constexpr (QJL) load_split(smem + Lay::kMhi, smem + Lay::kMlo, p.SPiT);
  if (tid < L) cb[tid] = p.codebook[tid];
  if (tid == 0) {
    mbar_init(bar1, 1);
    mbar_init(bar2, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tc::alloc(sbase + Lay::kTslot, Lay::kTmemCols);
    tc::relinquish();
  }
  if (n_my > 0) store_x<NW>(xr, xtile, nrm_s, warp, lane);
  tc::fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (tid < L - 1) cb[16 + tid] = 0.5f * (cb[tid] + cb[tid + 1]);
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + Lay::kTslot);
  const uint32_t d1 = tmem, d2 = tmem + 128;           // accumulator columns
  const uint32_t idesc = tc::idesc_bf16(kTT, kTD);
  auto issue_pi = [&]() {     // D1 = x Pi_hi^T + x Pi_lo^T
    tc::fence_after();
#pragma unroll 1
    for (int part = 0; part < 2; ++part) {
      const uint32_t b = sbase + (part == 0 ? Lay::kPhi : Lay::kPlo);
#pragma unroll 1
      for (int s = 0; s < 8; ++s)
        tc::mma_bf16(d1, tc::smem_desc(sbase + Lay::kX + s * 2 * kLBO, kLBO, kSBO),
                     tc::smem_desc(b + s * 2 * kLBO, kLBO, kSBO), idesc, (part | s) ? 1u : 0u);
    }
    tc::commit(bar1);
  };
  if (tid == 0 && n_my > 0) issue_pi();
  if (n_my > 1) load_x<NW>(xr, x, row0_of(1), p.rows, warp, lane);   // prefetch the next tile
  __syncthreads();
  float th[L - 1], cv[L];
#pragma unroll
  for (int j = 0; j < L - 1; ++j) th[j] = cb[16 + j];
#pragma unroll
  for (int j = 0; j < L; ++j) cv[j] = cb[j];

  // epilogue role: token t = tensor-memory lane, column block h of CPT columns
  const int t_ep = 32 * (warp & 3) + lane, h = warp >> 2;
  const uint32_t lane_ofs = (uint32_t)(32 * (warp & 3)) << 16;
  bool ok = true;
  int it = 0;
  int last_pi = n_my > 0 ? 0 : -1;   // index of the last tile whose first product was issued

  for (; it < n_my; ++it) {
    const int64_t row0 = row0_of(it);
    const float *nrm_cur = nrm_s + 128 * (it & 1);
    // (A) the first product of this tile is done: D1 full, the A tile free
    if (__syncthreads_or(!mbar_wait(bar1, it & 1))) { ok = false; break; }
    tc::fence_after();
    // (B) next tile's rows into the A tile (prefetched into registers one step ago)
    if (it + 1 < n_my) store_x<NW>(xr, xtile, nrm_s + 128 * ((it + 1) & 1), warp, lane);
    // (C) epilogue 1: codes, code-stream words (kept in registers), residual parts
    const float n = nrm_cur[t_ep];
    const float inv = n > 0.f ? 1.0f / n : 0.f;
    uint32_t words[WPT];
#pragma unroll
    for (int w = 0; w < WPT; ++w) words[w] = 0u;
    float e2 = 0.f;
    uint32_t r[CPT];
#pragma unroll
    for (int c = 0; c < CPT / 32; ++c) tc::ld32(d1 + lane_ofs + CPT * h + 32 * c, *reinterpret_cast<uint32_t (*)[32]>(r + 32 * c));
    tc::wait_ld();
#pragma unroll
    for (int g = 0; g < CPT / 8; ++g) {
      float ev[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int j = 8 * g + q;                      // column within this block
        const float y = __uint_as_float(r[j]) * inv;
        uint32_t code = 0;
        float c_sel = cv[0];
#pragma unroll
        for (int k = 0; k < L - 1; ++k) {
          const bool above = y > th[k];
          code += above ? 1u : 0u;
          c_sel = above ? cv[k + 1] : c_sel;
        }
        const int bit = BITS * j, wd = bit >> 5, off = bit & 31;
        words[wd] |= code << off;
        if (off + BITS > 32) words[wd + 1] |= code >> (32 - off);
        ev[q] = n > 0.f ? y - c_sel : 0.f;
        e2 = fmaf(ev[q], ev[q], e2);
      }
      if constexpr (QJL) {
        // e = e_hi + e_lo (bf16 pairs)
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162 hb = __floats2bfloat162_rn(ev[2 * q], ev[2 * q + 1]);
          const float2 hf = __bfloat1622float2(hb);
          const __nv_bfloat162 lb = __floats2bfloat162_rn(ev[2 * q] - hf.x, ev[2 * q + 1] - hf.y);
          hi[q] = *reinterpret_cast<const uint32_t *>(&hb);
          lo[q] = *reinterpret_cast<const uint32_t *>(&lb);
        }
        const uint32_t off = tc::tile_off(kTT, t_ep, CPT * h + 8 * g);
        *reinterpret_cast<uint4 *>(smem + Lay::kEhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(smem + Lay::kElo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    if constexpr (!QJL) {
#pragma unroll
      for (int w = 0; w < WPT; ++w) rec_s[t_ep * RS + WPT * h + w] = words[w];
      if (h == 0) {
        const int64_t row = row0 + t_ep;
        if (row < p.rows) {
          const int64_t sh = row / p.n_tokens, tt = row - sh * p.n_tokens;
          slot_s[t_ep] = sh * p.capacity + p.pos + tt;
        }
      }
    }
    // (D) residual tiles and the next A tile visible to the tensor core; D1 read out
    tc::fence_proxy_async();
    tc::fence_before();
    __syncthreads();
    // (E) sketch product of this tile, then the first product of the next tile
    if (tid == 0) {
      if constexpr (QJL) {
        tc::fence_after();
#pragma unroll 1
        for (int part = 0; part < 4; ++part) {
          const uint32_t a = sbase + ((part >> 1) == 0 ? Lay::kEhi : Lay::kElo);
          const uint32_t b = sbase + ((part & 1) == 0 ? Lay::kMhi : Lay::kMlo);
#pragma unroll 1
          for (int s = 0; s < 8; ++s)
            tc::mma_bf16(d2, tc::smem_desc(a + s * 2 * kLBO, kLBO, kSBO), tc::smem_desc(b + s * 2 * kLBO, kLBO, kSBO),
                         idesc, (part | s) ? 1u : 0u);
        }
        tc::commit(bar2);
      }
      if (it + 1 < n_my) issue_pi();
    }
    if (it + 1 < n_my) last_pi = it + 1;
    // (F) prefetch the tile after next
    if (it + 2 < n_my) load_x<NW>(xr, x, row0_of(it + 2), p.rows, warp, lane);
    if constexpr (QJL) {
      // (G) epilogue 2: sign words; records staged in the (now free) E tiles
      if (__syncthreads_or(!mbar_wait(bar2, it & 1))) { ok = false; break; }
      tc::fence_after();
#pragma unroll
      for (int c = 0; c < CPT / 32; ++c) tc::ld32(d2 + lane_ofs + CPT * h + 32 * c, *reinterpret_cast<uint32_t (*)[32]>(r + 32 * c));
      tc::wait_ld();
#pragma unroll
      for (int w = 0; w < WPT; ++w) rec_s[t_ep * RS + WPT * h + w] = words[w];
#pragma unroll
      for (int c = 0; c < CPT / 32; ++c) {
        uint32_t wsum = 0u;
#pragma unroll
        for (int q = 0; q < 32; ++q) wsum |= (__uint_as_float(r[32 * c + q]) >= 0.f ? 1u : 0u) << q;
        rec_s[t_ep * RS + IW + (CPT / 32) * h + c] = wsum;
      }
      rho_s[128 * h + t_ep] = e2;
      if (h == 0) {
        const int64_t row = row0 + t_ep;
        if (row < p.rows) {
          const int64_t sh = row / p.n_tokens, tt = row - sh * p.n_tokens;
          slot_s[t_ep] = sh * p.capacity + p.pos + tt;
        }
      }
      tc::fence_before();
    }
    __syncthreads();
    // (H) records and norms to the cache
    for (int e = tid; e < kTT * RW; e += NT) {
      const int t = e / RW, w = e - t * RW;
      if (row0 + t < p.rows) p.records[slot_s[t] * RW + w] = rec_s[t * RS + w];
    }
    if (h == 0 && row0 + t_ep < p.rows) {
      p.norm[slot_s[t_ep]] = n;
      if constexpr (QJL) {
        float rr = 0.f;
#pragma unroll
        for (int q = 0; q < NSPLIT; ++q) rr += rho_s[128 * q + t_ep];
        p.rnorm[slot_s[t_ep]] = sqrtf(rr);
      }
    }
    __syncthreads();
  }

  // ---- tear-down: no MMA may still write tensor memory when it is freed ----
  if (!ok) {
    if (last_pi >= 0) mbar_wait(bar1, last_pi & 1);
    if constexpr (QJL) mbar_wait(bar2, it & 1);
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::dealloc(tmem, Lay::kTmemCols);
}

template <bool QJL, int BITS>
cudaError_t launch_tc(const QuantParams &p, cudaStream_t st) {
  auto kern = quantize_tc_kernel<QJL, BITS>;
  constexpr size_t smem = TcLayout<QJL>::kBytes;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (p.rows + kTT - 1) / kTT;
  const int64_t slots = (int64_t)device_sm_count() * (QJL ? 1 : 2);   // values: two CTAs per SM
  const int grid = (int)(tiles < slots ? tiles : slots);
  kern<<<grid, tc_threads<QJL>(), smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Tensor-core quantize for d = 128 bf16 inputs; returns cudaErrorNotSupported for other shapes.
cudaError_t launch_quantize_tc(const QuantParams &p, int bits, bool qjl, cudaStream_t st) {
  if (p.d != 128) return cudaErrorNotSupported;
  switch (bits) {
    case 1: return qjl ? launch_tc<true, 1>(p, st) : launch_tc<false, 1>(p, st);
    case 2: return qjl ? launch_tc<true, 2>(p, st) : launch_tc<false, 2>(p, st);
    case 3: return qjl ? launch_tc<true, 3>(p, st) : launch_tc<false, 3>(p, st);
    default: return qjl ? launch_tc<true, 4>(p, st) : launch_tc<false, 4>(p, st);
  }
}

}  // namespace tq
