// Quantize-append on the tcgen05 tensor cores, for bf16 or fp16 inputs with d = 128.
//
// The method is the encoder of zubnet.ai news, "Google's TurboQuant quantizes
// LLM KV cache to 3.5 bits per channel", paragraph 2, and winningdata.io,
// "TurboQuant: Google comprime KV cache para 3 bits sem perder acuracia",
// "Como o TurboQuant funciona": n = ||x||, y = Pi x / n, code_i = #{j : y_i > t_j},
// and for keys e = y - c[code], rho = ||e||, sign bits of (S Pi^T) e.
//
// Precision. The codes must agree with a float64 encoder except within 1e-5
// of a threshold, so the projections need about 1e-6 of the vectors' scale:
// more than one bf16 product gives. A 16-bit input x is exact in its own type
// (bf16 or fp16; both MMA operands then use that type); each float32 matrix is
// split into two parts of that type, P = P_hi + P_lo with
// |P - P_hi - P_lo| <= 2^-16 |P| elementwise (bf16; fp16 is finer), and Pi x = x Pi_hi^T + x Pi_lo^T
// accumulates in float32 in tensor memory. The residual e (float32) is split
// the same way, and (S Pi^T) e = E_hi M_hi^T + E_hi M_lo^T + E_lo M_hi^T
// (three products; the dropped E_lo M_lo^T is below 2^-16 of the scale).
//
// Warp roles (one persistent CTA per SM, 128-token tiles):
//   - 4 loader warps: global -> registers one tile ahead, ||x|| (written to
//     the cache), registers -> one of two A tiles in shared memory
//     once the tensor core has finished reading it;
//   - one MMA thread: for tile i, D1 = x Pi^T (two products); then, keys, the
//     sketch product of tile i - 1, D2 = E M^T, with E (the split residual) read
//     from tensor memory;
//   - 8 epilogue warps, a warp pair per tensor-memory lane quarter splitting
//     the 128 columns (one token per thread): D1 -> codes -> record words;
//     keys also write the residual parts into tensor memory (two E buffers, so
//     tile i's residual never waits for tile i - 1's sketch product) and then
//     turn D2 of tile i - 1 into sign words and ||e||.
// Tensor memory (keys): D1 [0, 128), D2 [128, 256), E[b] at 256 + 128 b
// (E_hi: 64 columns of bf16 pairs, E_lo: the next 64). D1 and D2 are read
// into registers and released at once, so one buffer of each suffices.
// Every stage hand-off is an mbarrier; every wait is bounded (a timed-out
// role stops and the others time out behind it; no MMA is in flight when
// tensor memory is freed).
// Shared-memory operand tiles use the no-swizzle K-major core-matrix layout of tc.cuh.
#include "common.cuh"
#include "tc.cuh"

namespace tq {

namespace {

constexpr int kTD = 128;                   // head dimension
constexpr int kTT = 128;                   // tokens per tile (MMA M)
constexpr uint32_t kTile = kTT * kTD * 2;  // bytes of one bf16 operand tile (32 KB)
constexpr uint32_t kLBO = kTT * 16;        // K-direction core-matrix stride (2048 B)
constexpr uint32_t kSBO = 128;             // row-direction core-matrix stride
constexpr int kEpiWarps = 8;               // epilogue warps: 2 per lane quarter, 64 columns each
constexpr int kNormRing = 4;               // n_full barriers (the loaders run at most 3 tiles ahead)

// The 16-bit operand type: bf16 (inputs in bf16) or f16 (inputs in fp16). A split
// P = P_hi + P_lo rounds to nearest twice; RN pairs pack two values (lower index
// in the low half).
template <bool F16>
struct H16 {
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    if constexpr (F16) {
      const __half2 h = __floats2half2_rn(a, b);
      return *reinterpret_cast<const uint32_t *>(&h);
    } else {
      const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
      return *reinterpret_cast<const uint32_t *>(&h);
    }
  }
  static __device__ __forceinline__ float lo(uint32_t w) {
    if constexpr (F16) {
      float f;
      asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n cvt.f32.f16 %0, l;\n}" : "=f"(f) : "r"(w));
      return f;
    } else {
      return __uint_as_float(w << 16);
    }
  }
  static __device__ __forceinline__ float hi(uint32_t w) {
    if constexpr (F16) {
      float f;
      asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n cvt.f32.f16 %0, h;\n}" : "=f"(f) : "r"(w));
      return f;
    } else {
      return __uint_as_float(w & 0xFFFF0000u);
    }
  }
  // pair of (hi, lo) words for two floats: hi = RN(v), lo = RN(v - hi)
  static __device__ __forceinline__ void split2(float a, float b, uint32_t &hw, uint32_t &lw) {
    hw = pack(a, b);
    lw = pack(a - lo(hw), b - hi(hw));
  }
};

template <bool QJL>
struct Ws {
  static constexpr int kLoadWarps = 4;
  static constexpr int kMmaWarp = kEpiWarps + kLoadWarps;
  static constexpr int kThreads = 32 * (kMmaWarp + 1);   // 416: at most 4 warps per SM sub-partition (128 registers)
  // dynamic shared memory, byte offsets
  static constexpr uint32_t kPhi = 0, kPlo = kTile;
  static constexpr uint32_t kMhi = 2 * kTile, kMlo = 3 * kTile;              // keys only
  static constexpr uint32_t kX = QJL ? 4 * kTile : 2 * kTile;                // two A tiles
  static constexpr uint32_t kRho = kX + 2 * kTile;                           // float[3][128] (keys)
  static constexpr uint32_t kCb = kRho + (QJL ? 3 * 128 * 4 : 0);            // float[16] centroids
  static constexpr uint32_t kBar = kCb + 64;
  // barriers: x_full[2], x_empty[2], d1_full, d1_empty, e_full, d2_full, d2_empty, n_full[4]
  static constexpr int kBars = 2 + 2 + 1 + 1 + 1 + 1 + 1 + kNormRing;
  static constexpr uint32_t kTslot = kBar + 8 * kBars;
  static constexpr uint32_t kBytes = kTslot + 16;
  static constexpr uint32_t kTmemCols = QJL ? 512 : 128;
  static constexpr uint32_t kD2 = 128, kE = 256;   // tensor-memory column offsets (keys)
  static_assert(kBytes <= 232448, "shared memory over the per-CTA limit");
};

// Barrier addresses (shared-memory offsets from the dynamic base).
template <bool QJL>
struct Bars {
  uint32_t base;
  __device__ uint32_t x_full(int s) const { return base + 8u * s; }
  __device__ uint32_t x_empty(int s) const { return base + 8u * (2 + s); }
  __device__ uint32_t d1_full() const { return base + 8u * 4; }
  __device__ uint32_t d1_empty() const { return base + 8u * 5; }
  __device__ uint32_t e_full() const { return base + 8u * 6; }
  __device__ uint32_t d2_full() const { return base + 8u * 7; }
  __device__ uint32_t d2_empty() const { return base + 8u * 8; }
  __device__ uint32_t n_full(int k) const { return base + 8u * (9 + k); }
};

// Position of a CTA's current tile in the (sequence x head, token) grid, kept
// incrementally so that the tile loop needs no 64-bit division: row0 =
// sh * n_tokens + tt with 0 <= tt < n_tokens; the persistent CTA advances by
// gridDim.x tiles = step_q * n_tokens + step_r rows.
struct TileCursor {
  int64_t sh, tt, step_q, step_r;
  __device__ void init(const QuantParams &p) {
    const int64_t row0 = (int64_t)blockIdx.x * 128, step = (int64_t)gridDim.x * 128;
    sh = row0 / p.n_tokens;
    tt = row0 - sh * p.n_tokens;
    step_q = step / p.n_tokens;
    step_r = step - step_q * p.n_tokens;
  }
  __device__ void advance(const QuantParams &p) {
    tt += step_r;
    sh += step_q;
    if (tt >= p.n_tokens) {
      tt -= p.n_tokens;
      ++sh;
    }
  }
  // cache slot of tile row r
  __device__ int64_t slot(const QuantParams &p, int r) const {
    int64_t t2 = tt + r, s2 = sh;
    while (t2 >= p.n_tokens) {
      t2 -= p.n_tokens;
      ++s2;
    }
    return s2 * p.capacity + p.pos + t2;
  }
};

// Split float32 matrix rows into hi/lo bf16 operand tiles (rows = output coordinates).
// A work item is one 16-byte core-matrix row chunk (8 consecutive k of one row;
// consecutive threads take consecutive rows, so each quarter-warp stores one
// contiguous 128-byte block); every thread issues all of its loads before
// converting, so the L2 round trips overlap instead of serialising.
// src must be 16-byte aligned.
template <int NTHREADS, bool F16>
__device__ __forceinline__ void load_split(unsigned char *hi, unsigned char *lo, const float *__restrict__ src) {
  constexpr int kChunks = kTD * kTD / 8;                       // 2048
  constexpr int kPer = (kChunks + NTHREADS - 1) / NTHREADS;
  float4 v[kPer][2];
#pragma unroll
  for (int c = 0; c < kPer; ++c) {
    const int e = threadIdx.x + c * NTHREADS;
    if (e < kChunks) {
      const float4 *s4 = reinterpret_cast<const float4 *>(src + (e & 127) * kTD + 8 * (e >> 7));
      v[c][0] = __ldg(s4);
      v[c][1] = __ldg(s4 + 1);
    }
  }
#pragma unroll
  for (int c = 0; c < kPer; ++c) {
    const int e = threadIdx.x + c * NTHREADS;
    if (e < kChunks) {
      const float f[8] = {v[c][0].x, v[c][0].y, v[c][0].z, v[c][0].w, v[c][1].x, v[c][1].y, v[c][1].z, v[c][1].w};
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) H16<F16>::split2(f[2 * qq], f[2 * qq + 1], hw[qq], lw[qq]);
      const int n = e & 127, k = 8 * (e >> 7);
      const uint32_t off = tc::tile_off(kTT, n, k);
      *reinterpret_cast<uint4 *>(hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4 *>(lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
}

__device__ __forceinline__ void st_global_v2(uint32_t *p, uint32_t a, uint32_t b) {
  *reinterpret_cast<uint2 *>(p) = make_uint2(a, b);
}

// Code search on masks. gt(a, b) is all ones when a > b (one set.gt: a NaN
// compares false), bsel(m, a, b) = m ? a : b bitwise (one three-input logic op),
// so a code bit costs one compare and each threshold choice one select, with no
// predicate round trips; bits enter the code-stream words by integer
// multiply-add on the FMA pipe (word += -m * 2^pos), leaving the ALU pipe to the
// compares and selects.
__device__ __forceinline__ uint32_t gt(float a, float b) {
  uint32_t m;
  asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(m) : "f"(a), "f"(b));
  return m;
}
__device__ __forceinline__ uint32_t ge0(float a) {
  uint32_t m;
  asm("set.ge.u32.f32 %0, %1, 0f00000000;" : "=r"(m) : "f"(a));
  return m;
}
__device__ __forceinline__ float bsel(uint32_t m, float a, float b) {
  return __uint_as_float((m & __float_as_uint(a)) | (~m & __float_as_uint(b)));
}
// word |= bit at `pos` when m is all ones (the bit is known to be clear)
__device__ __forceinline__ void put_bit(uint32_t &word, uint32_t m, int pos) { word += m * (0u - (1u << pos)); }

// m[k] = all ones iff bit k of code = #{j : y > th[j]} is set (ascending
// thresholds th[0 .. 2^BITS - 2]): a binary search, top bit first.
template <int BITS>
__device__ __forceinline__ void code_masks(float y, const float (&th)[(1 << BITS) - 1], uint32_t (&m)[BITS]) {
  if constexpr (BITS == 1) {
    m[0] = gt(y, th[0]);
  } else if constexpr (BITS == 2) {
    m[1] = gt(y, th[1]);
    m[0] = gt(y, bsel(m[1], th[2], th[0]));
  } else if constexpr (BITS == 3) {
    m[2] = gt(y, th[3]);
    m[1] = gt(y, bsel(m[2], th[5], th[1]));
    m[0] = gt(y, bsel(m[2], bsel(m[1], th[6], th[4]), bsel(m[1], th[2], th[0])));
  } else {
    m[3] = gt(y, th[7]);
    m[2] = gt(y, bsel(m[3], th[11], th[3]));
    m[1] = gt(y, bsel(m[3], bsel(m[2], th[13], th[9]), bsel(m[2], th[5], th[1])));
    const float lo = bsel(m[2], bsel(m[1], th[6], th[4]), bsel(m[1], th[2], th[0]));
    const float hi = bsel(m[2], bsel(m[1], th[14], th[12]), bsel(m[1], th[10], th[8]));
    m[0] = gt(y, bsel(m[3], hi, lo));
  }
}

// c[code] from the code's bit masks.
template <int BITS>
__device__ __forceinline__ float centroid_of(const uint32_t (&m)[BITS], const float (&c)[1 << BITS]) {
  if constexpr (BITS == 1) {
    return bsel(m[0], c[1], c[0]);
  } else {
    auto quad = [&](int o) { return bsel(m[1], bsel(m[0], c[o + 3], c[o + 2]), bsel(m[0], c[o + 1], c[o])); };
    if constexpr (BITS == 2) {
      return quad(0);
    } else if constexpr (BITS == 3) {
      return bsel(m[2], quad(4), quad(0));
    } else {
      return bsel(m[3], bsel(m[2], quad(12), quad(8)), bsel(m[2], quad(4), quad(0)));
    }
  }
}

// Code of coordinate j (BITS bits at stream bit BITS * j) into this thread's words.
template <int BITS, int NW>
__device__ __forceinline__ void put_code(uint32_t (&w)[NW], const uint32_t (&m)[BITS], int j) {
#pragma unroll
  for (int k = 0; k < BITS; ++k) {
    const int bit = BITS * j + k;
    put_bit(w[bit >> 5], m[k], bit & 31);
  }
}

// --------------------------------------------------------------------------
// loader: a group of 4 warps moves whole 128-token tiles. Warp w of the group
// owns tile rows [32 w, 32 w + 32); lane l loads row 32 w + 8 g + (l & 7),
// 16-byte chunks 4 i + (l >> 3) (g, i < 4), so each quarter-warp stores one
// contiguous 128-byte core matrix row block.
// --------------------------------------------------------------------------
struct XRegs {
  uint4 v[4][4];
};

__device__ __forceinline__ void load_tile(XRegs &xr, const uint16_t *__restrict__ x, int64_t row0, int64_t rows,
                                          int w, int lane) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int64_t row = row0 + 32 * w + 8 * g + (lane & 7);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int kc = 4 * i + (lane >> 3);
      xr.v[g][i] = row < rows ? __ldg(reinterpret_cast<const uint4 *>(x + row * kTD + 8 * kc))
                              : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// ||x|| of the four rows this lane holds; every lane of a row's quartet ends
// with the full value. bf16 and fp16 squares are exact in float32, and a float32 sum of
// 128 of them is within 128 * 2^-24 of ||x||^2 (half that on ||x||, inside the
// 1e-5 tolerance); a row whose sum is outside [2^-100, 2^126) (an overflowed
// or underflowed square, or a zero vector) is redone with rescaled values.
// Each row's result depends on that row alone.
template <bool F16>
__device__ __forceinline__ void tile_norms(const XRegs &xr, float (&nrm)[4]) {
  float sf[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t wv[4] = {xr.v[g][i].x, xr.v[g][i].y, xr.v[g][i].z, xr.v[g][i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = H16<F16>::lo(wv[q]), b = H16<F16>::hi(wv[q]);
        s = fmaf(a, a, fmaf(b, b, s));
      }
    }
    s += __shfl_xor_sync(0xffffffffu, s, 8);
    s += __shfl_xor_sync(0xffffffffu, s, 16);
    sf[g] = s;
  }
  bool bad[4], any = false;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    bad[g] = !(sf[g] >= 0x1p-100f && sf[g] < 0x1p126f);
    any |= bad[g];
    nrm[g] = sqrtf(sf[g]);
  }
  // fp16 values are below 2^16 and at least 2^-24, so their sums of squares never leave float32's
  // range (a zero vector sums to exactly 0); for bf16 a row out of range is summed again with its
  // values scaled by a power of two taken from its largest magnitude (exact scaling; squares more
  // than 2^-100 below the largest one are negligible)
  if (!F16 && __any_sync(0xffffffffu, any)) {   // the whole warp takes part in the shuffles
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t mx = 0;   // largest |x| as a bit pattern (ordered like the magnitudes)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t wv[4] = {xr.v[g][i].x, xr.v[g][i].y, xr.v[g][i].z, xr.v[g][i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) mx = max(mx, max((wv[q] << 16) & 0x7FFFFFFFu, wv[q] & 0x7FFF0000u));
      }
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const int e = (int)(mx >> 23) - 127;            // exponent of the largest magnitude
      const float sc = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e (e in [-127, 127])
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t wv[4] = {xr.v[g][i].x, xr.v[g][i].y, xr.v[g][i].z, xr.v[g][i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = H16<F16>::lo(wv[q]) * sc, b = H16<F16>::hi(wv[q]) * sc;
          s = fmaf(a, a, fmaf(b, b, s));
        }
      }
      s += __shfl_xor_sync(0xffffffffu, s, 8);
      s += __shfl_xor_sync(0xffffffffu, s, 16);
      if (bad[g]) nrm[g] = mx == 0 ? 0.f : ldexpf(sqrtf(s), e);
    }
  }
}

__device__ __forceinline__ void store_tile(const XRegs &xr, unsigned char *xtile, int w, int lane) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int t = 32 * w + 8 * g + (lane & 7);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4 *>(xtile + tc::tile_off(kTT, t, 8 * (4 * i + (lane >> 3)))) = xr.v[g][i];
  }
}

// D[tmem] (+)= A[tmem] * B[smem]^T, A in tensor memory (row m = lane m, two bf16
// K-elements per 32-bit column, the lower K index in the low half), issued by one thread.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 4 consecutive 32-bit columns of this warp's 32 lanes (one lane per thread).
__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// The 8 K-steps of one split product D (+)= A B^T with A in tensor memory (64 columns).
__device__ __forceinline__ void mma_tile_ts(uint32_t d, uint32_t a_tmem, uint32_t b, uint32_t idesc,
                                            bool accumulate_first) {
#pragma unroll 1
  for (int s = 0; s < 8; ++s)
    mma_bf16_ts(d, a_tmem + 8 * s, tc::smem_desc(b + s * 2 * kLBO, kLBO, kSBO), idesc,
                (accumulate_first || s) ? 1u : 0u);
}

// Issue the 8 K-steps of one split product D (+)= A B^T (A, B: 128 x 128 bf16 tiles).
__device__ __forceinline__ void mma_tile(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool accumulate_first) {
#pragma unroll 1
  for (int s = 0; s < 8; ++s)
    tc::mma_bf16(d, tc::smem_desc(a + s * 2 * kLBO, kLBO, kSBO), tc::smem_desc(b + s * 2 * kLBO, kLBO, kSBO), idesc,
                 (accumulate_first || s) ? 1u : 0u);
}

template <bool QJL, int BITS, bool F16>
__global__ void __launch_bounds__(Ws<QJL>::kThreads, 1) quantize_tc_kernel(const QuantParams p) {
  using L = Ws<QJL>;
  constexpr int CPT = 64;                         // columns per epilogue thread
  constexpr int WPT = CPT * BITS / 32;            // code-stream words per epilogue thread
  constexpr int IW = BITS * kTD / 32;             // code-stream words per record
  constexpr int RW = IW + (QJL ? kTD / 32 : 0);   // record words
  constexpr int NL = 1 << BITS;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  const Bars<QJL> bar{sbase + L::kBar};
  float *cb = reinterpret_cast<float *>(smem + L::kCb);
  const uint16_t *x = static_cast<const uint16_t *>(p.x);
  const int64_t n_tiles = (p.rows + kTT - 1) / kTT;
  const int n_my = n_tiles > blockIdx.x ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  auto row0_of = [&](int i) -> int64_t { return ((int64_t)blockIdx.x + (int64_t)i * gridDim.x) * kTT; };

  // ---- set-up: split matrices, codebook, barriers, tensor memory ----
  load_split<L::kThreads, F16>(smem + L::kPhi, smem + L::kPlo, p.Pi);
  if constexpr (QJL) load_split<L::kThreads, F16>(smem + L::kMhi, smem + L::kMlo, p.SPiT);
  if (tid < NL) cb[tid] = p.codebook[tid];
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.x_full(s), 128);
      mbar_init(bar.x_empty(s), 1);
    }
    mbar_init(bar.d1_full(), 1);
    mbar_init(bar.d1_empty(), kEpiWarps);
    mbar_init(bar.e_full(), kEpiWarps);
    mbar_init(bar.d2_full(), 1);
    mbar_init(bar.d2_empty(), kEpiWarps);
    for (int k = 0; k < kNormRing; ++k) mbar_init(bar.n_full(k), 128);
    mbar_fence_init();
  }
  if (warp == 0) {
    tc::alloc(sbase + L::kTslot, L::kTmemCols);
    tc::relinquish();
  }
  tc::fence_proxy_async();   // the split matrices, written by generic stores, are read by the tensor core
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + L::kTslot);
  bool ok = true;

  if (warp >= kEpiWarps && warp < L::kMmaWarp) {
    // ------------------------------- loaders -------------------------------
    const int w = warp - kEpiWarps;
    XRegs xr;
    TileCursor cur;
    cur.init(p);
    if (n_my > 0) load_tile(xr, x, row0_of(0), p.rows, w, lane);
    for (int i = 0; i < n_my; ++i) {
      const int64_t row0 = row0_of(i);
      float nrm[4];
      tile_norms<F16>(xr, nrm);
      if ((lane >> 3) == 0) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int r = 32 * w + 8 * g + lane;
          if (row0 + r < p.rows) p.norm[cur.slot(p, r)] = nrm[g];
        }
      }
      cur.advance(p);
      mbar_arrive(bar.n_full(i & (kNormRing - 1)));   // releases this lane's norm stores
      // A tile i & 1 is free once the first product of tile i - 2 is done
      if (i >= 2 && !mbar_wait(bar.x_empty(i & 1), ((i >> 1) - 1) & 1)) {
        ok = false;
        break;
      }
      store_tile(xr, smem + L::kX + (i & 1) * kTile, w, lane);
      tc::fence_proxy_async();
      mbar_arrive(bar.x_full(i & 1));
      if (i + 1 < n_my) load_tile(xr, x, row0_of(i + 1), p.rows, w, lane);
    }
  } else if (warp == L::kMmaWarp) {
    // ----------------------------- MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(kTT, kTD, !F16);
      int last_pi = -1, last_sk = -1;
      auto sketch = [&](int j) -> bool {   // D2 = E_hi M_hi^T + E_hi M_lo^T + E_lo M_hi^T
        if (!mbar_wait(bar.e_full(), j & 1)) return false;
        if (j >= 1 && !mbar_wait(bar.d2_empty(), (j - 1) & 1)) return false;
        tc::fence_after();
        const uint32_t d2 = tmem + L::kD2, e = tmem + L::kE + 128 * (j & 1);
        mma_tile_ts(d2, e, sbase + L::kMhi, idesc, false);
        mma_tile_ts(d2, e, sbase + L::kMlo, idesc, true);
        mma_tile_ts(d2, e + 64, sbase + L::kMhi, idesc, true);
        tc::commit(bar.d2_full());
        last_sk = j;
        return true;
      };
      for (int i = 0; i < n_my && ok; ++i) {
        if (!mbar_wait(bar.x_full(i & 1), (i >> 1) & 1) || (i >= 1 && !mbar_wait(bar.d1_empty(), (i - 1) & 1))) {
          ok = false;
          break;
        }
        tc::fence_after();
        const uint32_t xa = sbase + L::kX + (i & 1) * kTile;
        mma_tile(tmem, xa, sbase + L::kPhi, idesc, false);
        mma_tile(tmem, xa, sbase + L::kPlo, idesc, true);
        tc::commit(bar.x_empty(i & 1));
        tc::commit(bar.d1_full());
        last_pi = i;
        if constexpr (QJL)
          if (i >= 1) ok = sketch(i - 1);
      }
      if constexpr (QJL)
        if (ok && n_my > 0) ok = sketch(n_my - 1);
      // nothing may still write tensor memory when it is freed
      if (last_pi >= 0) mbar_wait(bar.d1_full(), last_pi & 1);
      if (last_sk >= 0) mbar_wait(bar.d2_full(), last_sk & 1);
    }
  } else {
    // ------------------------------- epilogue -------------------------------
    // thread: token t = tensor-memory lane, columns [64 h, 64 h + 64)
    const int q = warp & 3, h = warp >> 2, t = 32 * q + lane;
    const uint32_t lane_ofs = (uint32_t)(32 * q) << 16;
    // thresholds: midpoints of consecutive centroids; keys also keep the centroids
    constexpr int NC = QJL ? NL : 1;
    float th[NL - 1], cvk[NC];
#pragma unroll
    for (int j = 0; j < NL - 1; ++j) th[j] = 0.5f * (cb[j] + cb[j + 1]);
#pragma unroll
    for (int j = 0; j < NC; ++j) cvk[j] = QJL && j < NL ? cb[j] : 0.f;
    float *rho = reinterpret_cast<float *>(smem + L::kRho);   // [3][128]: the h = 1 half's sum of e^2
    float e2prev = 0.f;
    int64_t slot_prev = 0;
    bool vprev = false;
    // slot and ||x|| of the next tile, fetched one tile ahead so that the L2
    // round trip of the loader's norm store overlaps the current tile's work
    float n_next = 0.f;
    int64_t slot_next = 0;
    bool valid_next = false;
    TileCursor cur;
    cur.init(p);
    auto fetch_norm = [&](int i) -> bool {   // tiles are fetched in order 0, 1, 2, ...
      if (!mbar_wait(bar.n_full(i & (kNormRing - 1)), (i / kNormRing) & 1)) return false;
      valid_next = row0_of(i) + t < p.rows;
      slot_next = valid_next ? cur.slot(p, t) : 0;
      n_next = valid_next ? __ldcg(p.norm + slot_next) : 0.f;
      cur.advance(p);
      return true;
    };
    if (n_my > 0) ok = fetch_norm(0);

    // Every epilogue thread runs all n_my + 1 iterations (after a failed wait it
    // skips the work but still meets the pair barrier of each iteration).
    for (int i = 0; i <= n_my; ++i) {
      float e2 = 0.f;
      int64_t slot = 0;
      bool valid = false;
      if (i < n_my && ok) {
        // ---- first epilogue of tile i: codes (and, keys, the residual into E[i & 1]) ----
        if (!mbar_wait(bar.d1_full(), i & 1)) {
          ok = false;
        } else {
          tc::fence_after();
          uint32_t r[CPT];
          tc::ld32(tmem + lane_ofs + CPT * h, *reinterpret_cast<uint32_t (*)[32]>(r));
          tc::ld32(tmem + lane_ofs + CPT * h + 32, *reinterpret_cast<uint32_t (*)[32]>(r + 32));
          tc::wait_ld();
          tc::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar.d1_empty());   // D1 may take the next tile's product
          valid = valid_next;
          slot = slot_next;
          const float n = n_next;
          uint32_t wcur[WPT];
#pragma unroll
          for (int w = 0; w < WPT; ++w) wcur[w] = 0u;
          if constexpr (QJL) {
            // keys: y = D1 / n, code, residual e = y - c[code] (0 for a zero vector), split into
            // bf16 parts and stored to E[i & 1] (free: the sketch product of tile i - 2 is done)
            const float inv = n > 0.f ? 1.0f / n : 0.f;
            const float nz = n > 0.f ? 1.f : 0.f;
            const uint32_t e_hi = tmem + lane_ofs + L::kE + 128 * (i & 1) + 32 * h;
#pragma unroll
            for (int g = 0; g < CPT / 8; ++g) {
              float ev[8];
#pragma unroll
              for (int qq = 0; qq < 8; ++qq) {
                const int j = 8 * g + qq;
                const float y = __uint_as_float(r[j]) * inv;   // 0 for a zero vector
                uint32_t m[BITS];
                code_masks<BITS>(y, th, m);
                put_code<BITS>(wcur, m, j);
                ev[qq] = fmaf(-nz, centroid_of<BITS>(m, cvk), y);
                e2 = fmaf(ev[qq], ev[qq], e2);
              }
              uint32_t hp[4], lp[4];
#pragma unroll
              for (int qq = 0; qq < 4; ++qq) H16<F16>::split2(ev[2 * qq], ev[2 * qq + 1], hp[qq], lp[qq]);
              tmem_st4(e_hi + 4 * g, hp[0], hp[1], hp[2], hp[3]);
              tmem_st4(e_hi + 64 + 4 * g, lp[0], lp[1], lp[2], lp[3]);
            }
            tmem_wait_st();
            tc::fence_before();
            if (h == 1) rho[(i % 3) * 128 + t] = e2;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.e_full());
          } else {
            // values need only the codes: compare D1 = n y against n th (th itself for a zero vector,
            // whose D1 row is 0), which equals y > th up to one rounding
            const float sc = n > 0.f ? n : 1.f;
            float ths[NL - 1];
#pragma unroll
            for (int k = 0; k < NL - 1; ++k) ths[k] = th[k] * sc;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
              uint32_t m[BITS];
              code_masks<BITS>(__uint_as_float(r[j]), ths, m);
              put_code<BITS>(wcur, m, j);
            }
          }
          if (valid) {
            uint32_t *rec = p.records + slot * RW + WPT * h;
#pragma unroll
            for (int w = 0; w < WPT; w += 2) st_global_v2(rec + w, wcur[w], wcur[w + 1]);
          }
        }
      }
      if (i + 1 < n_my && ok) ok = fetch_norm(i + 1);
      if constexpr (QJL) {
        if (i >= 1) {
          // ---- second epilogue of tile i - 1: sign words and ||e|| ----
          const int j = i - 1;
          uint32_t sw[2] = {0u, 0u};
          if (ok && mbar_wait(bar.d2_full(), j & 1)) {
            tc::fence_after();
            uint32_t r[CPT];
            tc::ld32(tmem + lane_ofs + L::kD2 + CPT * h, *reinterpret_cast<uint32_t (*)[32]>(r));
            tc::ld32(tmem + lane_ofs + L::kD2 + CPT * h + 32, *reinterpret_cast<uint32_t (*)[32]>(r + 32));
            tc::wait_ld();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.d2_empty());
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int qq = 0; qq < 32; ++qq) put_bit(sw[c], ge0(__uint_as_float(r[32 * c + qq])), qq);
          } else {
            ok = false;
          }
          // pair barrier (warps q and q + 4): the h = 1 partner's sum of e^2 for tile j is visible
          asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory");
          if (ok && vprev) {
            st_global_v2(p.records + slot_prev * RW + IW + 2 * h, sw[0], sw[1]);
            if (h == 0) p.rnorm[slot_prev] = sqrtf(e2prev + rho[(j % 3) * 128 + t]);
          }
        }
        e2prev = e2;
        slot_prev = slot;
        vprev = valid;
      }
    }
  }

  // ---- tear-down ----
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::dealloc(tmem, L::kTmemCols);
}

template <bool QJL, int BITS, bool F16>
cudaError_t launch_tc(const QuantParams &p, cudaStream_t st) {
  auto kern = quantize_tc_kernel<QJL, BITS, F16>;
  constexpr size_t smem = Ws<QJL>::kBytes;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (p.rows + kTT - 1) / kTT;
  const int64_t slots = (int64_t)device_sm_count();
  const int grid = (int)(tiles < slots ? tiles : slots);
  kern<<<grid, Ws<QJL>::kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <bool F16>
cudaError_t launch_tc_t(const QuantParams &p, int bits, bool qjl, cudaStream_t st) {
  switch (bits) {
    case 1: return qjl ? launch_tc<true, 1, F16>(p, st) : launch_tc<false, 1, F16>(p, st);
    case 2: return qjl ? launch_tc<true, 2, F16>(p, st) : launch_tc<false, 2, F16>(p, st);
    case 3: return qjl ? launch_tc<true, 3, F16>(p, st) : launch_tc<false, 3, F16>(p, st);
    default: return qjl ? launch_tc<true, 4, F16>(p, st) : launch_tc<false, 4, F16>(p, st);
  }
}

}  // namespace

// Tensor-core quantize for d = 128 bf16 or fp16 inputs; returns cudaErrorNotSupported for other shapes.
cudaError_t launch_quantize_tc(const QuantParams &p, int bits, bool qjl, bool f16, cudaStream_t st) {
  if (p.d != 128) return cudaErrorNotSupported;
  return f16 ? launch_tc_t<true>(p, bits, qjl, st) : launch_tc_t<false>(p, bits, qjl, st);
}

}  // namespace tq
