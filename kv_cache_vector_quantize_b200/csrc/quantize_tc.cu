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
// ||x|| is taken as ||Pi x|| (Pi orthogonal) from the same float32 product: the
// split's error moves it by about 2^-17 / sqrt(d) of ||x||, far inside the 1e-5
// tolerance, and no warp has to read the tile a second time.
//
// Warp roles (one persistent CTA per SM, 128-token tiles; keys take them from
// a per-launch counter, so that a CTA on a slower SM takes fewer of them):
//   - one copy thread: takes the next tile (keys: publishes it to the other roles)
//     and copies its x rows by tensor map straight into a ring of A tiles
//     in shared memory (2 for keys, 4 for values), in the 128-byte swizzle layout;
//   - one MMA thread: for tile i, D1 = x Pi^T (two products); then, keys, the
//     sketch product of tile i - 1, D2 = E M^T, with E (the split residual) read
//     from tensor memory;
//   - 16 epilogue warps, 4 per tensor-memory lane quarter, splitting the 128
//     columns into 4 parts of 32 (4 threads per token):
//     D1 -> ||x|| (the token's threads add their parts' squares through shared
//     memory) -> codes -> record words;
//     keys also write the residual parts into tensor memory (two E buffers, so
//     tile i's residual never waits for tile i - 1's sketch product) and then
//     turn D2 of tile i - 1 into sign words and ||e||;
//   - integer-rate keys with 2- or more-bit codes: that last step runs on 4
//     sign warps of its own (a whole token per thread), so the epilogue warps
//     never wait for the sketch product.
// Tensor memory (keys): D1 [0, 128), D2 [128, 256), E[b] at 256 + 128 b
// (E_hi: 64 columns of bf16 pairs, E_lo: the next 64). D1 and D2 are read
// into registers and released at once, so one buffer of each suffices.
// Every stage hand-off is an mbarrier; every wait is bounded (a timed-out
// role stops and the others time out behind it; no MMA is in flight when
// tensor memory is freed).
// Shared-memory operand tiles use the 128-byte swizzle K-major layout of tc.cuh (sw128_off).
//
// Mixed rate (MIXED: fractional bits per channel, the first 64 rotated
// coordinates at BITS + 1 code bits): the epilogue threads of columns [0, 64)
// search the wider codebook and write their 64 (BITS+1)-bit codes first, the
// threads of columns [64, 128) the BITS-bit codebook and codes after them; the
// products are the same.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "tc.cuh"

namespace tq {

namespace {

constexpr int kTD = 128;                   // head dimension
constexpr int kTT = 128;                   // tokens per tile (MMA M)
constexpr uint32_t kTile = kTT * kTD * 2;  // bytes of one bf16 operand tile (32 KB)

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

// Tile schedule of the keys. The copy thread takes the CTA's tiles one at a time, from a per-launch counter
// when QuantParams::tiles is set (dynamic: a CTA on a slower SM simply takes fewer tiles) or else as
// blockIdx.x + i gridDim.x, and publishes each as entry i of a ring in shared memory: the tile's first row
// and its position in the (sequence x head, token) grid, row0 = sh n_tokens + tt with 0 <= tt < n_tokens,
// or row0 = -1 after the last tile. The other roles read entry i when they start tile i. The ring has
// kRingN entries: no role is more than 6 tiles behind the copy thread (the input stages, the D1 and D2
// hand-offs and the two E buffers bound the lead), so an entry is never overwritten before all have read it.
// Measured on the large-model layer's fresh inputs: keys 2.92 -> 2.80 ms; values, whose per-CTA times
// hardly differ, 1.78 -> 1.83 ms, so they keep the fixed order (blockIdx.x + i gridDim.x) and no ring.
constexpr int kRingN = 16;
struct TileSlot {
  int64_t row0, sh, tt;
};

// Keys with 2- and 3-bit codes at the integer rate: 4 sign warps (one per lane quarter, a whole token per
// thread) turn D2 into sign words and rho, so the epilogue warps run only the first epilogue (measured:
// 3-bit codes 16% faster, 2-bit codes 1-2%, 1-bit codes 3% slower, so those keep one epilogue loop); the
// mixed rate's epilogue warps do both (measured 6% faster than with sign warps at 2 + 3 bits).
template <bool QJL, int BITS, bool MIXED>
constexpr bool epi_split() { return QJL && !MIXED && BITS >= 2; }
// The 2-bit mixed-rate keys issue each K step's descriptors afresh, one step at a time: measured 4.10 ms
// per 16.8 M keys against 4.46 ms with the precomputed descriptors of the other widths.
template <bool QJL, int BITS, bool MIXED>
constexpr bool mma_paced() { return QJL && MIXED && BITS >= 2; }

// Four epilogue threads per token (parts of kTD / 4 columns), four warps per tensor-memory lane quarter:
// measured against two threads per token, keys 15-20% faster (the residual's tensor-memory stores and
// its split wait less), values 3% (2-bit codes) to 10% (4-bit codes).
template <bool QJL, bool SPLIT>
struct Ws {
  static constexpr int kParts = 4;                       // epilogue threads per token
  static constexpr int kEpiWarps = 4 * kParts;
  static constexpr bool kSplit = SPLIT;
  static constexpr int kSignWarps = kSplit ? 4 : 0;
  static constexpr int kTmaWarp = kEpiWarps + kSignWarps;
  static constexpr int kMmaWarp = kTmaWarp + 1;
  static constexpr int kThreads = 32 * (kMmaWarp + 1);   // 576 (96 registers) or, with sign warps, 704 (80)
  static constexpr int kNX = QJL ? 2 : 4;                // A-tile stages (tensor-map copies in flight)
  // D1 = x Pi_hi^T + x Pi_lo^T: two N = 128 products accumulated into one buffer (keys: one buffer,
  // values: two, so a tile's products run while the epilogue reads the previous one)
  static constexpr int kND1 = QJL ? 1 : 2;
  // dynamic shared memory, byte offsets
  static constexpr uint32_t kPhi = 0, kPlo = kTile;
  static constexpr uint32_t kMhi = 2 * kTile, kMlo = 3 * kTile;              // keys only
  static constexpr uint32_t kX = QJL ? 4 * kTile : 2 * kTile;                // kNX A tiles
  static constexpr uint32_t kRho = kX + kNX * kTile;                         // float[3][kParts][128] (keys)
  static constexpr uint32_t kXch = kRho + (QJL ? 3 * kParts * 128 * 4 : 0);  // float2[2][kParts][128]: ||x|| parts
  static constexpr uint32_t kCb = kXch + 2 * kParts * 128 * 8;               // float[32] centroids (two codebooks if mixed)
  static constexpr uint32_t kRing = kCb + 128;                               // TileSlot[kRingN]: the tile schedule
  static constexpr uint32_t kBar = kRing + kRingN * sizeof(TileSlot);
  // barriers: x_full[4], x_empty[4], d1_full[2], d1_empty[2], e_full, d2_full, d2_empty, rho_full[3], slot_full[kRingN]
  static constexpr int kBars = 4 + 4 + 2 + 2 + 1 + 1 + 1 + 3 + kRingN;
  static constexpr uint32_t kTslot = kBar + 8 * kBars;
  static constexpr uint32_t kBytes = kTslot + 16;
  static constexpr uint32_t kTmemCols = QJL ? 512 : 256;   // keys: D1, D2, E[0], E[1]; values: D1[0], D1[1]
  static constexpr uint32_t kD2 = 128, kE = 256;   // tensor-memory column offsets (keys)
  static_assert(kBytes <= 232448, "shared memory over the per-CTA limit");
};

// Barrier addresses (shared-memory offsets from the dynamic base).
template <bool QJL>
struct Bars {
  uint32_t base;
  __device__ uint32_t x_full(int s) const { return base + 8u * s; }
  __device__ uint32_t x_empty(int s) const { return base + 8u * (4 + s); }
  __device__ uint32_t d1_full(int b) const { return base + 8u * (8 + b); }
  __device__ uint32_t d1_empty(int b) const { return base + 8u * (10 + b); }
  __device__ uint32_t e_full() const { return base + 8u * 12; }
  __device__ uint32_t d2_full() const { return base + 8u * 13; }
  __device__ uint32_t d2_empty() const { return base + 8u * 14; }
  __device__ uint32_t rho_full(int k) const { return base + 8u * (15 + k); }   // rho of tile i in slot i % 3
  __device__ uint32_t slot_full(int k) const { return base + 8u * (18 + k); }  // schedule entry i in slot i % kRingN
};

// Position of a CTA's current tile in the fixed order (values), kept incrementally so that the tile loop
// needs no 64-bit division: row0 = sh * n_tokens + tt with 0 <= tt < n_tokens; the persistent CTA
// advances by gridDim.x tiles = step_q * n_tokens + step_r rows.
struct TileCursor {
  int64_t sh, tt, step_q, step_r, base;   // base = slot of the tile's first row
  __device__ void init(const QuantParams &p) {
    const int64_t row0 = (int64_t)blockIdx.x * 128, step = (int64_t)gridDim.x * 128;
    sh = row0 / p.n_tokens;
    tt = row0 - sh * p.n_tokens;
    step_q = step / p.n_tokens;
    step_r = step - step_q * p.n_tokens;
    base = sh * p.capacity + p.pos + tt;
  }
  __device__ void advance(const QuantParams &p) {
    tt += step_r;
    sh += step_q;
    if (tt >= p.n_tokens) {
      tt -= p.n_tokens;
      ++sh;
    }
    base = sh * p.capacity + p.pos + tt;
  }
  // cache slot of tile row r
  __device__ int64_t slot(const QuantParams &p, int r) const {
    if (tt + r < p.n_tokens) return base + r;   // the row is in the tile's first (sequence, head)
    int64_t t2 = tt + r, s2 = sh;
    while (t2 >= p.n_tokens) {
      t2 -= p.n_tokens;
      ++s2;
    }
    return s2 * p.capacity + p.pos + t2;
  }
};

// Cache slot of row r of a tile whose first row is (sh, tt).
__device__ __forceinline__ int64_t tile_row_slot(const QuantParams &p, const TileSlot &ts, int r) {
  int64_t t2 = ts.tt + r, s2 = ts.sh;
  while (t2 >= p.n_tokens) {
    t2 -= p.n_tokens;
    ++s2;
  }
  return s2 * p.capacity + p.pos + t2;
}

// Split float32 matrix rows into hi/lo bf16 operand tiles (rows = output coordinates).
// A work item is one 16-byte row chunk (8 consecutive k of one row;
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
      const uint32_t o = tc::sw128_off(kTT, n, k);
      *reinterpret_cast<uint4 *>(hi + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4 *>(lo + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
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

// Sign word of the 32 sketch values v[o, o + 32): bit k = (v[o + k] >= 0). The values' sign bits are
// shifted in from the top, one funnel shift each, and the word inverted: that is v >= 0 for every value
// but -0.0, which it reads as negative. The product gives an exact zero only for a zero residual (a
// zero vector); the caller sets that token's words to all ones, as the sign of 0 is +1.
template <int O, int N>
__device__ __forceinline__ uint32_t sign_word(const uint32_t (&v)[N]) {
  static_assert(O + 32 <= N, "32 values from offset O");
  uint32_t w = 0u;
#pragma unroll
  for (int k = 31; k >= 0; --k) w = __funnelshift_l(v[O + k], w, 1);
  return ~w;
}

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

// Code search on the FMA pipe. With B = 2^126, sat(y B - t B) is 1.0 when y > t and 0.0 when
// y <= t for the coordinates of a unit vector (|y - t| is either 0 or at least one float32 ulp of
// t, times 2^126 >= 1; the middle threshold 0 is passed by any normal y > 0). The code is built as
// a float (sum of its bit flags times their weights) plus 2^23, whose bit pattern is 0x4B000000 +
// code, and added into the words by integer multiply-add; the 0x4B000000 parts are subtracted per
// word once (kMagicSum). Threshold choices of the binary search are multiply-adds of the flags.
__device__ __forceinline__ float sat_gt(float y, float tb) {   // 1.0 if y > t else 0.0 (tb = t B)
  float r;
  asm("fma.rn.sat.f32 %0, %1, 0f7E800000, %2;" : "=f"(r) : "f"(y), "f"(-tb));
  return r;
}

// bit flags f[k] (0.0 or 1.0) of code = #{j : y > th[j]}; tb[] = th[] * 2^126, dt[] precomputed differences
template <int BITS>
struct FmaSearch {
  float tb[(1 << BITS) - 1];
  __device__ void init(const float (&th)[(1 << BITS) - 1]) {
#pragma unroll
    for (int k = 0; k < (1 << BITS) - 1; ++k) tb[k] = th[k] * 0x1p126f;
  }
  __device__ __forceinline__ void flags(float y, float (&f)[BITS]) const {
    if constexpr (BITS == 1) {
      f[0] = sat_gt(y, tb[0]);
    } else if constexpr (BITS == 2) {
      f[1] = sat_gt(y, tb[1]);
      f[0] = sat_gt(y, fmaf(f[1], tb[2] - tb[0], tb[0]));
    } else if constexpr (BITS == 3) {
      f[2] = sat_gt(y, tb[3]);
      f[1] = sat_gt(y, fmaf(f[2], tb[5] - tb[1], tb[1]));
      const float lo = fmaf(f[1], tb[2] - tb[0], tb[0]), hi = fmaf(f[1], tb[6] - tb[4], tb[4]);
      f[0] = sat_gt(y, fmaf(f[2], hi - lo, lo));
    } else {
      f[3] = sat_gt(y, tb[7]);
      f[2] = sat_gt(y, fmaf(f[3], tb[11] - tb[3], tb[3]));
      const float l1 = fmaf(f[2], tb[5] - tb[1], tb[1]), h1 = fmaf(f[2], tb[13] - tb[9], tb[9]);
      f[1] = sat_gt(y, fmaf(f[3], h1 - l1, l1));
      const float a = fmaf(f[1], tb[2] - tb[0], tb[0]), b = fmaf(f[1], tb[6] - tb[4], tb[4]);
      const float c = fmaf(f[1], tb[10] - tb[8], tb[8]), d = fmaf(f[1], tb[14] - tb[12], tb[12]);
      const float lo = fmaf(f[2], b - a, a), hi = fmaf(f[2], d - c, c);
      f[0] = sat_gt(y, fmaf(f[3], hi - lo, lo));
    }
  }
};

// 0x4B000000 + v for a small integer-valued float v >= 0
__device__ __forceinline__ uint32_t magic(float v) { return __float_as_uint(v + 8388608.0f); }

// Adds the code of coordinate j (flags f) into this thread's words; the words carry
// 0x4B000000-multiples that fix_words removes.
template <int BITS, int NW>
__device__ __forceinline__ void put_code_f(uint32_t (&w)[NW], const float (&f)[BITS], int j) {
  const int bit = BITS * j, wd = bit >> 5, off = bit & 31;
  if (off + BITS <= 32) {
    float v = f[0];
#pragma unroll
    for (int k = 1; k < BITS; ++k) v = fmaf(f[k], (float)(1 << k), v);
    w[wd] += magic(v) * (1u << off);
  } else {
#pragma unroll
    for (int k = 0; k < BITS; ++k) {
      const int b = bit + k;
      w[b >> 5] += magic(f[k]) * (1u << (b & 31));
    }
  }
}

// Subtracts the 0x4B000000 terms put_code_f added for coordinates [0, n) of this thread.
template <int BITS, int NW>
__device__ __forceinline__ void fix_words(uint32_t (&w)[NW], int n) {
  uint32_t corr[NW];
#pragma unroll
  for (int k = 0; k < NW; ++k) corr[k] = 0u;
#pragma unroll
  for (int j = 0; j < n; ++j) {
    const int bit = BITS * j, off = bit & 31;
    if (off + BITS <= 32) {
      corr[bit >> 5] += 0x4B000000u * (1u << off);
    } else {
#pragma unroll
      for (int k = 0; k < BITS; ++k) corr[(bit + k) >> 5] += 0x4B000000u * (1u << ((bit + k) & 31));
    }
  }
#pragma unroll
  for (int k = 0; k < NW; ++k) w[k] -= corr[k];
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

// One 2-D tensor-map copy: 64 columns (128 bytes) x 128 rows, landing as one K block of the
// 128-byte swizzle layout (16 KB); completion counted on `bar`.
__device__ __forceinline__ void tma_x_chunk(uint32_t dst, const CUtensorMap *map, int col, int row, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(row), "r"(bar)
      : "memory");
}

// ||x|| = ||Pi x|| of token t from its D1 row, whose 128 columns are split over
// the NP epilogue threads of the token (part h; warps q + 4 h). Each thread sums
// its part's squares; a part whose sum leaves [2^-100, 2^125) (a zero part,
// underflowed or overflowed squares) is summed again with its values scaled by
// 2^-e, e the exponent of its largest magnitude, so that it stands for s * 4^e.
// The threads swap (s, e) through shared memory (xs: float2[NP][128]) and each
// combines the NP parts in the same order, so all get the same n. All 32 lanes
// of the NP warps must call it (named barrier 1 + q).
template <int CPT, int NP>
__device__ __forceinline__ float part_norm(const uint32_t (&r)[CPT], float2 *xs, int h, int t, int q) {
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < CPT; ++j) s = fmaf(__uint_as_float(r[j]), __uint_as_float(r[j]), s);
  int e = 0;
  if (!(s >= 0x1p-100f && s < 0x1p125f)) {
    uint32_t mx = 0;   // largest magnitude as a bit pattern (ordered like the magnitudes)
#pragma unroll
    for (int j = 0; j < CPT; ++j) mx = max(mx, r[j] & 0x7FFFFFFFu);
    if (mx == 0) {
      s = 0.f;
      e = -512;   // an all-zero part: never the larger exponent, and its share underflows to 0
    } else {
      e = max(-126, min(126, (int)(mx >> 23) - 127));
      const float sc = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e, a normal number
      s = 0.f;
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const float v = __uint_as_float(r[j]) * sc;
        s = fmaf(v, v, s);
      }
    }
  }
  xs[h * 128 + t] = make_float2(s, __int_as_float(e));
  asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "n"(32 * NP) : "memory");
  float2 a[NP];
  int any = 0, E = -512;
#pragma unroll
  for (int k = 0; k < NP; ++k) {
    a[k] = xs[k * 128 + t];
    any |= __float_as_int(a[k].y);
    E = max(E, __float_as_int(a[k].y));
  }
  if (any == 0) {   // no part rescaled: the plain sum (fewer than 2^126 in total)
    float tot = a[0].x;
#pragma unroll
    for (int k = 1; k < NP; ++k) tot += a[k].x;
    return sqrtf(tot);
  }
  float tot = 0.f;
#pragma unroll
  for (int k = 0; k < NP; ++k) tot += ldexpf(a[k].x, 2 * (__float_as_int(a[k].y) - E));
  return ldexpf(sqrtf(tot), E);
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

// The MMA thread builds each operand's shared-memory descriptor once per product and steps it along K by
// adding the step's byte offset / 16 to the start-address field (the field cannot carry: shared
// addresses stay below 256 KB), so a K step costs one add instead of a descriptor build. PACED: the
// descriptors are built at each step, a loop of one step per iteration.

// The 8 K-steps of one split product D (+)= A B^T with A in tensor memory (64 columns).
template <bool PACED>
__device__ __forceinline__ void mma_tile_ts(uint32_t d, uint32_t a_tmem, uint32_t b, uint32_t idesc,
                                            bool accumulate_first) {
  if constexpr (PACED) {
#pragma unroll 1
    for (int s = 0; s < 8; ++s)
      mma_bf16_ts(d, a_tmem + 8 * s, tc::smem_desc_sw128(tc::sw128_kstep(b, kTT, s)), idesc,
                  (accumulate_first || s) ? 1u : 0u);
  } else {
    const uint64_t db = tc::smem_desc_sw128(b);
#pragma unroll
    for (int s = 0; s < 8; ++s)
      mma_bf16_ts(d, a_tmem + 8 * s, db + (tc::sw128_kstep(0, kTT, s) >> 4), idesc,
                  (accumulate_first || s) ? 1u : 0u);
  }
}

// Issue the 8 K-steps of one split product D (+)= A B^T (A, B: 128 x 128 bf16 tiles).
template <bool PACED>
__device__ __forceinline__ void mma_tile(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool accumulate_first) {
  if constexpr (PACED) {
#pragma unroll 1
    for (int s = 0; s < 8; ++s)
      tc::mma_bf16(d, tc::smem_desc_sw128(tc::sw128_kstep(a, kTT, s)), tc::smem_desc_sw128(tc::sw128_kstep(b, kTT, s)),
                   idesc, (accumulate_first || s) ? 1u : 0u);
  } else {
    const uint64_t da = tc::smem_desc_sw128(a), db = tc::smem_desc_sw128(b);
#pragma unroll
    for (int s = 0; s < 8; ++s)
      tc::mma_bf16(d, da + (tc::sw128_kstep(0, kTT, s) >> 4), db + (tc::sw128_kstep(0, kTT, s) >> 4), idesc,
                   (accumulate_first || s) ? 1u : 0u);
  }
}

template <bool QJL, int BITS, bool F16, bool MIXED = false>
__global__ void __launch_bounds__(Ws<QJL, epi_split<QJL, BITS, MIXED>()>::kThreads, 1)
    quantize_tc_kernel(const QuantParams p, const __grid_constant__ CUtensorMap xmap) {
  using L = Ws<QJL, epi_split<QJL, BITS, MIXED>()>;
  constexpr bool kPaced = mma_paced<QJL, BITS, MIXED>();
  constexpr int kParts = L::kParts;
  constexpr int kEpiWarps = L::kEpiWarps;
  constexpr int CPT = kTD / kParts;               // columns per epilogue thread
  constexpr int B0 = MIXED ? BITS + 1 : BITS;     // code bits of columns [0, 64) (the other half: BITS)
  constexpr int IW = (B0 + BITS) * (kTD / 2) / 32;   // code-stream words per record
  constexpr int RW = IW + (QJL ? kTD / 32 : 0);   // record words
  constexpr int NL = 1 << BITS;
  constexpr int NLM = 1 << B0;                    // levels of the wider codebook
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();   // launched as a dependent of the previous work: it must be finished first
  const uint32_t sbase = smem_u32(smem);
  const Bars<QJL> bar{sbase + L::kBar};
  float *cb = reinterpret_cast<float *>(smem + L::kCb);
  const int64_t n_tiles = (p.rows + kTT - 1) / kTT;
  constexpr bool kSched = QJL;   // keys: the tile schedule through the ring; values: the fixed order
  const int n_fixed = n_tiles > blockIdx.x ? (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  auto row0_of = [&](int i) -> int64_t { return ((int64_t)blockIdx.x + (int64_t)i * gridDim.x) * kTT; };
  TileSlot *ring = reinterpret_cast<TileSlot *>(smem + L::kRing);
  // schedule entry i (row0 = -1: no more tiles, also after a failed wait)
  auto take = [&](int i) -> TileSlot {
    TileSlot ts{-1, 0, 0};
    if (mbar_wait(bar.slot_full(i % kRingN), (i / kRingN) & 1)) {
      const volatile TileSlot *e = ring + i % kRingN;
      ts.row0 = e->row0;
      ts.sh = e->sh;
      ts.tt = e->tt;
    }
    return ts;
  };

  // ---- set-up: split matrices, codebook, barriers, tensor memory ----
  load_split<L::kThreads, F16>(smem + L::kPhi, smem + L::kPlo, p.Pi);
  if constexpr (QJL) load_split<L::kThreads, F16>(smem + L::kMhi, smem + L::kMlo, p.SPiT);
  if (tid < NL + (MIXED ? NLM : 0)) cb[tid] = p.codebook[tid];
  if (tid == 0) {
    for (int s = 0; s < L::kNX; ++s) {
      mbar_init(bar.x_full(s), 1);                         // the copy thread's expect_tx
      mbar_init(bar.x_empty(s), 1);   // the first product's commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar.d1_full(b), 1);
      mbar_init(bar.d1_empty(b), kEpiWarps);
    }
    mbar_init(bar.e_full(), kEpiWarps);
    mbar_init(bar.d2_full(), 1);
    mbar_init(bar.d2_empty(), L::kSplit ? L::kSignWarps : kEpiWarps);
    for (int k = 0; k < 3; ++k) mbar_init(bar.rho_full(k), kEpiWarps);
    for (int k = 0; k < kRingN; ++k) mbar_init(bar.slot_full(k), 1);   // the copy thread's arrive
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

  if (warp == L::kTmaWarp) {
    // --------------------------- tensor-map copies ---------------------------
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
      int issued = 0;
      if constexpr (kSched) {
        // the next tile's ticket is drawn one tile ahead, so the atomic's round trip overlaps the copies
        int64_t ticket = p.tiles ? (int64_t)atomicAdd(p.tiles, 1u) : (int64_t)blockIdx.x;
        for (int i = 0;; ++i) {
          const int64_t tile = ticket < n_tiles ? ticket : -1;
          const int s = i % L::kNX;
          // A tile s is free once tile i - kNX's first product is done
          const bool go = tile >= 0 && (i < L::kNX || mbar_wait(bar.x_empty(s), ((i / L::kNX) - 1) & 1));
          TileSlot *e = ring + i % kRingN;
          if (go) {
            const int64_t row0 = tile * kTT, sh = row0 / p.n_tokens;
            e->row0 = row0;
            e->sh = sh;
            e->tt = row0 - sh * p.n_tokens;
            ticket = p.tiles ? (int64_t)atomicAdd(p.tiles, 1u) : ticket + gridDim.x;
          } else {
            e->row0 = -1;
          }
          mbar_arrive(bar.slot_full(i % kRingN));   // release: the entry is visible to whoever waits on it
          if (!go) break;
          mbar_arrive_expect_tx(bar.x_full(s), kTile);
          const uint32_t dst = sbase + L::kX + s * kTile;
#pragma unroll 1
          for (int kb = 0; kb < 2; ++kb) tma_x_chunk(dst + kb * (kTile / 2), &xmap, 64 * kb, (int)e->row0, bar.x_full(s));
          ++issued;
        }
      } else {
        for (int i = 0; i < n_fixed; ++i) {
          const int s = i % L::kNX;
          // A tile s is free once tile i - kNX's first product is done
          if (i >= L::kNX && !mbar_wait(bar.x_empty(s), ((i / L::kNX) - 1) & 1)) break;
          mbar_arrive_expect_tx(bar.x_full(s), kTile);
          const uint32_t dst = sbase + L::kX + s * kTile;
          const int row0 = (int)row0_of(i);
#pragma unroll 1
          for (int kb = 0; kb < 2; ++kb) tma_x_chunk(dst + kb * (kTile / 2), &xmap, 64 * kb, row0, bar.x_full(s));
          ++issued;
        }
      }
      // no copy may still be landing when the CTA exits
      for (int i = max(0, issued - L::kNX); i < issued; ++i) mbar_wait(bar.x_full(i % L::kNX), (i / L::kNX) & 1);
    }
  } else if (L::kSplit && warp >= kEpiWarps && warp < L::kTmaWarp) {
    // ------------------------------- sign warps -------------------------------
    // thread: token t = tensor-memory lane, all 128 sketch columns. Tile j: wait for the epilogue's
    // sums of e^2 (rho_full) and the sketch product (d2_full), read both, release D2, store.
    const int q = warp & 3, t = 32 * q + lane;
    const uint32_t lane_ofs = (uint32_t)(32 * q) << 16;
    const float *rho = reinterpret_cast<const float *>(smem + L::kRho);   // [3][kParts][128]
    for (int j = 0;; ++j) {
      const TileSlot ts = take(j);   // the same entry for the whole warp (a failed wait: row0 = -1 for all)
      if (!__all_sync(0xffffffffu, ts.row0 >= 0)) break;
      const bool valid = ts.row0 + t < p.rows;
      const int64_t slot = valid ? tile_row_slot(p, ts, t) : 0;
      // the tensor-memory loads are warp-wide: the whole warp loads or none of it does
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(bar.rho_full(j % 3), (j / 3) & 1) &&
                                       mbar_wait_sleep(bar.d2_full(), j & 1)))
        break;
      tc::fence_after();
      uint32_t sw[4];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[64];
        tc::ld32(tmem + lane_ofs + L::kD2 + 64 * hh, *reinterpret_cast<uint32_t (*)[32]>(r));
        tc::ld32(tmem + lane_ofs + L::kD2 + 64 * hh + 32, *reinterpret_cast<uint32_t (*)[32]>(r + 32));
        tc::wait_ld();
        // (the sign words by compare and multiply-add: sign_word's shift chain spills here at 80 registers)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          sw[2 * hh + c] = 0u;
#pragma unroll
          for (int qq = 0; qq < 32; ++qq) put_bit(sw[2 * hh + c], ge0(__uint_as_float(r[32 * c + qq])), qq);
        }
      }
      // rho of tile j is read before D2 is released: the epilogue cannot reuse its slot until the sketch
      // of tile j + 1, which waits for that release, has been issued
      float e2s = 0.f;
#pragma unroll
      for (int k = 0; k < L::kParts; ++k) e2s += rho[((j % 3) * L::kParts + k) * 128 + t];
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.d2_empty());   // D2 may take the next tile's sketch
      if (valid) {
        uint32_t *sdst = p.records + slot * RW + IW;
        st_global_v2(sdst, sw[0], sw[1]);
        st_global_v2(sdst + 2, sw[2], sw[3]);
        p.rnorm[slot] = sqrtf(e2s);
      }
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
        mma_tile_ts<kPaced>(d2, e, sbase + L::kMhi, idesc, false);
        mma_tile_ts<kPaced>(d2, e, sbase + L::kMlo, idesc, true);
        mma_tile_ts<kPaced>(d2, e + 64, sbase + L::kMhi, idesc, true);
        tc::commit(bar.d2_full());
        last_sk = j;
        return true;
      };
      int n_my = 0;
      for (int i = 0; ok; ++i) {
        if constexpr (kSched) {
          if (take(i).row0 < 0) break;
        } else {
          if (i >= n_fixed) break;
        }
        const int xs = i % L::kNX;
        const int db = i % L::kND1;
        if (!mbar_wait(bar.x_full(xs), (i / L::kNX) & 1) ||
            (i >= L::kND1 && !mbar_wait(bar.d1_empty(db), ((i / L::kND1) - 1) & 1))) {
          ok = false;
          break;
        }
        tc::fence_after();
        const uint32_t xa = sbase + L::kX + xs * kTile;
        mma_tile<kPaced>(tmem + 128 * db, xa, sbase + L::kPhi, idesc, false);
        mma_tile<kPaced>(tmem + 128 * db, xa, sbase + L::kPlo, idesc, true);
        tc::commit(bar.x_empty(xs));
        tc::commit(bar.d1_full(db));
        last_pi = i;
        n_my = i + 1;
        if constexpr (QJL)
          if (i >= 1) ok = sketch(i - 1);
      }
      if constexpr (QJL)
        if (ok && n_my > 0) ok = sketch(n_my - 1);
      // nothing may still write tensor memory when it is freed
      if (last_pi >= 0) mbar_wait(bar.d1_full(last_pi % L::kND1), (last_pi / L::kND1) & 1);
      if (last_sk >= 0) mbar_wait(bar.d2_full(), last_sk & 1);
    }
  } else {
    // ------------------------------- epilogue -------------------------------
    // thread: token t = tensor-memory lane, columns [CPT h, CPT h + CPT)
    const int q = warp & 3, h = warp >> 2, t = 32 * q + lane;
    const uint32_t lane_ofs = (uint32_t)(32 * q) << 16;
    // thresholds: midpoints of consecutive centroids of this part's codebook (mixed: the wider one
    // for columns [0, 64), stored after the narrower one); keys also keep the centroids
    const bool wide = MIXED && h < kParts / 2;
    // this part's first code-stream word: mixed, the wider parts come first
    const int woff = !MIXED ? h * (CPT * BITS / 32)
                            : (wide ? h * (CPT * B0 / 32) : (kParts / 2) * (CPT * B0 / 32) + (h - kParts / 2) * (CPT * BITS / 32));
    const float *cbh = wide ? cb + NL : cb;
    const int nlh = wide ? NLM : NL;
    constexpr int NC = QJL ? NLM : 1;
    float th[NLM - 1], cvk[NC];
#pragma unroll
    for (int j = 0; j < NLM - 1; ++j) th[j] = j < nlh - 1 ? 0.5f * (cbh[j] + cbh[j + 1]) : 0.f;
#pragma unroll
    for (int j = 0; j < NC; ++j) cvk[j] = QJL && j < nlh ? cbh[j] : 0.f;
    float *rho = reinterpret_cast<float *>(smem + L::kRho);   // [3][kParts][128]: each part's sum of e^2
    int64_t slot_prev = 0;
    bool vprev = false;
    float2 *xch = reinterpret_cast<float2 *>(smem + L::kXch);   // [2][kParts][128]: ||x|| parts, by tile parity
    TileCursor cur;   // the fixed order (values)
    if constexpr (!kSched) cur.init(p);
    // The token's threads (warps q + 4 h) run the same iterations: keys agree on whether tile i exists at
    // their named barrier (an AND over the group, so a failed wait in one warp ends the loop for all), values
    // run n_fixed + 1; after a failed D1 wait a thread skips the work but still meets the token's barriers.
    for (int i = 0;; ++i) {
      float e2 = 0.f;
      int64_t slot = 0;
      bool valid = false;
      uint32_t more;
      TileSlot ts{-1, 0, 0};
      if constexpr (kSched) {
        ts = take(i);
        asm volatile("{\n .reg .pred p, r;\n setp.ge.s64 p, %1, 0;\n bar.red.and.pred r, %2, %3, p;\n selp.u32 %0, 1, 0, r;\n}"
                     : "=r"(more) : "l"(ts.row0), "r"(1 + q), "n"(32 * kParts) : "memory");
      } else {
        more = i < n_fixed;
      }
      if (more) {
        // ---- first epilogue of tile i: ||x||, codes (and, keys, the residual into E[i & 1]) ----
        if constexpr (kSched) {
          valid = ts.row0 + t < p.rows;
          slot = valid ? tile_row_slot(p, ts, t) : 0;
        } else {
          valid = row0_of(i) + t < p.rows;
          slot = valid ? cur.slot(p, t) : 0;
          cur.advance(p);
        }
        const int db = i % L::kND1;
        uint32_t r[CPT];
        // the tensor-memory loads are warp-wide: the whole warp loads or none of it does
        const bool have = __all_sync(0xffffffffu, ok && mbar_wait_sleep(bar.d1_full(db), (i / L::kND1) & 1));
        if (have) {
          tc::fence_after();
          const uint32_t d1 = tmem + lane_ofs + 128 * db + CPT * h;
#pragma unroll
          for (int c = 0; c < CPT / 32; ++c) tc::ld32(d1 + 32 * c, *reinterpret_cast<uint32_t (*)[32]>(r + 32 * c));
          tc::wait_ld();
          tc::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar.d1_empty(db));   // D1 may take the next tile's product
        } else {
          ok = false;
#pragma unroll
          for (int j = 0; j < CPT; ++j) r[j] = 0u;
        }
        // the token's threads meet here every tile, whether or not their loads ran
        const float n = part_norm<CPT, kParts>(r, xch + (i & 1) * (kParts * 128), h, t, q);
        if (have) {
          if (valid && h == 0) p.norm[slot] = n;
          // the codes of this thread's CPT columns at CB bits (B0 for the wider parts, else BITS)
          auto codes = [&](auto cbits) {
            constexpr int CB = decltype(cbits)::value;
            constexpr int WPT = CPT * CB / 32;           // code-stream words of this thread
            const float(&thc)[(1 << CB) - 1] = *reinterpret_cast<const float(*)[(1 << CB) - 1]>(&th[0]);
            uint32_t wcur[WPT];
#pragma unroll
            for (int w = 0; w < WPT; ++w) wcur[w] = 0u;
            if constexpr (QJL) {
              // keys: y = D1 / n, code, residual e = y - c[code] (0 for a zero vector), split into
              // bf16 parts and stored to E[i & 1] (free: the sketch product of tile i - 2 is done)
              const float(&cvc)[1 << CB] = *reinterpret_cast<const float(*)[1 << CB]>(&cvk[0]);
              const float inv = n > 0.f ? 1.0f / n : 0.f;
              const float nz = n > 0.f ? 1.f : 0.f;
              const uint32_t e_hi = tmem + lane_ofs + L::kE + 128 * (i & 1) + (CPT / 2) * h;
#pragma unroll
              for (int g = 0; g < CPT / 8; ++g) {
                float ev[8];
#pragma unroll
                for (int qq = 0; qq < 8; ++qq) {
                  const int j = 8 * g + qq;
                  const float y = __uint_as_float(r[j]) * inv;   // 0 for a zero vector
                  uint32_t m[CB];
                  code_masks<CB>(y, thc, m);
                  put_code<CB>(wcur, m, j);
                  ev[qq] = fmaf(-nz, centroid_of<CB>(m, cvc), y);
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
              rho[((i % 3) * kParts + h) * 128 + t] = e2;
              __syncwarp();
              if (lane == 0) {
                mbar_arrive(bar.e_full());
                if constexpr (L::kSplit) mbar_arrive(bar.rho_full(i % 3));   // for the sign warps
              }
            } else {
              // values need only the codes (FMA-pipe search on y = D1 / n, 0 for a zero vector)
              FmaSearch<CB> fs;
              fs.init(thc);
              const float inv = n > 0.f ? 1.0f / n : 0.f;
#pragma unroll
              for (int j = 0; j < CPT; ++j) {
                float f[CB];
                fs.flags(__uint_as_float(r[j]) * inv, f);
                put_code_f<CB>(wcur, f, j);
              }
              fix_words<CB>(wcur, CPT);
            }
            if (valid) {
              uint32_t *rec = p.records + slot * RW + woff;
              if (WPT % 2 == 0 && (woff & 1) == 0) {
#pragma unroll
                for (int w = 0; w < WPT; w += 2) st_global_v2(rec + w, wcur[w], wcur[(w + 1) % WPT]);
              } else {
#pragma unroll
                for (int w = 0; w < WPT; ++w) rec[w] = wcur[w];
              }
            }
          };
          if (wide) codes(std::integral_constant<int, B0>{});
          else codes(std::integral_constant<int, BITS>{});
        }
      }
      if constexpr (QJL && !L::kSplit) {
        if (i >= 1) {
          // ---- second epilogue of tile i - 1: sign words and ||e|| ----
          const int j = i - 1;
          static_assert(CPT == 32, "one sign word per epilogue thread");
          uint32_t sw[1] = {0u};
          if (__all_sync(0xffffffffu, ok && mbar_wait_sleep(bar.d2_full(), j & 1))) {
            tc::fence_after();
            uint32_t r[CPT];
#pragma unroll
            for (int c = 0; c < CPT / 32; ++c)
              tc::ld32(tmem + lane_ofs + L::kD2 + CPT * h + 32 * c, *reinterpret_cast<uint32_t (*)[32]>(r + 32 * c));
            tc::wait_ld();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.d2_empty());
            sw[0] = sign_word<0>(r);
          } else {
            ok = false;
          }
          // the token's barrier (warps q + 4 h): every part's sum of e^2 for tile j is visible
          asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "n"(32 * kParts) : "memory");
          if (ok && vprev) {
            float e2s = 0.f;
#pragma unroll
            for (int k = 0; k < kParts; ++k) e2s += rho[((j % 3) * kParts + k) * 128 + t];
            if (e2s == 0.f) sw[0] = ~0u;   // a zero residual: every sign +1
            p.records[slot_prev * RW + IW + h] = sw[0];
            if (h == 0) p.rnorm[slot_prev] = sqrtf(e2s);
          }
        }
        slot_prev = slot;
        vprev = valid;
      }
      if (!more) break;
    }
  }

  // ---- tear-down ----
  tc::fence_before();
  __syncthreads();
  if (warp == 0) tc::dealloc(tmem, L::kTmemCols);
  // every ticket of this CTA was drawn before the barrier above; the last CTA to finish zeroes the counter
  // for the next launch on the stream
  if (p.tiles && tid == 0) {
    __threadfence();
    if (atomicAdd(p.tiles + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.tiles, 0u);
      atomicExch(p.tiles + 1, 0u);
    }
  }
}

// The x rows as a 2-D tensor map: 128 16-bit elements per row, `rows` rows of 256 bytes; a
// box of 64 elements x 128 rows with 128-byte swizzle is one K block of an A tile. Rows past the
// end read 0.
bool make_x_map(CUtensorMap *map, const QuantParams &p, bool f16) {
  static PFN_cuTensorMapEncodeTiled encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess || !fn)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(fn);
  }
  const cuuint64_t dims[2] = {(cuuint64_t)kTD, (cuuint64_t)p.rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kTD * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kTT};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                const_cast<void *>(p.x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool QJL, int BITS, bool F16, bool MIXED = false>
cudaError_t launch_tc(const QuantParams &p, cudaStream_t st) {
  CUtensorMap xmap;
  if (p.rows >= (int64_t)1 << 31 || !make_x_map(&xmap, p, F16)) return cudaErrorNotSupported;
  auto kern = quantize_tc_kernel<QJL, BITS, F16, MIXED>;
  using L = Ws<QJL, epi_split<QJL, BITS, MIXED>()>;
  constexpr size_t smem = L::kBytes;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (p.rows + kTT - 1) / kTT;
  const int64_t slots = (int64_t)device_sm_count();
  const int grid = (int)(tiles < slots ? tiles : slots);
  QuantParams q = p;
  q.tiles = QJL && tiles > grid ? tile_counters(st) : nullptr;   // keys only; one tile per CTA needs no schedule
  return launch_after(kern, dim3(grid), dim3(L::kThreads), smem, st, q, xmap);
}

template <bool F16>
cudaError_t launch_tc_t(const QuantParams &p, int bits, bool qjl, cudaStream_t st) {
  if (p.n_hi == 64) {   // mixed rate: columns [0, 64) one bit wider
    switch (bits) {
      case 1: return qjl ? launch_tc<true, 1, F16, true>(p, st) : launch_tc<false, 1, F16, true>(p, st);
      case 2: return qjl ? launch_tc<true, 2, F16, true>(p, st) : launch_tc<false, 2, F16, true>(p, st);
      case 3: return qjl ? launch_tc<true, 3, F16, true>(p, st) : launch_tc<false, 3, F16, true>(p, st);
      default: return cudaErrorNotSupported;
    }
  }
  if (p.n_hi != 0) return cudaErrorNotSupported;
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
