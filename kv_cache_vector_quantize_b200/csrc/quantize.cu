// Quantize-append kernel and the sketch-rotation product.
//
// TurboQuant encoder (zubnet.ai news, "Google's TurboQuant quantizes LLM KV
// cache to 3.5 bits per channel", paragraph 2; winningdata.io, "TurboQuant:
// Google comprime KV cache para 3 bits sem perder acuracia", "Como o TurboQuant
// funciona"): per vector x, n = ||x||, y = Pi x / n, code_i = #{j : y_i > t_j}
// with t_j the midpoints of the codebook, and for keys the residual
// e = y - c[code] (rotated domain), rho = ||e||, sign bits of (S Pi^T) e.
//
// Design: a persistent CTA of 8 warps owns a tile of 64 tokens, 8 per warp.
// Both d x d projections run as FP32 register-blocked products from shared
// memory (each lane owns columns lane + 32 m of 8 tokens), so every output
// column set of a warp is 32 consecutive coordinates: the code stream words
// come out of one warp reduction (redux.or) per word and the sign words out of
// one ballot, with no shared-memory transposition. The token rows of a warp
// are private to it, so after the one-time load of Pi and S Pi^T the tile loop
// needs no block barrier (d <= 128). For d > 128 the matrices are streamed in
// 32-column chunks between block barriers.
#include "common.cuh"

namespace tq {

namespace {

constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / 32;
constexpr int kQTpw = 8;                    // tokens per warp
constexpr int kQTile = kQWarps * kQTpw;     // 64 tokens per tile
constexpr int kMaxRecWords = kMaxBits * (kMaxD / 32) + kMaxD / 32;

template <int DP>
struct QLayout {
  static constexpr bool kResident = DP <= 128;
  static constexpr int KC = kResident ? DP : 32;   // matrix columns per shared-memory chunk
  static constexpr int PS = KC + 1;                // padded row stride of a matrix chunk
  static constexpr int CPL = DP / 32;              // output columns per lane
  static constexpr int XS = DP + 4;                // row stride of the token tile
  static constexpr int kMatFloats = DP * PS;
};

template <int DP, bool QJL>
constexpr size_t quant_smem_bytes() {
  using Lay = QLayout<DP>;
  size_t f = (size_t)Lay::kMatFloats * ((QJL && Lay::kResident) ? 2 : 1)
           + (size_t)kQTile * Lay::XS + 64;
  return f * sizeof(float) + (size_t)kQTile * kMaxRecWords * sizeof(uint32_t);
}

// Copy columns [k0, k0 + KC) of a d x d row-major matrix into dst[j][kk]
// (row stride PS), zero outside d. Consecutive threads read consecutive k.
template <int DP>
__device__ __forceinline__ void load_matrix_chunk(float *dst, const float *__restrict__ src, int d, int k0) {
  using Lay = QLayout<DP>;
  for (int e = threadIdx.x; e < DP * Lay::KC; e += kQThreads) {
    const int j = e / Lay::KC, kk = e - j * Lay::KC, k = k0 + kk;
    dst[j * Lay::PS + kk] = (j < d && k < d) ? __ldg(src + (size_t)j * d + k) : 0.f;
  }
}

// acc[i][m] += sum_{kk < KC} X[row_i][k0 + kk] * Mat[lane + 32 m][kk]
template <int DP>
__device__ __forceinline__ void gemm_chunk(const float *mat, const float *xw, int k0, int lane,
                                           float (&acc)[kQTpw][QLayout<DP>::CPL]) {
  using Lay = QLayout<DP>;
#pragma unroll 1
  for (int kk = 0; kk < Lay::KC; kk += 4) {
    float4 xv[kQTpw];
#pragma unroll
    for (int i = 0; i < kQTpw; ++i) xv[i] = *reinterpret_cast<const float4 *>(xw + i * Lay::XS + k0 + kk);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float pv[Lay::CPL];
#pragma unroll
      for (int m = 0; m < Lay::CPL; ++m) pv[m] = mat[(lane + 32 * m) * Lay::PS + kk + u];
#pragma unroll
      for (int i = 0; i < kQTpw; ++i) {
        const float xs = u == 0 ? xv[i].x : u == 1 ? xv[i].y : u == 2 ? xv[i].z : xv[i].w;
#pragma unroll
        for (int m = 0; m < Lay::CPL; ++m) acc[i][m] = fmaf(xs, pv[m], acc[i][m]);
      }
    }
  }
}

template <int DP>
__device__ __forceinline__ void project(const float *__restrict__ gmat, float *mat, const float *xw, int d, int lane,
                                        float (&acc)[kQTpw][QLayout<DP>::CPL]) {
  using Lay = QLayout<DP>;
#pragma unroll
  for (int i = 0; i < kQTpw; ++i)
#pragma unroll
    for (int m = 0; m < Lay::CPL; ++m) acc[i][m] = 0.f;
  for (int k0 = 0; k0 < DP; k0 += Lay::KC) {
    if constexpr (!Lay::kResident) {
      __syncthreads();
      load_matrix_chunk<DP>(mat, gmat, d, k0);
      __syncthreads();
    }
    gemm_chunk<DP>(mat, xw, k0, lane, acc);
  }
}

// y = H (s * x) / sqrt(d) for the kQTpw rows of a warp (structured rotation, winningdata.io
// "1. PolarQuant": the rotation's cost per vector; a Hadamard product is O(d log d)). H is the
// Sylvester-Hadamard matrix in natural order, so log2(d) rounds of pairs (i, i + h), i & h = 0,
// become (a + b, a - b). Lane l holds coordinates l + 32 m: rounds h < 32 pair lanes (one
// shuffle), rounds h >= 32 pair registers m and m + h / 32. DP = d, a power of two.
template <int DP>
__device__ __forceinline__ void fwht_rows(const float *xw, const float *__restrict__ signs, int lane,
                                          float (&acc)[kQTpw][QLayout<DP>::CPL]) {
  using Lay = QLayout<DP>;
  constexpr int CPL = Lay::CPL;
  float sg[CPL];
#pragma unroll
  for (int m = 0; m < CPL; ++m) sg[m] = __ldg(signs + lane + 32 * m);
  const float scale = 1.0f / sqrtf((float)DP);
#pragma unroll
  for (int i = 0; i < kQTpw; ++i) {
    float v[CPL];
#pragma unroll
    for (int m = 0; m < CPL; ++m) v[m] = xw[i * Lay::XS + lane + 32 * m] * sg[m];
#pragma unroll
    for (int h = 1; h < 32 && h < DP; h <<= 1) {
      const bool hi = (lane & h) != 0;
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        const float o = __shfl_xor_sync(0xffffffffu, v[m], h);
        v[m] = hi ? o - v[m] : v[m] + o;
      }
    }
#pragma unroll
    for (int hm = 1; hm < CPL; hm <<= 1)
#pragma unroll
      for (int m = 0; m < CPL; ++m)
        if ((m & hm) == 0) {
          const float a = v[m], b = v[m + hm];
          v[m] = a + b;
          v[m + hm] = a - b;
        }
#pragma unroll
    for (int m = 0; m < CPL; ++m) acc[i][m] = v[m] * scale;
  }
}

// Blocks per SM: d > 128 streams the matrices in chunks between block barriers, so two CTAs per
// SM let one CTA's barrier waits overlap the other's products.
template <int DP>
constexpr int q_blocks_per_sm() { return DP > 128 ? 2 : 1; }

template <int DP, bool QJL, typename Tin, bool HAD = false>
__global__ void __launch_bounds__(kQThreads, q_blocks_per_sm<DP>()) quantize_kernel(const QuantParams p, const int bits) {
  using Lay = QLayout<DP>;
  constexpr int CPL = Lay::CPL;
  extern __shared__ __align__(16) float smem[];
  float *matP = smem;
  float *matM = (QJL && Lay::kResident) ? smem + Lay::kMatFloats : smem;
  float *xs = smem + Lay::kMatFloats * ((QJL && Lay::kResident) ? 2 : 1);
  // [16] centroids and [16] thresholds of the `bits` codebook, then the same of the
  // bits + 1 codebook of a mixed-rate cache (unused thresholds +huge)
  float *cb = xs + kQTile * Lay::XS;
  uint32_t *rs = reinterpret_cast<uint32_t *>(cb + 64);      // [kQTile][rec_words]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d, L = 1 << bits, rw = p.rec_words, iw = p.idx_words;
  const int LH = p.n_hi > 0 ? 2 * L : 0;                    // levels of the wider codebook
  const int mhi = p.n_hi / 32;                              // 32-column groups at bits + 1 code bits
  if (tid < L) cb[tid] = p.codebook[tid];
  if (tid < LH) cb[32 + tid] = p.codebook[L + tid];
  __syncthreads();
  if (tid < L - 1) cb[16 + tid] = 0.5f * (cb[tid] + cb[tid + 1]);
  if (tid < 15) cb[48 + tid] = tid < LH - 1 ? 0.5f * (cb[32 + tid] + cb[32 + tid + 1]) : 3.0e38f;
  if constexpr (Lay::kResident) {
    if constexpr (!HAD) load_matrix_chunk<DP>(matP, p.Pi, d, 0);
    if constexpr (QJL) load_matrix_chunk<DP>(matM, p.SPiT, d, 0);
  }
  __syncthreads();
  float th[15];
#pragma unroll
  for (int j = 0; j < 15; ++j) th[j] = j < L - 1 ? cb[16 + j] : 3.0e38f;

  float *xw = xs + warp * kQTpw * Lay::XS;                   // this warp's token rows
  uint32_t *rw_s = rs + warp * kQTpw * rw;
  const Tin *x = static_cast<const Tin *>(p.x);
  const int64_t n_tiles = (p.rows + kQTile - 1) / kQTile;

  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t row0 = tile * kQTile + warp * kQTpw;
    // ---- load this warp's rows, widened to float, zero padded ----
#pragma unroll 1
    for (int i = 0; i < kQTpw; ++i) {
      const int64_t row = row0 + i;
      for (int k = lane; k < DP; k += 32)
        xw[i * Lay::XS + k] = (row < p.rows && k < d) ? to_float(x[row * d + k]) : 0.f;
    }
    __syncwarp();
    float nrm[kQTpw], rho[kQTpw];
#pragma unroll
    for (int i = 0; i < kQTpw; ++i) {
      // sum of squares in double: no overflow or underflow for any finite float input
      double s = 0.0;
#pragma unroll
      for (int m = 0; m < CPL; ++m) { const double v = xw[i * Lay::XS + lane + 32 * m]; s = fma(v, v, s); }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      nrm[i] = (float)sqrt(s);
    }
    // ---- y = Pi x / n ----
    float acc[kQTpw][CPL];
    if constexpr (HAD) fwht_rows<DP>(xw, p.signs, lane, acc);
    else project<DP>(p.Pi, matP, xw, d, lane, acc);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < kQTpw; ++i) {
      const float inv = nrm[i] > 0.f ? 1.0f / nrm[i] : 0.f;
      float e2 = 0.f;
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        const int col = lane + 32 * m;
        const bool valid = col < d;
        const float y = acc[i][m] * inv;
        // group m (32 columns) is at bits + 1 code bits when m < mhi (warp-uniform)
        const bool ghi = m < mhi;
        const int gb = ghi ? bits + 1 : bits;
        const int gbase = ghi ? (bits + 1) * m : (bits + 1) * mhi + bits * (m - mhi);
        const float *gcb = ghi ? cb + 32 : cb;
        uint32_t code = 0;
        if (ghi) {
#pragma unroll
          for (int j = 0; j < 15; ++j) code += (y > cb[48 + j]) ? 1u : 0u;
        } else {
#pragma unroll
          for (int j = 0; j < 15; ++j) code += (y > th[j]) ? 1u : 0u;
        }
        if (!valid) code = 0;
        // code stream: the 32 columns of group m fill stream words [gbase, gbase + gb)
        const int off = gb * lane, ww = off >> 5, sh = off & 31;
        for (int w = 0; w < gb; ++w) {
          uint32_t v = 0;
          if (ww == w) v = code << sh;
          else if (ww + 1 == w && sh + gb > 32) v = code >> (32 - sh);
          const uint32_t word = __reduce_or_sync(0xffffffffu, v);
          if (lane == 0 && gbase + w < iw) rw_s[i * rw + gbase + w] = word;
        }
        if constexpr (QJL) {
          const float e = (valid && nrm[i] > 0.f) ? y - gcb[code] : 0.f;
          e2 = fmaf(e, e, e2);
          xw[i * Lay::XS + col] = e;    // residual replaces x (row private to this warp)
        }
      }
      rho[i] = QJL ? sqrtf(warp_sum(e2)) : 0.f;
    }
    if constexpr (QJL) {
      __syncwarp();
      // ---- sign bits of S Pi^T e ----
      project<DP>(p.SPiT, matM, xw, d, lane, acc);
#pragma unroll
      for (int i = 0; i < kQTpw; ++i)
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
          const uint32_t word = __ballot_sync(0xffffffffu, (lane + 32 * m < d) && acc[i][m] >= 0.f);
          if (lane == 0 && m < (d + 31) / 32) rw_s[i * rw + iw + m] = word;
        }
    }
    __syncwarp();
    // ---- store records and norms ----
    for (int e = lane; e < kQTpw * rw; e += 32) {
      const int i = e / rw, w = e - i * rw;
      const int64_t row = row0 + i;
      if (row < p.rows) {
        const int64_t sh = row / p.n_tokens, t = row - sh * p.n_tokens;
        p.records[(sh * p.capacity + p.pos + t) * rw + w] = rw_s[e];
      }
    }
    if (lane < kQTpw) {
      float nv = 0.f, rv = 0.f;
#pragma unroll
      for (int i = 0; i < kQTpw; ++i) if (i == lane) { nv = nrm[i]; rv = rho[i]; }
      const int64_t row = row0 + lane;
      if (row < p.rows) {
        const int64_t sh = row / p.n_tokens, t = row - sh * p.n_tokens;
        const int64_t slot = sh * p.capacity + p.pos + t;
        p.norm[slot] = nv;
        if constexpr (QJL) p.rnorm[slot] = rv;
      }
    }
    __syncwarp();
  }
}

template <int DP, bool QJL, typename Tin, bool HAD = false>
cudaError_t launch_q(const QuantParams &p, int bits, cudaStream_t st) {
  auto kern = quantize_kernel<DP, QJL, Tin, HAD>;
  constexpr size_t smem = quant_smem_bytes<DP, QJL>();
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (p.rows + kQTile - 1) / kQTile;
  const int64_t slots = (int64_t)device_sm_count() * q_blocks_per_sm<DP>();
  const int grid = (int)(tiles < slots ? tiles : slots);
  kern<<<grid, kQThreads, smem, st>>>(p, bits);
  return cudaGetLastError();
}

template <int DP, bool QJL, bool HAD = false>
cudaError_t launch_q_dtype(const QuantParams &p, int bits, tq_dtype dt, cudaStream_t st) {
  switch (dt) {
    case TQ_BF16: return launch_q<DP, QJL, __nv_bfloat16, HAD>(p, bits, st);
    case TQ_FP16: return launch_q<DP, QJL, __half, HAD>(p, bits, st);
    default: return launch_q<DP, QJL, float, HAD>(p, bits, st);
  }
}

template <int DP, bool HAD = false>
cudaError_t launch_q_dp(const QuantParams &p, int bits, bool qjl, tq_dtype dt, cudaStream_t st) {
  return qjl ? launch_q_dtype<DP, true, HAD>(p, bits, dt, st) : launch_q_dtype<DP, false, HAD>(p, bits, dt, st);
}

// SPiT[i][j] = sum_k S[i][k] Pi[j][k], accumulated in double.
__global__ void sketch_rotation_kernel(int d, const float *__restrict__ Pi, const float *__restrict__ S,
                                       float *__restrict__ out) {
  const int i = blockIdx.x, j = threadIdx.x;
  if (j >= d) return;
  double acc = 0.0;
  for (int k = 0; k < d; ++k) acc += (double)S[(size_t)i * d + k] * (double)Pi[(size_t)j * d + k];
  out[(size_t)i * d + j] = (float)acc;
}

}  // namespace

cudaError_t launch_quantize(const QuantParams &p, int bits, bool qjl, tq_dtype dtype, cudaStream_t st) {
  // bf16 / fp16 heads of 128 with 16-byte aligned rows and matrices take the tensor-core kernel (quantize_tc.cu)
  auto a16 = [](const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (p.d == 128 && (p.n_hi == 0 || (p.n_hi == 64 && bits <= 3)) && (dtype == TQ_BF16 || dtype == TQ_FP16) &&
      a16(p.x) && a16(p.Pi) && (!qjl || a16(p.SPiT))) {
    const cudaError_t e = launch_quantize_tc(p, bits, qjl, dtype == TQ_FP16, st);
    if (e != cudaErrorNotSupported) return e;   // else (no tensor map for these rows): the FP32 kernel below
  }
  if (p.d <= 32) return launch_q_dp<32>(p, bits, qjl, dtype, st);
  if (p.d <= 64) return launch_q_dp<64>(p, bits, qjl, dtype, st);
  if (p.d <= 128) return launch_q_dp<128>(p, bits, qjl, dtype, st);
  if (p.d <= 224) return launch_q_dp<224>(p, bits, qjl, dtype, st);   // d = 200: 23% fewer products than 256
  return launch_q_dp<256>(p, bits, qjl, dtype, st);
}

cudaError_t launch_quantize_hadamard(const QuantParams &p, int bits, bool qjl, tq_dtype dtype, cudaStream_t st) {
  switch (p.d) {
    case 32: return launch_q_dp<32, true>(p, bits, qjl, dtype, st);
    case 64: return launch_q_dp<64, true>(p, bits, qjl, dtype, st);
    case 128: return launch_q_dp<128, true>(p, bits, qjl, dtype, st);
    case 256: return launch_q_dp<256, true>(p, bits, qjl, dtype, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sketch_rotation(int d, const float *Pi, const float *S, float *SPiT, cudaStream_t st) {
  sketch_rotation_kernel<<<d, 256, 0, st>>>(d, Pi, S, SPiT);
  return cudaGetLastError();
}

}  // namespace tq
