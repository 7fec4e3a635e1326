// Grouped-query lookup tables shared by the grouped-query logit scan (logits_gqa.cu) and the
// fused grouped-query decode step (decode_gqa.cu): record geometry of d = 128 keys with 1 or 2
// code bits, and the float16 table sums (see logits_gqa.cu for the table format).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace tq {
namespace gqa {

constexpr int kGD = 128;                        // head dimension
constexpr uint32_t kGHalf = 65536;              // bytes of one table half in shared memory

template <int BETA>
struct GKeys {
  static constexpr int IW = BETA * kGD / 32;     // code-stream words
  static constexpr int RW = IW + kGD / 32;       // record words
  static constexpr int NI = BETA == 1 ? 16 : 32; // index bytes per record
  static constexpr int G = 8 / BETA;             // coordinates per index byte
};

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32u(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ __half2 u2h2(uint32_t v) { return *reinterpret_cast<const __half2 *>(&v); }

// Permute N words by XOR of their index with c (N a power of two, c < N).
template <int N>
__device__ __forceinline__ void xor_perm(uint32_t (&w)[N], int c) {
#pragma unroll
  for (int bit = 1; bit < N; bit <<= 1) {
    uint32_t t[N];
    const bool take = (c & bit) != 0;
#pragma unroll
    for (int j = 0; j < N; ++j) t[j] = take ? w[j ^ bit] : w[j];
#pragma unroll
    for (int j = 0; j < N; ++j) w[j] = t[j];
  }
}

// NSTEP table reads at base offset OFF (0: index half, kGHalf: sign half),
// summed per head into acc (float32), with float16 partial sums over 16 reads.
template <int QH, int NSTEP, uint32_t OFF, int NW>
__device__ __forceinline__ void gqa_sum(const uint32_t (&w)[NW], const uint32_t (&sel)[4], const uint32_t (&x)[16],
                                        float (&acc)[QH]) {
  constexpr int NP = QH / 2;   // head pairs
  __half2 part[2][NP];
#pragma unroll
  for (int st = 0; st < NSTEP; ++st) {
    if ((st & 15) == 0) {
#pragma unroll
      for (int k = 0; k < NP; ++k) part[0][k] = part[1][k] = __float2half2_rn(0.f);
    }
    const uint32_t addr = __byte_perm(w[st >> 2], x[st >> 1], sel[st & 3]) + OFF;
    if constexpr (QH == 4) {
      const uint2 v = lds64(addr);
      part[st & 1][0] = __hadd2(part[st & 1][0], u2h2(v.x));
      part[st & 1][1] = __hadd2(part[st & 1][1], u2h2(v.y));
    } else {
      part[st & 1][0] = __hadd2(part[st & 1][0], u2h2(lds32u(addr)));
    }
    if ((st & 15) == 15 || st == NSTEP - 1) {
#pragma unroll
      for (int k = 0; k < NP; ++k) {
        const float2 a = __half22float2(part[0][k]), b = __half22float2(part[1][k]);
        acc[2 * k] += a.x + b.x;
        acc[2 * k + 1] += a.y + b.y;
      }
    }
  }
}

}  // namespace gqa
}  // namespace tq
