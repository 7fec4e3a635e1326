// Query preparation and the attention-logit scan on the packed key cache.
//
// Estimator (usedby.ai, "TurboQuant: Compresion de KV Cache a 3 bits y
// aceleracion de inferencia en H100", "El Pitch": logits on compressed keys;
// winningdata.io, "TurboQuant: Google comprime KV cache para 3 bits sem perder
// acuracia", "2. QJL Residual": the 1-bit sketch of the residual corrects the
// inner-product bias):
//   l_t = n_t ( <Pi q, c[code_t]> + rho_t sqrt(pi/2)/d <S q, 2 sign_t - 1> ).
//
// Both inner products are sums over small groups of coordinates, so each CTA
// turns its queries into lookup tables in shared memory once and then reads
// one table entry per group and key:
//   index tables: one per group of g = 8/bits coordinates (2 for 3 bits); the
//     entry for a group key (the g codes, as they sit in the code stream) is
//     sum_c (Pi q)_c * c[code_c];
//   sign tables: one per byte of the sign field; the entry for a byte is
//     sqrt(pi/2)/d * sum_c (S q)_c * (+1 or -1).
// A key then costs d/g + d/8 table reads and adds per query instead of 2d
// multiply-adds on unpacked values.
#include "common.cuh"

namespace tq {

namespace {

constexpr int kLThreads = 256;

// Pi q and S q for every query head: block (row, 32-output chunk); each warp
// produces 8 outputs, each lane holding 4 consecutive q values and reading the
// matching 4 matrix entries of a row with one vector load, so a warp's 8 rows
// are in flight together.
constexpr int kQpOut = 32;   // outputs per block
__global__ void __launch_bounds__(128) qprep_kernel(const float *__restrict__ q, int d, const float *__restrict__ Pi,
                                                    const float *__restrict__ S, float *__restrict__ qrot,
                                                    float *__restrict__ qsk, uint32_t *status) {
  const int row = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();                // launched as a dependent of the previous work: it must be finished first
  pdl_launch_dependents();   // the scan may start staging keys now; it waits for this grid before reading
  if (row == 0 && chunk == 0 && tid == 0) *status = 0u;   // this call's kernels report into a clean word
  const float *qr = q + (size_t)row * d;
  // lane covers k in [4 lane, 4 lane + 4) and, for d > 128, [128 + 4 lane, ...)
  float4 qv[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = 128 * h + 4 * lane;
    qv[h] = make_float4(k < d ? qr[k] : 0.f, k + 1 < d ? qr[k + 1] : 0.f, k + 2 < d ? qr[k + 2] : 0.f,
                        k + 3 < d ? qr[k + 3] : 0.f);
  }
  const bool vec = (d & 3) == 0 && ((reinterpret_cast<uintptr_t>(Pi) | reinterpret_cast<uintptr_t>(S)) & 15) == 0;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int o = chunk * kQpOut + warp * 8 + j;   // output index in [0, 2d)
    float s = 0.f;
    if (o < 2 * d) {
      const float *mrow = (o < d ? Pi : S) + (size_t)(o < d ? o : o - d) * d;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = 128 * h + 4 * lane;
        if (vec && k + 3 < d) {
          const float4 m = __ldg(reinterpret_cast<const float4 *>(mrow + k));
          s = fmaf(m.x, qv[h].x, fmaf(m.y, qv[h].y, fmaf(m.z, qv[h].z, fmaf(m.w, qv[h].w, s))));
        } else {
          for (int c = 0; c < 4; ++c)
            if (k + c < d) s = fmaf(__ldg(mrow + k + c), (&qv[h].x)[c], s);
        }
      }
    }
    acc[j] = s;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = warp_sum(acc[j]);
  if (lane < 8) {
    float v = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) if (j == lane) v = acc[j];
    const int o = chunk * kQpOut + warp * 8 + lane;
    if (o < 2 * d) (o < d ? qrot : qsk)[(size_t)row * d + (o < d ? o : o - d)] = v;
  }
}

template <int BITS>
struct Keys {
  static constexpr int G = BITS == 1 ? 8 : BITS == 2 ? 4 : 2;   // coordinates per index key
  static constexpr int KB = G * BITS;                           // key width in bits
  static constexpr int E = 1 << KB;                             // entries per index table
};

template <int BITS>
__global__ void __launch_bounds__(kLThreads) logits_kernel(const LogitsParams p) {
  using K = Keys<BITS>;
  constexpr int L = 1 << BITS;
  extern __shared__ __align__(16) float tab[];
  __shared__ float cbs[16];
  const int tid = threadIdx.x;
  const int qb = blockIdx.y % p.qblocks;
  const int sk = blockIdx.y / p.qblocks;            // sequence * n_kv_heads + kv head
  const int seq = sk / p.n_kv_heads, kvh = sk - seq * p.n_kv_heads;
  const int h0 = kvh * p.group + qb * p.q_per_cta;
  const int nq = min(p.q_per_cta, p.group - qb * p.q_per_cta);
  const int d = p.d, nk = d / K::G, ns = d / 8;
  const int per_q = nk * K::E + ns * 256;
  const float kappa = 1.2533141373155003f / (float)d;   // sqrt(pi/2) / d

  if (tid < L) cbs[tid] = p.codebook[tid];
  __syncthreads();
  for (int qq = 0; qq < nq; ++qq) {
    const size_t qrow = ((size_t)seq * p.n_q_heads + h0 + qq) * d;
    const float *qr = p.qrot + qrow;
    const float *qs = p.qsk + qrow;
    float *ti = tab + (size_t)qq * per_q;
    for (int e = tid; e < nk * K::E; e += kLThreads) {
      const int j = e / K::E, key = e - j * K::E;
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < K::G; ++c) v = fmaf(__ldg(qr + j * K::G + c), cbs[(key >> (BITS * c)) & (L - 1)], v);
      ti[e] = v;
    }
    float *ts = ti + nk * K::E;
    for (int e = tid; e < ns * 256; e += kLThreads) {
      const int j = e >> 8, b = e & 255;
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float s = __ldg(qs + 8 * j + c);
        v += ((b >> c) & 1) ? s : -s;
      }
      ts[e] = kappa * v;
    }
  }
  __syncthreads();

  const int64_t t0 = (int64_t)blockIdx.x * p.chunk;
  const int64_t t1 = min(p.n_tokens, t0 + p.chunk);
  const int sw = (d + 31) / 32;
  for (int64_t t = t0 + tid; t < t1; t += kLThreads) {
    const size_t slot = (size_t)sk * p.capacity + t;
    const uint32_t *rec = p.records + slot * p.rec_words;
    const float n = __ldg(p.norm + slot), rho = __ldg(p.rnorm + slot);
    for (int qq = 0; qq < nq; ++qq) {
      const float *ti = tab + (size_t)qq * per_q;
      const float *ts = ti + nk * K::E;
      float ai = 0.f, as = 0.f;
      for (int j = 0; j < nk; ++j) ai += ti[j * K::E + stream_bits(rec, K::KB * j, K::KB, p.idx_words)];
      for (int j = 0; j < ns; ++j) as += ts[j * 256 + stream_bits(rec + p.idx_words, 8 * j, 8, sw)];
      p.logits[((size_t)seq * p.n_q_heads + h0 + qq) * p.n_tokens + t] = n * fmaf(rho, as, ai);
    }
  }
}

// Mixed-rate keys: the first n_hi coordinates carry BL + 1 code bits, the rest BL,
// codes back to back in the stream (n_hi a multiple of 32, so both groups start on a
// key boundary). The same estimator with one set of index tables per group: the
// high group's keys of Keys<BL + 1> at stream bits KB_h j (coordinates G_h j ...),
// the low group's keys of Keys<BL> at stream bits (BL + 1) n_hi + KB_l j
// (coordinates n_hi + G_l j ...), and the sign tables as above.
template <int BL>
__global__ void __launch_bounds__(kLThreads) logits_mixed_kernel(const LogitsParams p) {
  constexpr int BH = BL + 1;
  using KH = Keys<BH>;
  using KL = Keys<BL>;
  constexpr int LL = 1 << BL, LH = 1 << BH;
  extern __shared__ __align__(16) float tab[];
  __shared__ float cbl[16], cbh[16];
  const int tid = threadIdx.x;
  const int qb = blockIdx.y % p.qblocks;
  const int sk = blockIdx.y / p.qblocks;
  const int seq = sk / p.n_kv_heads, kvh = sk - seq * p.n_kv_heads;
  const int h0 = kvh * p.group + qb * p.q_per_cta;
  const int nq = min(p.q_per_cta, p.group - qb * p.q_per_cta);
  const int d = p.d, m = p.n_hi;
  const int nkh = m / KH::G, nkl = (d - m) / KL::G, ns = d / 8;
  const int lo_bit0 = BH * m;
  const int per_q = nkh * KH::E + nkl * KL::E + ns * 256;
  const float kappa = 1.2533141373155003f / (float)d;   // sqrt(pi/2) / d

  if (tid < LL) cbl[tid] = p.codebook[tid];
  if (tid < LH) cbh[tid] = p.codebook[LL + tid];
  __syncthreads();
  for (int qq = 0; qq < nq; ++qq) {
    const size_t qrow = ((size_t)seq * p.n_q_heads + h0 + qq) * d;
    const float *qr = p.qrot + qrow;
    const float *qs = p.qsk + qrow;
    float *th = tab + (size_t)qq * per_q;
    for (int e = tid; e < nkh * KH::E; e += kLThreads) {
      const int j = e / KH::E, key = e - j * KH::E;
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < KH::G; ++c) v = fmaf(__ldg(qr + j * KH::G + c), cbh[(key >> (BH * c)) & (LH - 1)], v);
      th[e] = v;
    }
    float *tl = th + nkh * KH::E;
    for (int e = tid; e < nkl * KL::E; e += kLThreads) {
      const int j = e / KL::E, key = e - j * KL::E;
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < KL::G; ++c) v = fmaf(__ldg(qr + m + j * KL::G + c), cbl[(key >> (BL * c)) & (LL - 1)], v);
      tl[e] = v;
    }
    float *ts = tl + nkl * KL::E;
    for (int e = tid; e < ns * 256; e += kLThreads) {
      const int j = e >> 8, b = e & 255;
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float sv = __ldg(qs + 8 * j + c);
        v += ((b >> c) & 1) ? sv : -sv;
      }
      ts[e] = kappa * v;
    }
  }
  __syncthreads();

  const int64_t t0 = (int64_t)blockIdx.x * p.chunk;
  const int64_t t1 = min(p.n_tokens, t0 + p.chunk);
  const int sw = (d + 31) / 32;
  for (int64_t t = t0 + tid; t < t1; t += kLThreads) {
    const size_t slot = (size_t)sk * p.capacity + t;
    const uint32_t *rec = p.records + slot * p.rec_words;
    const float n = __ldg(p.norm + slot), rho = __ldg(p.rnorm + slot);
    for (int qq = 0; qq < nq; ++qq) {
      const float *th = tab + (size_t)qq * per_q;
      const float *tl = th + nkh * KH::E;
      const float *ts = tl + nkl * KL::E;
      float ai = 0.f, as = 0.f;
      for (int j = 0; j < nkh; ++j) ai += th[j * KH::E + stream_bits(rec, KH::KB * j, KH::KB, p.idx_words)];
      for (int j = 0; j < nkl; ++j)
        ai += tl[j * KL::E + stream_bits(rec, lo_bit0 + KL::KB * j, KL::KB, p.idx_words)];
      for (int j = 0; j < ns; ++j) as += ts[j * 256 + stream_bits(rec + p.idx_words, 8 * j, 8, sw)];
      p.logits[((size_t)seq * p.n_q_heads + h0 + qq) * p.n_tokens + t] = n * fmaf(rho, as, ai);
    }
  }
}

template <int BL>
cudaError_t launch_lm(const LogitsParams &p, int n_seq, int n_chunks, size_t smem, cudaStream_t st) {
  auto kern = logits_mixed_kernel<BL>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_chunks, n_seq * p.n_kv_heads * p.qblocks);
  kern<<<grid, kLThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_l(const LogitsParams &p, int n_seq, int n_chunks, size_t smem, cudaStream_t st) {
  auto kern = logits_kernel<BITS>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_chunks, n_seq * p.n_kv_heads * p.qblocks);
  kern<<<grid, kLThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t logits_smem_per_query(int d, int bits, int n_hi) {
  auto tables = [](int coords, int b) {
    const int g = b == 1 ? 8 : b == 2 ? 4 : 2;
    return (size_t)(coords / g) * ((size_t)1 << (g * b));
  };
  return (tables(n_hi, bits + 1) + tables(d - n_hi, bits) + (size_t)(d / 8) * 256) * sizeof(float);
}

cudaError_t launch_qprep(const float *q, int rows, int d, const float *Pi, const float *S, float *qrot, float *qsk,
                         uint32_t *status, cudaStream_t st) {
  dim3 grid((2 * d + kQpOut - 1) / kQpOut, rows);
  return launch_after(qprep_kernel, grid, dim3(128), 0, st, q, d, Pi, S, qrot, qsk, status);
}

cudaError_t launch_logits(const LogitsParams &p, int bits, int n_seq, int n_chunks, size_t smem, cudaStream_t st) {
  if (p.n_hi > 0) {
    switch (bits) {
      case 1: return launch_lm<1>(p, n_seq, n_chunks, smem, st);
      case 2: return launch_lm<2>(p, n_seq, n_chunks, smem, st);
      default: return launch_lm<3>(p, n_seq, n_chunks, smem, st);
    }
  }
  switch (bits) {
    case 1: return launch_l<1>(p, n_seq, n_chunks, smem, st);
    case 2: return launch_l<2>(p, n_seq, n_chunks, smem, st);
    case 3: return launch_l<3>(p, n_seq, n_chunks, smem, st);
    default: return launch_l<4>(p, n_seq, n_chunks, smem, st);
  }
}

}  // namespace tq
