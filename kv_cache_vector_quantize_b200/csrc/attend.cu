// Softmax-weighted value accumulation on the packed value cache, split over
// token chunks, and the log-sum-exp merge of the chunks.
//
// zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5 bits per
// channel", paragraph 1: the cache holds keys and values; values are stored
// MSE-only (norm + codes). With p = softmax(scale * logits):
//   out = Pi^T sum_t p_t n_t c[code_t].
// The sum runs in the rotated domain, so the d x d rotation is undone once per
// query head (in the merge) instead of once per token.
//
// Chunk kernel: one CTA per (token chunk, sequence, KV head, query block).
// It finds the chunk maximum m and sum l of exp(scale*logit - m) for each of
// its query heads, keeps w_t = exp(scale*l_t - m) * n_t in shared memory, and
// accumulates acc_i = sum_t w_t c[code_ti] with one thread per coordinate
// (the codes of a token are read once and reused by every query head of the
// group). Merge kernel: M = max_c m_c, L = sum_c l_c e^{m_c - M},
// A = sum_c acc_c e^{m_c - M}, out = Pi^T A / L.
#include <cstdio>
#include <mutex>

#include <cuda.h>

#include "common.cuh"

namespace tq {

namespace {

constexpr int kAThreads = 256;
constexpr int kAMaxQ = 4;   // query heads per CTA (one 16-byte weight load per token)

__device__ __forceinline__ float block_reduce(float v, float *red, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = is_max ? warp_max(v) : warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

// Shared memory of the chunk kernel: the chunk's records, the weights w[t][4],
// the codebooks, a reduction scratch and the per-phase accumulators.
size_t chunk_smem(int d, int rw, int64_t chunk) {
  const int phases = kAThreads / (d / 4);
  return (size_t)chunk * rw * 4 + (size_t)chunk * 4 * 4 + (32 + 32) * 4 + (size_t)phases * 4 * d * 4;
}

// One CTA per (token chunk, sequence, KV head, query block of <= 4 heads).
// Softmax statistics of the chunk, then each thread owns 4 consecutive
// coordinates of one token phase: per token it reads the code bits of its 4
// coordinates once, looks up their centroids and updates 4 x (query heads)
// accumulators with one 16-byte weight load. Phases are summed in a fixed
// order (deterministic). MIXED: a mixed-rate cache, whose first n_hi coordinates
// carry BITS + 1 code bits (n_hi a multiple of 32, so a thread's 4 coordinates
// are all in one group).
template <int BITS, bool MIXED>
__global__ void __launch_bounds__(kAThreads) attend_chunk_kernel(const AttendParams p) {
  constexpr int L = 1 << BITS;
  extern __shared__ __align__(16) float sm[];
  const int d = p.d, rw = p.rec_words;
  uint32_t *rec_s = reinterpret_cast<uint32_t *>(sm);          // [chunk][rw]
  float4 *w_s = reinterpret_cast<float4 *>(sm + p.chunk * rw);  // [chunk] (one lane per query head)
  float *cbs = reinterpret_cast<float *>(w_s + p.chunk);         // [16] BITS codebook, [16] BITS + 1 codebook
  float *red = cbs + 32;                                         // [32]
  float *accs = red + 32;                                        // [phases][4][d]
  const int tid = threadIdx.x;
  const int qb = blockIdx.y % p.qblocks;
  const int sk = blockIdx.y / p.qblocks;
  const int seq = sk / p.n_kv_heads, kvh = sk - seq * p.n_kv_heads;
  const int h0 = kvh * p.group + qb * p.q_per_cta;
  const int nq = min(p.q_per_cta, p.group - qb * p.q_per_cta);
  const int c = blockIdx.x;
  const int64_t t0 = (int64_t)c * p.chunk;
  const int nt = (int)min((int64_t)p.chunk, p.n_tokens - t0);
  const size_t slot0 = (size_t)sk * p.capacity + t0;

  if (tid < L) cbs[tid] = p.codebook[tid];
  if (MIXED && tid < 2 * L) cbs[16 + tid] = p.codebook[L + tid];
  // the chunk's records (contiguous in the cache) into shared memory
  const uint32_t *src = p.records + slot0 * rw;
  for (int e = tid; e < nt * rw; e += kAThreads) rec_s[e] = __ldg(src + e);
  // softmax statistics per query head, weights w_t = exp(scale l_t - m) n_t
  for (int qq = 0; qq < 4; ++qq) {
    float *wq = reinterpret_cast<float *>(w_s) + qq;
    if (qq >= nq) {
      for (int t = tid; t < nt; t += kAThreads) wq[4 * t] = 0.f;
      continue;
    }
    const size_t hrow = (size_t)seq * p.n_q_heads + h0 + qq;
    const float *lg = p.logits + hrow * p.n_tokens + t0;
    float m = -INFINITY;
    for (int t = tid; t < nt; t += kAThreads) m = fmaxf(m, p.scale * lg[t]);
    m = block_reduce(m, red, true);
    float s = 0.f;
    for (int t = tid; t < nt; t += kAThreads) {
      const float e = expf(p.scale * lg[t] - m);
      s += e;
      wq[4 * t] = e * __ldg(p.norm + slot0 + t);
    }
    s = block_reduce(s, red, false);
    if (tid == 0) {
      float *part = p.partial + (hrow * p.n_chunks + c) * (size_t)(d + 2);
      part[0] = m;
      part[1] = s;
    }
  }
  __syncthreads();

  // accumulate: thread = (token phase, group of 4 coordinates)
  const int npt = d / 4, phases = kAThreads / npt;
  const int ph = tid / npt, i0 = 4 * (tid - ph * npt);
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) acc[a][qq] = 0.f;
  if (ph < phases) {
    // this thread's code width, first stream bit and codebook (compile-time unless MIXED)
    int B = BITS, bit0 = BITS * i0;
    const float *cbc = cbs;
    if constexpr (MIXED) {
      if (i0 < p.n_hi) {
        B = BITS + 1;
        bit0 = (BITS + 1) * i0;
        cbc = cbs + 16;
      } else {
        bit0 = (BITS + 1) * p.n_hi + BITS * (i0 - p.n_hi);
      }
    }
    const uint32_t msk = (1u << B) - 1u;
    const int wd = bit0 >> 5, sh = bit0 & 31;
    const bool two = sh + 4 * B > 32 && wd + 1 < rw;
    for (int t = ph; t < nt; t += phases) {
      const uint32_t *rec = rec_s + t * rw;
      const uint32_t lo = rec[wd], hi = two ? rec[wd + 1] : 0u;
      const uint32_t bits = __funnelshift_r(lo, hi, sh);      // codes of the 4 coordinates
      const float4 wt = w_s[t];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float cv = cbc[(bits >> (B * a)) & msk];
        acc[a][0] = fmaf(wt.x, cv, acc[a][0]);
        acc[a][1] = fmaf(wt.y, cv, acc[a][1]);
        acc[a][2] = fmaf(wt.z, cv, acc[a][2]);
        acc[a][3] = fmaf(wt.w, cv, acc[a][3]);
      }
    }
#pragma unroll
    for (int qq = 0; qq < 4; ++qq)
#pragma unroll
      for (int a = 0; a < 4; ++a) accs[(ph * 4 + qq) * d + i0 + a] = acc[a][qq];
  }
  __syncthreads();
  for (int e = tid; e < nq * d; e += kAThreads) {
    const int qq = e / d, ii = e - qq * d;
    float v = 0.f;
    for (int q2 = 0; q2 < phases; ++q2) v += accs[(q2 * 4 + qq) * d + ii];
    const size_t hrow = (size_t)seq * p.n_q_heads + h0 + qq;
    p.partial[(hrow * p.n_chunks + c) * (size_t)(d + 2) + 2 + ii] = v;
  }
}

// Merge of the chunks of one query head: scale factors e^{m_c - M} once, the
// chunk sums split over all threads with independent loads in flight, then
// out = Pi^T A / L, with Pi staged in shared memory when it fits. Launched as a
// programmatic dependent of the chunk grid: it stages Pi while that grid's last
// CTAs run and waits for the grid before reading any partial. With `merged`
// given it writes the merged partial (M, L, A) there instead (Pi unused): the
// part of a token range that another merge combines with other ranges.
constexpr int kCThreads = 512;
__global__ void __launch_bounds__(kCThreads) attend_combine_kernel(const float *__restrict__ partial, int n_chunks,
                                                                   int d, const float *__restrict__ Pi,
                                                                   float *__restrict__ out, int pi_in_smem,
                                                                   float *__restrict__ merged) {
  extern __shared__ __align__(16) float cs[];          // [n_chunks] scale factors, then Pi (d x d) if staged
  __shared__ float a[kMaxD];
  __shared__ float part_sum[kCThreads];
  __shared__ float red[32];
  const int row = blockIdx.x, tid = threadIdx.x;
  const float *part = partial + (size_t)row * n_chunks * (d + 2);
  float *pis = cs + ((n_chunks + 3) & ~3);
  if (pi_in_smem) {
    const float4 *src = reinterpret_cast<const float4 *>(Pi);
    for (int e = tid; e < d * d / 4; e += kCThreads) reinterpret_cast<float4 *>(pis)[e] = __ldg(src + e);
  }
  pdl_wait();   // the partials come from the chunk grid (a programmatic primary, or plainly finished)
  float m = -INFINITY;
  for (int c = tid; c < n_chunks; c += kCThreads) m = fmaxf(m, part[(size_t)c * (d + 2)]);
  m = block_reduce(m, red, true);
  float l = 0.f;
  for (int c = tid; c < n_chunks; c += kCThreads) {
    // every part empty (merging token ranges that hold no tokens): nothing has weight
    const float f = m == -INFINITY ? 0.f : expf(part[(size_t)c * (d + 2)] - m);
    cs[c] = f;
    l = fmaf(part[(size_t)c * (d + 2) + 1], f, l);
  }
  l = block_reduce(l, red, false);   // also orders the cs[] and Pi writes before their reads
  // chunk sums: thread = (coordinate i, chunk phase)
  const int nsplit = kCThreads / d;
  const int i = tid % d, ph = tid / d;
  if (ph < nsplit) {
    float s[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) s[u] = 0.f;
    int c = ph;
    for (; c + 7 * nsplit < n_chunks; c += 8 * nsplit) {
#pragma unroll
      for (int u = 0; u < 8; ++u) s[u] = fmaf(part[(size_t)(c + u * nsplit) * (d + 2) + 2 + i], cs[c + u * nsplit], s[u]);
    }
    for (; c < n_chunks; c += nsplit) s[0] = fmaf(part[(size_t)c * (d + 2) + 2 + i], cs[c], s[0]);
    part_sum[tid] = ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
  }
  __syncthreads();
  if (tid < d) {
    float v = 0.f;
    for (int q = 0; q < nsplit; ++q) v += part_sum[q * d + tid];
    a[tid] = v;
    if (merged) merged[(size_t)row * (d + 2) + 2 + tid] = v;
  }
  if (merged) {
    if (tid == 0) {
      merged[(size_t)row * (d + 2)] = m;
      merged[(size_t)row * (d + 2) + 1] = l;
    }
    return;
  }
  __syncthreads();
  // out_j = sum_i Pi[i][j] a_i / L, the i range split over the threads of column j
  const float inv = l > 0.f ? 1.0f / l : 0.f;   // no weight anywhere: zeros
  const int j = tid % d, seg = tid / d, nseg = kCThreads / d;
  if (seg < nseg) {
    const int i0 = seg * ((d + nseg - 1) / nseg), i1 = min(d, i0 + (d + nseg - 1) / nseg);
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int ii = i0;
    if (pi_in_smem) {
      for (; ii + 4 <= i1; ii += 4) {
        s0 = fmaf(pis[ii * d + j], a[ii], s0);
        s1 = fmaf(pis[(ii + 1) * d + j], a[ii + 1], s1);
        s2 = fmaf(pis[(ii + 2) * d + j], a[ii + 2], s2);
        s3 = fmaf(pis[(ii + 3) * d + j], a[ii + 3], s3);
      }
      for (; ii < i1; ++ii) s0 = fmaf(pis[ii * d + j], a[ii], s0);
    } else {
      for (; ii + 4 <= i1; ii += 4) {
        s0 = fmaf(__ldg(Pi + (size_t)ii * d + j), a[ii], s0);
        s1 = fmaf(__ldg(Pi + (size_t)(ii + 1) * d + j), a[ii + 1], s1);
        s2 = fmaf(__ldg(Pi + (size_t)(ii + 2) * d + j), a[ii + 2], s2);
        s3 = fmaf(__ldg(Pi + (size_t)(ii + 3) * d + j), a[ii + 3], s3);
      }
      for (; ii < i1; ++ii) s0 = fmaf(__ldg(Pi + (size_t)ii * d + j), a[ii], s0);
    }
    part_sum[tid] = (s0 + s1) + (s2 + s3);
  }
  __syncthreads();
  if (tid < d) {
    float v = 0.f;
    for (int q = 0; q < nseg; ++q) v += part_sum[q * d + tid];
    out[(size_t)row * d + tid] = v * inv;
  }
}

template <int BITS, bool MIXED>
cudaError_t launch_a(const AttendParams &p, int n_seq, size_t smem, cudaStream_t st) {
  auto kern = attend_chunk_kernel<BITS, MIXED>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_chunks, n_seq * p.n_kv_heads * p.qblocks);
  kern<<<grid, kAThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend(const AttendParams &p, int bits, int n_seq, size_t smem, cudaStream_t st) {
  if (p.n_hi > 0) {
    switch (bits) {
      case 1: return launch_a<1, true>(p, n_seq, smem, st);
      case 2: return launch_a<2, true>(p, n_seq, smem, st);
      default: return launch_a<3, true>(p, n_seq, smem, st);
    }
  }
  switch (bits) {
    case 1: return launch_a<1, false>(p, n_seq, smem, st);
    case 2: return launch_a<2, false>(p, n_seq, smem, st);
    case 3: return launch_a<3, false>(p, n_seq, smem, st);
    default: return launch_a<4, false>(p, n_seq, smem, st);
  }
}

cudaError_t launch_combine(const float *partial, int rows, int n_chunks, int d, const float *Pi, float *out,
                           cudaStream_t st, float *merged) {
  const size_t cs_bytes = (size_t)((n_chunks + 3) & ~3) * sizeof(float);
  const size_t pi_bytes = (size_t)d * d * sizeof(float);
  const int pi_in_smem = (!merged && cs_bytes + pi_bytes <= 160 * 1024 && (reinterpret_cast<uintptr_t>(Pi) & 15) == 0 &&
                          (d * d) % 4 == 0) ? 1 : 0;
  const size_t smem = cs_bytes + (pi_in_smem ? pi_bytes : 0);
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(attend_combine_kernel), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(kCThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attend_combine_kernel, partial, n_chunks, d, Pi, out, pi_in_smem, merged);
}

size_t attend_chunk_smem(int d, int rec_words, int64_t chunk) { return chunk_smem(d, rec_words, chunk); }

namespace {
__global__ void empty_partial_kernel(float *partial, int rows, int d) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)rows * (d + 2)) return;
  partial[e] = (e % (d + 2)) == 0 ? -INFINITY : 0.f;
}
}  // namespace

// The partial of a token range without tokens: (M, L, A) = (-inf, 0, 0) per row.
cudaError_t launch_empty_partial(float *partial, int rows, int d, cudaStream_t st) {
  const int64_t n = (int64_t)rows * (d + 2);
  empty_partial_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(partial, rows, d);
  return cudaGetLastError();
}

}  // namespace tq

// ---------------------------------------------------------------------------
// tq_attend_v_noalloc: softmax.V whose scratch lives in a fixed device array of
// this library, for callers that cannot allocate device memory (see tq.h).
// ---------------------------------------------------------------------------

namespace tq {

namespace {

// Scratch for the chunk partials and the status word of tq_attend_v. Every
// call on a device uses this one array; it is not cleared between calls (the
// status word is reset by every call and every partial a call reads was
// written by that same call).
static __device__ __align__(256) unsigned char g_attend_scratch[TQ_ATTEND_NOALLOC_SCRATCH_BYTES];

// The array's device address differs per CUDA context (a context created after
// cudaDeviceReset loads the module again), so it is cached per (device, context
// id). Context ids are unique for the life of the process, unlike context handles,
// which a new context may reuse.
constexpr int kScratchMaxDevices = 64;
struct ScratchEntry {
  unsigned long long ctx_id;
  void *addr;
};
ScratchEntry g_scratch[kScratchMaxDevices] = {};
std::mutex g_scratch_mutex;

typedef CUresult (*PfnCtxGetCurrent)(CUcontext *);
typedef CUresult (*PfnCtxGetId)(CUcontext, unsigned long long *);

// Id of the current context (after a runtime call made the primary context current).
tq_status current_context_id(unsigned long long *id) {
  static PfnCtxGetCurrent get_current = nullptr;
  static PfnCtxGetId get_id = nullptr;
  if (!get_current || !get_id) {
    void *f1 = nullptr, *f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess || !f1 ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess || !f2)
      return report_error(TQ_ERR_CUDA, "tq_attend_v_noalloc: driver entry points cuCtxGetCurrent/cuCtxGetId not found");
    get_current = reinterpret_cast<PfnCtxGetCurrent>(f1);
    get_id = reinterpret_cast<PfnCtxGetId>(f2);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS)
    return report_error(TQ_ERR_CUDA, "tq_attend_v_noalloc: cuCtxGetCurrent failed");
  if (ctx == nullptr) {
    // no context on this thread yet: since CUDA 12, cudaSetDevice initialises the device's
    // primary context and makes it current (it allocates nothing)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess ||
        get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
      return report_error(TQ_ERR_CUDA, "tq_attend_v_noalloc: no current CUDA context");
  }
  if (get_id(ctx, id) != CUDA_SUCCESS) return report_error(TQ_ERR_CUDA, "tq_attend_v_noalloc: cuCtxGetId failed");
  return TQ_OK;
}

// Device address of g_attend_scratch in the current context. Looked up with the
// device current, once per (device, context); the host-side symbol is only a
// stand-in and must never reach a kernel.
tq_status scratch_address(void **out, const char *what) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof msg, "%s: cudaGetDevice: %s", what, cudaGetErrorString(e));
    return report_error(TQ_ERR_CUDA, msg);
  }
  if (dev < 0 || dev >= kScratchMaxDevices) return report_error(TQ_ERR_UNSUPPORTED, "tq_attend_v_noalloc: device index too large");
  unsigned long long id = 0;
  tq_status s = current_context_id(&id);
  if (s != TQ_OK) return s;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch[dev].addr == nullptr || g_scratch[dev].ctx_id != id) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attend_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[256];
      snprintf(msg, sizeof msg, "%s: cudaGetSymbolAddress: %s", what, cudaGetErrorString(e));
      return report_error(TQ_ERR_CUDA, msg);
    }
    g_scratch[dev] = ScratchEntry{id, p};
  }
  *out = g_scratch[dev].addr;
  return TQ_OK;
}

}  // namespace

}  // namespace tq

extern "C" tq_status tq_attend_v_noalloc(const tq_cache *v, const float *logits, float scale, int32_t n_q_heads,
                                         int64_t n_tokens, const float *Pi, const float *codebook, float *out,
                                         tq_stream stream) {
  tq::clear_error();
  // the same argument checks as tq_attend_v first, so a bad argument gets the same status
  tq_status s = tq::check_attend_args(v, logits, scale, n_q_heads, n_tokens, Pi, codebook, out,
                                      "tq_attend_v_noalloc");
  if (s != TQ_OK) return s;
  const size_t need = tq_attend_workspace_size(v, n_q_heads, n_tokens);
  if (need > TQ_ATTEND_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "tq_attend_v_noalloc: this shape needs %zu bytes of scratch but the built-in array holds %zu; "
             "use tq_attend_v with a caller workspace", need, (size_t)TQ_ATTEND_NOALLOC_SCRATCH_BYTES);
    return tq::report_error(TQ_ERR_WORKSPACE, msg);
  }
  void *scratch = nullptr;
  s = tq::scratch_address(&scratch, "tq_attend_v_noalloc");
  if (s != TQ_OK) return s;
  return tq_attend_v(v, logits, scale, n_q_heads, n_tokens, Pi, codebook, out, scratch,
                     TQ_ATTEND_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" tq_status tq_attend_v_noalloc_status(tq_stream stream) {
  tq::clear_error();
  void *scratch = nullptr;
  tq_status s = tq::scratch_address(&scratch, "tq_attend_v_noalloc_status");
  if (s != TQ_OK) return s;
  return tq_workspace_status(scratch, stream);
}
