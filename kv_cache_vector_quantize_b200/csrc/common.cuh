// Shared device helpers and launch parameter blocks for the TurboQuant kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq.h"

namespace tq {

constexpr int kMaxBits = 4;           // code bits per coordinate handled by the kernels
constexpr int kMaxD = 256;            // largest head dimension
constexpr size_t kWsHeader = 256;     // bytes reserved at the start of every workspace

// Status bits a kernel may set in the workspace status word.
enum : uint32_t {
  kDevBadShape = 1u << 0,   // a kernel met an argument its launch should have excluded
};

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_float(__half v) { return __half2float(v); }

// Two float32 values in one 64-bit register (the lower coordinate in the low half) and the
// packed two-lane float32 arithmetic of sm_100.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Bits [pos, pos + nbits) of a little-endian word stream (nbits <= 25), read
// through the read-only path. `words` is the number of valid words.
__device__ __forceinline__ uint32_t stream_bits(const uint32_t *__restrict__ s, int pos, int nbits, int words) {
  const int w = pos >> 5, sh = pos & 31;
  uint32_t lo = __ldg(s + w);
  uint32_t hi = (sh + nbits > 32 && w + 1 < words) ? __ldg(s + w + 1) : 0u;
  return __funnelshift_r(lo, hi, sh) & ((1u << nbits) - 1u);
}

// ---------------------------------------------------------------------------
// parameter blocks (plain structs passed by value to the kernels)
// ---------------------------------------------------------------------------

struct QuantParams {
  const void *x;            // [rows][d]
  uint32_t *records;        // cache records
  float *norm;
  float *rnorm;
  const float *Pi;          // [d][d]
  const float *SPiT;        // [d][d]
  const float *codebook;    // [2^bits]
  int64_t rows;             // n_seq * n_kv_heads * n_tokens
  int64_t n_tokens;
  int64_t capacity;
  int64_t pos;
  int d;
  int rec_words;
  int idx_words;
  int n_hi;                 // mixed rate: leading coordinates at bits + 1 code bits (0: integer rate)
  const float *signs;       // structured rotation Pi = H diag(signs) / sqrt(d) (then Pi is unused), or NULL
  uint32_t *tiles;          // tensor-core quantizer: [2] zeroed tile-schedule counters (NULL: a fixed tile order)
};

struct LogitsParams {
  const uint32_t *records;
  const float *norm;
  const float *rnorm;
  const float *qrot;        // [n_seq][n_q_heads][d]  Pi q
  const float *qsk;         // [n_seq][n_q_heads][d]  S q
  const float *codebook;
  float *logits;            // [n_seq][n_q_heads][n_tokens]
  uint32_t *status;
  int64_t n_tokens;
  int64_t capacity;
  int64_t chunk;            // tokens per CTA
  int d;
  int rec_words;
  int idx_words;
  int n_kv_heads;
  int n_q_heads;
  int group;                // n_q_heads / n_kv_heads
  int q_per_cta;            // query heads handled by one CTA
  int qblocks;              // ceil(group / q_per_cta)
  int n_hi;                 // mixed rate: leading coordinates at bits + 1 code bits (0: integer rate)
};

// Lookup tables of the grouped-query scan (logits_gqa.cu).
struct GqaParams {
  const float *q;           // [n_seq][n_q_heads][d]
  const float *Pi, *S;      // [d][d]
  const float *codebook;
  unsigned char *tables;    // units x 128 KB
  float *sigma;             // [n_seq][n_q_heads] table scale of each head
  uint32_t *status;
  int n_kv_heads, n_q_heads, group, qblocks;
};

struct AttendParams {
  const uint32_t *records;
  const float *norm;
  const float *logits;      // [n_seq][n_q_heads][n_tokens]
  const float *codebook;
  float *partial;           // [n_seq][n_q_heads][n_chunks][d + 2]
  uint32_t *status;
  int64_t n_tokens;
  int64_t capacity;
  int64_t chunk;
  int n_chunks;
  float scale;
  int d;
  int rec_words;
  int n_kv_heads;
  int n_q_heads;
  int group;
  int q_per_cta;
  int qblocks;
  int n_hi;                 // mixed rate: leading coordinates at bits + 1 code bits (0: integer rate)
  // failure-detection test hook (tq_debug_stall_consumers): > 0 makes the d = 128 softmax.V kernel's
  // consumers wait on a barrier that nothing completes, for this many tries, and its copy thread give up
  // on the stages they never release after as many; 0 in normal use
  uint32_t stall_tries;
};

// Tries of the stalled consumer wait the next tq_attend_v call's kernel is launched with (0: none).
uint32_t debug_stall_tries();

// launchers (defined in the .cu files)
cudaError_t launch_sketch_rotation(int d, const float *Pi, const float *S, float *SPiT, cudaStream_t st);
cudaError_t launch_quantize(const QuantParams &p, int bits, bool qjl, tq_dtype dtype, cudaStream_t st);
// The FP32-core quantizer with y = H (signs * x) / (sqrt(d) ||x||) by a fast Walsh-Hadamard transform
// (d a power of two, 32..256); keys still project the residual with the dense S Pi^T.
cudaError_t launch_quantize_hadamard(const QuantParams &p, int bits, bool qjl, tq_dtype dtype, cudaStream_t st);
cudaError_t launch_quantize_tc(const QuantParams &p, int bits, bool qjl, bool f16, cudaStream_t st);
cudaError_t launch_qprep(const float *q, int rows, int d, const float *Pi, const float *S,
                         float *qrot, float *qsk, uint32_t *status, cudaStream_t st);
cudaError_t launch_logits(const LogitsParams &p, int bits, int n_seq, int n_chunks, size_t smem, cudaStream_t st);
size_t logits_smem_per_query(int d, int bits, int n_hi = 0);
int logits_fast_stages(int bits, int q, size_t limit, int n_hi = 0);
cudaError_t launch_logits_fast(const LogitsParams &p, int bits, int n_seq, size_t limit, cudaStream_t st);
bool gqa_supported(int d, int bits, int group);
size_t gqa_table_bytes(int units);
cudaError_t launch_logits_gqa(const LogitsParams &p, const GqaParams &g, int bits, int n_seq, size_t limit,
                              cudaStream_t st);
cudaError_t launch_attend(const AttendParams &p, int bits, int n_seq, size_t smem, cudaStream_t st);
// Fused decode attention (decode_fused.cu): one query head per KV head, d = 128, 1- or 2-bit key
// codes; writes the chunk partials of the softmax.V merge.
struct DecodeFusedArgs {
  const uint32_t *krec;
  const float *knorm, *krnorm;
  const uint32_t *vrec;
  const float *vnorm;
  const float *qrot, *qsk;    // [n_seq][n_heads][128]
  const float *cbk, *cbv;
  float *partial;             // [n_seq][n_heads][n_chunks][130]
  uint32_t *status;
  int64_t n_tokens, cap_k, cap_v, chunk;
  int n_seq, n_heads, n_chunks, kbits, vbits;
  float scale;
  size_t smem_limit;
};
bool decode_fused_supported(int d, int kbits, int vbits, int n_q_heads, int n_kv_heads, const void *krec,
                            const void *vrec, size_t limit);
cudaError_t launch_decode_fused(const DecodeFusedArgs &a, cudaStream_t st);
cudaError_t launch_status_or(uint32_t *dst, const uint32_t *a, const uint32_t *b, cudaStream_t st);
// Grouped-query tables alone (logits_gqa.cu): the four- or two-head float16 tables and scales of every unit.
cudaError_t launch_gqa_tables(const GqaParams &g, int bits, int qh, int units, cudaStream_t st);
// Fused decode for grouped queries (decode_gqa.cu): 2, 4 or 8 query heads per KV head, d = 128,
// 1- or 2-bit key codes, 1..3-bit value codes; consumes the grouped-query tables and writes the
// chunk partials of the softmax.V merge, bit-equal to tq_logits + tq_attend_v.
struct DecodeGqaArgs {
  const uint32_t *krec;
  const float *knorm, *krnorm;
  const uint32_t *vrec;
  const float *vnorm;
  const unsigned char *tables;
  const float *sigma;
  const float *cbv;
  float *partial;
  uint32_t *status;
  int64_t n_tokens, cap_k, cap_v, chunk;
  int n_seq, n_kv_heads, n_q_heads, qblocks, n_chunks, kbits, vbits;
  float scale;
  size_t smem_limit;
};
bool decode_gqa_supported(int d, int kbits, int vbits, int group, size_t limit);
cudaError_t launch_decode_gqa(const DecodeGqaArgs &a, cudaStream_t st);
// d = 128 softmax.V streamed by bulk copies (attend_fast.cu); p.chunk from attend_fast_chunk.
bool attend_fast_supported(int d, int bits, int q_per_cta, const void *records, int n_hi, int64_t capacity);
int64_t attend_fast_chunk(int64_t n_tokens, int units);
cudaError_t launch_attend_fast(const AttendParams &p, int bits, int n_seq, cudaStream_t st);
size_t attend_chunk_smem(int d, int rec_words, int64_t chunk);
cudaError_t launch_combine(const float *partial, int rows, int n_chunks, int d, const float *Pi,
                           float *out, cudaStream_t st, float *merged = nullptr);
cudaError_t launch_empty_partial(float *partial, int rows, int d, cudaStream_t st);
cudaError_t launch_nn_list_merge(const float *ps, const int64_t *pi, int n_parts, int n_q, int k, float *top_s,
                                 int64_t *top_i, cudaStream_t st);
// Nearest-neighbour search (nn_search.cu): running top-k of the key estimator over one packed
// database stream for a batch of queries.
struct NnArgs {
  const uint32_t *records;
  const float *norm, *rnorm;
  const float *q;             // [n_q][d]
  const float *Pi, *S, *codebook;
  float *top_s;               // [n_q][k]
  int64_t *top_i;             // [n_q][k]
  unsigned char *qimg;        // workspace: fp16 query rows
  float *sigma;               // workspace: per-query scale
  float *part_s;              // workspace: per-CTA top-k lists
  int *part_i;
  uint32_t *status;
  int64_t n_db;
  int n_q, d, bits, k, grid;
};
constexpr int kNnMaxGrid = 256;     // upper bound on the search grid (sizes the workspace)
constexpr int kNnMaxK = 16;
bool nn_supported(int d, int bits);
int nn_kp(int d);                   // padded K of a query row (fp16 elements)
cudaError_t launch_nn_search(const NnArgs &a, cudaStream_t st);
int device_sm_count();
// A pair of zeroed tile-schedule counters for a quantizer launch on `st` (tq_api.cu), or NULL.
uint32_t *tile_counters(cudaStream_t st);
// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t set_smem_once(const void *kernel, size_t bytes);
size_t device_smem_optin();
tq_status report_error(tq_status s, const char *msg);
void clear_error();   // empties this thread's tq_last_error() text
// The argument checks of tq_attend_v that do not involve the workspace (tq_api.cu).
tq_status check_attend_args(const tq_cache *v, const float *logits, float scale, int32_t n_q_heads,
                            int64_t n_tokens, const float *Pi, const float *codebook, const float *out,
                            const char *what, bool need_pi = true);

}  // namespace tq

// ---------------------------------------------------------------------------
// mbarrier / bulk-copy helpers (sm_90+ PTX) with bounded waits
// ---------------------------------------------------------------------------
namespace tq {

enum : uint32_t { kDevTimeout = 1u << 1 };   // an mbarrier wait gave up (status word bit)
// Programmatic dependent launch (sm_90 and later). A grid launched with the
// programmatic-serialization attribute may start while the previous grid in
// the stream still runs; it must call pdl_wait() before it reads that grid's
// results or writes anything that grid writes. Both are no-ops for a grid
// launched without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch a grid as a programmatic dependent of the work before it in the stream,
// so that its launch is processed while that work finishes. The kernel must
// call pdl_wait() before it reads or writes global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

constexpr uint32_t kSpinLimit = 1u << 24;    // try_wait attempts before a wait gives up

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Waits for the phase with the given parity to complete; false after `limit` tries.
__device__ __forceinline__ bool mbar_wait_n(uint32_t bar, uint32_t parity, uint32_t limit) {
  for (uint32_t it = 0; it < limit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// Waits for the phase with the given parity to complete; false after kSpinLimit tries.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) { return mbar_wait_n(bar, parity, kSpinLimit); }

// As mbar_wait, for waits that overlap other warps' work: each try may suspend the thread for up to
// kSleepHintNs (it resumes as soon as the phase completes), so a waiting warp takes few issue slots
// from the warps that share its scheduler. Bounded by kSleepLimit tries: at most about 2 s when every
// try sleeps its full hint, at least 2^21 tries when the hardware resumes earlier.
constexpr uint32_t kSleepHintNs = 1000;
constexpr uint32_t kSleepLimit = 1u << 21;
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity) {
  for (uint32_t it = 0; it < kSleepLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "n"(kSleepHintNs)
        : "memory");
    if (done) return true;
  }
  return false;
}

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_u128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

}  // namespace tq
