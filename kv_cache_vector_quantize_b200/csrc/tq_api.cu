// C ABI entry points (include/tq.h): host-side argument checks, workspace
// carving, launch configuration and status reporting. Every compute step runs
// in the kernels of quantize.cu, logits.cu and attend.cu.
#include <cuda.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "common.cuh"

namespace tq {
bool fit_lloyd_max(int d, int bits, float *out);

namespace {

thread_local char g_err[512] = "";
std::atomic<int> g_inject_count{0};
std::atomic<int> g_inject_status{0};
std::atomic<uint32_t> g_stall_tries{0};   // tq_debug_stall_consumers

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
int g_smem_optin[kMaxDevices] = {0};

tq_status fail(tq_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

tq_status cuda_fail(cudaError_t e, const char *where) {
  return fail(TQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// Host-side fault injection (tests): consume one armed failure, if any.
bool injected(tq_status *s) {
  int n = g_inject_count.load();
  while (n > 0) {
    if (g_inject_count.compare_exchange_weak(n, n - 1)) {
      *s = fail((tq_status)g_inject_status.load(), "injected failure (tq_debug_inject)");
      return true;
    }
  }
  return false;
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  return dev;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

tq_status check_cache(const tq_cache *c, const char *what) {
  if (!c) return fail(TQ_ERR_INVALID, "%s: cache descriptor is NULL", what);
  if (c->d < 8 || c->d > kMaxD || c->d % 8 != 0)
    return fail(TQ_ERR_UNSUPPORTED, "%s: d=%d (need 8..%d, multiple of 8)", what, c->d, kMaxD);
  if (c->idx_bits < 1 || c->idx_bits > kMaxBits)
    return fail(TQ_ERR_UNSUPPORTED, "%s: idx_bits=%d (need 1..%d)", what, c->idx_bits, kMaxBits);
  if (c->qjl != 0 && c->qjl != 1) return fail(TQ_ERR_INVALID, "%s: qjl=%d (need 0 or 1)", what, c->qjl);
  if (c->n_seq <= 0 || c->n_kv_heads <= 0 || c->capacity < 0)
    return fail(TQ_ERR_INVALID, "%s: n_seq=%d n_kv_heads=%d capacity=%lld", what, c->n_seq, c->n_kv_heads,
                (long long)c->capacity);
  if (c->n_hi != 0 && (c->n_hi < 0 || c->n_hi % 32 != 0 || c->n_hi >= c->d || c->idx_bits + 1 > kMaxBits))
    return fail(TQ_ERR_UNSUPPORTED, "%s: n_hi=%d (need 0, or a multiple of 32 below d=%d with idx_bits + 1 <= %d)",
                what, c->n_hi, c->d, kMaxBits);
  if (!c->records || !aligned(c->records, 16)) return fail(TQ_ERR_INVALID, "%s: records NULL or not 16-byte aligned", what);
  if (!c->norm || !aligned(c->norm, 4)) return fail(TQ_ERR_INVALID, "%s: norm NULL or misaligned", what);
  if (c->qjl && (!c->rnorm || !aligned(c->rnorm, 4))) return fail(TQ_ERR_INVALID, "%s: key cache needs rnorm", what);
  if (!c->qjl && c->rnorm) return fail(TQ_ERR_INVALID, "%s: value cache must have rnorm == NULL", what);
  return TQ_OK;
}

// Code-stream words: n_hi coordinates at bits + 1 code bits, the others at bits (mixed rate).
int idx_words_of(int d, int bits, int n_hi = 0) { return ((bits + 1) * n_hi + bits * (d - n_hi) + 31) / 32; }
int rec_words_of(int d, int bits, int qjl, int n_hi = 0) {
  return idx_words_of(d, bits, n_hi) + (qjl ? (d + 31) / 32 : 0);
}

struct LogitsPlan {
  int q_per_cta, qblocks, n_chunks;
  int64_t chunk;
  size_t smem;
};

LogitsPlan plan_logits(const tq_cache *k, int n_q_heads, int64_t n_tokens) {
  LogitsPlan pl{};
  const int group = n_q_heads / k->n_kv_heads;
  const size_t per_q = logits_smem_per_query(k->d, k->idx_bits, k->n_hi);
  const size_t budget = device_smem_optin() - 1024;
  int qpc = (int)(budget / per_q);
  if (qpc > group) qpc = group;
  pl.q_per_cta = qpc;
  pl.qblocks = qpc > 0 ? (group + qpc - 1) / qpc : 0;
  pl.smem = per_q * (size_t)(qpc > 0 ? qpc : 1);
  const int64_t units = (int64_t)k->n_seq * k->n_kv_heads * (pl.qblocks > 0 ? pl.qblocks : 1);
  const int64_t want = 4LL * device_sm_count();
  int64_t chunks = (want + units - 1) / units;
  const int64_t max_chunks = (n_tokens + 255) / 256;
  if (chunks > max_chunks) chunks = max_chunks;
  if (chunks < 1) chunks = 1;
  int64_t chunk = (n_tokens + chunks - 1) / chunks;
  chunk = (chunk + 127) / 128 * 128;
  if (chunk < 128) chunk = 128;
  pl.chunk = chunk;
  pl.n_chunks = (int)((n_tokens + chunk - 1) / chunk);
  return pl;
}

// Launch shape of the d = 128 table scan: one CTA per SM; two query heads per
// CTA when their tables leave room for at least three stages, else one.
struct FastPlan {
  bool use;
  int q_per_cta;
  size_t limit;
};

FastPlan plan_fast(const tq_cache *k, int n_q_heads) {
  FastPlan f{false, 0, 0};
  if (k->d != 128 || k->idx_bits > 3 || !k->qjl) return f;
  // mixed rate: the first 64 coordinates one bit wider, 2.5 or 3.5 bits per channel; the rows of
  // every (sequence, head) start on 16 bytes (a record is 40 or 56 bytes: an even capacity)
  if (k->n_hi != 0 && !(k->n_hi == 64 && k->idx_bits <= 2 && k->capacity % 2 == 0)) return f;
  const int group = n_q_heads / k->n_kv_heads;
  const size_t limit = device_smem_optin() - 1024;
  int q = 0;
  if (group >= 2 && logits_fast_stages(k->idx_bits, 2, limit, k->n_hi) >= 3) q = 2;
  else if (logits_fast_stages(k->idx_bits, 1, limit, k->n_hi) >= 2) q = 1;
  if (q == 0) return f;
  f = FastPlan{true, q, limit};
  return f;
}

constexpr int64_t kAttendChunk = 512;
constexpr int kAttendMaxQ = 4;

}  // namespace

uint32_t debug_stall_tries() { return g_stall_tries.load(); }

// Tile-schedule counters of the tensor-core key quantizer. Per device and CUDA context a pool of counter
// pairs (8 KB, allocated by the first call that needs it; the library's one allocation): one pair per
// stream (keyed by the stream's unique id, so launches that share a pair are stream-ordered) and a pair
// of its own for every launch recorded into a graph. A pair is zeroed by a stream-ordered memset when
// it is handed out, and the launch's last CTA zeroes it again. NULL (the kernel then takes its tiles in
// a fixed order) when the pool is used up, when a graph is being recorded before the pool exists, or when
// the context cannot be identified. A new context (after cudaDeviceReset) gets a new pool: the old
// pool's memory went with the old context.
namespace {
constexpr int kTilePairs = 1024;
struct TilePool {
  unsigned long long ctx_id = 0;
  uint32_t *base = nullptr;
  int used = 0;
  std::unordered_map<unsigned long long, int> by_stream;
};
TilePool g_tile_pool[kMaxDevices];
std::mutex g_tile_mu;

typedef CUresult (*PfnCtxGetCurrent)(CUcontext *);
typedef CUresult (*PfnCtxGetId)(CUcontext, unsigned long long *);

// Id of the calling thread's current context (unique for the life of the process, unlike the handle).
bool current_ctx_id(unsigned long long *id) {
  static PfnCtxGetCurrent get_current = nullptr;
  static PfnCtxGetId get_id = nullptr;
  if (!get_current || !get_id) {
    void *f1 = nullptr, *f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess || !f1 ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess || !f2) {
      cudaGetLastError();
      return false;
    }
    get_current = reinterpret_cast<PfnCtxGetCurrent>(f1);
    get_id = reinterpret_cast<PfnCtxGetId>(f2);
  }
  CUcontext ctx = nullptr;
  return get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr && get_id(ctx, id) == CUDA_SUCCESS;
}
}  // namespace

uint32_t *tile_counters(cudaStream_t st) {
  const int dev = current_device();
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  const bool capturing = cs != cudaStreamCaptureStatusNone;
  unsigned long long ctx_id = 0;
  if (!current_ctx_id(&ctx_id)) return nullptr;
  std::lock_guard<std::mutex> lock(g_tile_mu);
  TilePool &tp = g_tile_pool[dev];
  if (!tp.base || tp.ctx_id != ctx_id) {
    if (capturing) return nullptr;
    void *b = nullptr;
    if (cudaMalloc(&b, kTilePairs * 2 * sizeof(uint32_t)) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    tp = TilePool{};
    tp.ctx_id = ctx_id;
    tp.base = static_cast<uint32_t *>(b);
  }
  unsigned long long id = 0;
  if (!capturing) {
    if (cudaStreamGetId(st, &id) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    auto it = tp.by_stream.find(id);
    if (it != tp.by_stream.end()) return tp.base + 2 * it->second;
  }
  if (tp.used == kTilePairs) return nullptr;
  uint32_t *c = tp.base + 2 * tp.used;
  if (cudaMemsetAsync(c, 0, 2 * sizeof(uint32_t), st) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (!capturing) tp.by_stream.emplace(id, tp.used);
  ++tp.used;
  return c;
}

int device_sm_count() {
  const int dev = current_device();
  if (g_sm_count[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 1;
    g_sm_count[dev] = v;
  }
  return g_sm_count[dev];
}

size_t device_smem_optin() {
  const int dev = current_device();
  if (g_smem_optin[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || v <= 0) v = 232448;  // sm_100 opt-in limit
    g_smem_optin[dev] = v;
  }
  return (size_t)g_smem_optin[dev];
}

cudaError_t set_smem_once(const void *kernel, size_t bytes) {
  // (kernel, device) pairs already raised; a small open table is enough for the
  // few dozen kernel instantiations of this library.
  struct Entry { const void *k; int dev; size_t bytes; };
  static Entry table[512];
  static std::atomic<int> used{0};
  const int dev = current_device();
  const int n = used.load();
  for (int i = 0; i < n && i < 512; ++i)
    if (table[i].k == kernel && table[i].dev == dev && table[i].bytes >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  const int slot = used.fetch_add(1);
  if (slot < 512) table[slot] = Entry{kernel, dev, bytes};
  return cudaSuccess;
}

// Record a failure message for tq_last_error() from another translation unit.
tq_status report_error(tq_status s, const char *msg) { return fail(s, "%s", msg); }

}  // namespace tq

namespace tq {

// Bytes of the softmax.V chunk partials plus the header, or SIZE_MAX when the product overflows.
size_t attend_ws_bytes(const tq_cache *v, int32_t n_q_heads, int64_t n_tokens) {
  const int64_t n_chunks = (n_tokens + kAttendChunk - 1) / kAttendChunk;
  size_t b = sizeof(float);
  if (__builtin_mul_overflow(b, (size_t)v->n_seq, &b) || __builtin_mul_overflow(b, (size_t)n_q_heads, &b) ||
      __builtin_mul_overflow(b, (size_t)n_chunks, &b) || __builtin_mul_overflow(b, (size_t)(v->d + 2), &b) ||
      __builtin_add_overflow(b, kWsHeader, &b))
    return SIZE_MAX;
  return b;
}

void clear_error() { g_err[0] = 0; }

// Every check of tq_attend_v that does not involve the workspace, in order; shared with
// tq_attend_v_noalloc so that both report the same status for the same bad argument.
tq_status check_attend_args(const tq_cache *v, const float *logits, float scale, int32_t n_q_heads,
                            int64_t n_tokens, const float *Pi, const float *codebook, const float *out,
                            const char *what, bool need_pi) {
  tq_status s = check_cache(v, what);
  if (s != TQ_OK) return s;
  if (v->qjl) return fail(TQ_ERR_INVALID, "%s: the cache is a key cache (qjl == 1)", what);
  if (n_q_heads <= 0 || n_q_heads % v->n_kv_heads != 0)
    return fail(TQ_ERR_INVALID, "%s: n_q_heads=%d is not a positive multiple of n_kv_heads=%d", what, n_q_heads,
                v->n_kv_heads);
  if (n_tokens < 0 || n_tokens > v->capacity)
    return fail(TQ_ERR_CAPACITY, "%s: n_tokens=%lld outside [0, capacity=%lld]", what, (long long)n_tokens,
                (long long)v->capacity);
  if ((!logits && n_tokens > 0) || (need_pi && !Pi) || !codebook || !out)
    return fail(TQ_ERR_INVALID, "%s: NULL tensor argument", what);
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(TQ_ERR_INVALID, "%s: scale is not finite", what);
  const int group = n_q_heads / v->n_kv_heads;
  const int q_per_cta = group < kAttendMaxQ ? group : kAttendMaxQ;
  const int64_t grid_y = (int64_t)v->n_seq * v->n_kv_heads * ((group + q_per_cta - 1) / q_per_cta);
  if (grid_y > 65535 || (int64_t)v->n_seq * n_q_heads > 0x7fffffffLL)
    return fail(TQ_ERR_UNSUPPORTED, "%s: n_seq x n_kv_heads x query blocks = %lld exceeds 65535", what,
                (long long)grid_y);
  if (attend_ws_bytes(v, n_q_heads, n_tokens) == SIZE_MAX)
    return fail(TQ_ERR_UNSUPPORTED, "%s: the chunk partials of this shape overflow a size_t", what);
  return TQ_OK;
}

}  // namespace tq

using namespace tq;

extern "C" {

int32_t tq_record_words(int32_t d, int32_t idx_bits, int32_t qjl) {
  if (d < 8 || d > kMaxD || d % 8 != 0 || idx_bits < 1 || idx_bits > kMaxBits || (qjl != 0 && qjl != 1)) return -1;
  return rec_words_of(d, idx_bits, qjl);
}

int32_t tq_record_words_mixed(int32_t d, int32_t idx_bits, int32_t n_hi, int32_t qjl) {
  if (tq_record_words(d, idx_bits, qjl) < 0) return -1;
  if (n_hi != 0 && (n_hi < 0 || n_hi % 32 != 0 || n_hi >= d || idx_bits + 1 > kMaxBits)) return -1;
  return rec_words_of(d, idx_bits, qjl, n_hi);
}

tq_status tq_codebook_fit(int32_t d, int32_t idx_bits, float *centroids_host) {
  g_err[0] = 0;
  if (d < 3 || d > 4096 || idx_bits < 1 || idx_bits > 8)
    return fail(TQ_ERR_UNSUPPORTED, "tq_codebook_fit: d=%d idx_bits=%d (need d 3..4096, bits 1..8)", d, idx_bits);
  if (!centroids_host) return fail(TQ_ERR_INVALID, "tq_codebook_fit: output is NULL");
  if (!fit_lloyd_max(d, idx_bits, centroids_host)) return fail(TQ_ERR_INVALID, "tq_codebook_fit: iteration diverged");
  return TQ_OK;
}

tq_status tq_sketch_rotation(int32_t d, const float *Pi, const float *S, float *SPiT, tq_stream stream) {
  g_err[0] = 0;
  if (d < 8 || d > kMaxD) return fail(TQ_ERR_UNSUPPORTED, "tq_sketch_rotation: d=%d", d);
  if (!Pi || !S || !SPiT) return fail(TQ_ERR_INVALID, "tq_sketch_rotation: NULL matrix");
  tq_status s;
  if (injected(&s)) return s;
  cudaError_t e = launch_sketch_rotation(d, Pi, S, SPiT, (cudaStream_t)stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_sketch_rotation");
}

tq_status tq_quantize_append(const tq_cache *cache, const void *x, tq_dtype dtype, int64_t pos, int64_t n_tokens,
                             const float *Pi, const float *SPiT, const float *codebook, tq_stream stream) {
  g_err[0] = 0;
  tq_status s = check_cache(cache, "tq_quantize_append");
  if (s != TQ_OK) return s;
  if (dtype != TQ_BF16 && dtype != TQ_FP16 && dtype != TQ_FP32)
    return fail(TQ_ERR_INVALID, "tq_quantize_append: dtype=%d", (int)dtype);
  if (pos < 0 || n_tokens < 0) return fail(TQ_ERR_INVALID, "tq_quantize_append: pos=%lld n_tokens=%lld",
                                           (long long)pos, (long long)n_tokens);
  if (pos + n_tokens > cache->capacity)
    return fail(TQ_ERR_CAPACITY, "tq_quantize_append: pos %lld + n_tokens %lld > capacity %lld", (long long)pos,
                (long long)n_tokens, (long long)cache->capacity);
  if (n_tokens == 0) return TQ_OK;
  const size_t esz = dtype == TQ_FP32 ? 4 : 2;
  if (!x || !aligned(x, esz)) return fail(TQ_ERR_INVALID, "tq_quantize_append: x NULL or misaligned");
  if (!Pi || !codebook) return fail(TQ_ERR_INVALID, "tq_quantize_append: Pi or codebook NULL");
  if (cache->qjl && !SPiT) return fail(TQ_ERR_INVALID, "tq_quantize_append: key cache needs SPiT");
  if (injected(&s)) return s;
  QuantParams p{};
  p.x = x;
  p.records = cache->records;
  p.norm = cache->norm;
  p.rnorm = cache->rnorm;
  p.Pi = Pi;
  p.SPiT = SPiT;
  p.codebook = codebook;
  p.rows = (int64_t)cache->n_seq * cache->n_kv_heads * n_tokens;
  p.n_tokens = n_tokens;
  p.capacity = cache->capacity;
  p.pos = pos;
  p.d = cache->d;
  p.rec_words = rec_words_of(cache->d, cache->idx_bits, cache->qjl, cache->n_hi);
  p.idx_words = idx_words_of(cache->d, cache->idx_bits, cache->n_hi);
  p.n_hi = cache->n_hi;
  cudaError_t e = launch_quantize(p, cache->idx_bits, cache->qjl != 0, dtype, (cudaStream_t)stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_quantize_append");
}

tq_status tq_quantize_append_hadamard(const tq_cache *cache, const void *x, tq_dtype dtype, int64_t pos,
                                      int64_t n_tokens, const float *signs, const float *SPiT,
                                      const float *codebook, tq_stream stream) {
  g_err[0] = 0;
  tq_status s = check_cache(cache, "tq_quantize_append_hadamard");
  if (s != TQ_OK) return s;
  const int d = cache->d;
  if (d < 32 || d > 256 || (d & (d - 1)) != 0)
    return fail(TQ_ERR_UNSUPPORTED, "tq_quantize_append_hadamard: d=%d is not a power of two in [32, 256]", d);
  if (dtype != TQ_BF16 && dtype != TQ_FP16 && dtype != TQ_FP32)
    return fail(TQ_ERR_INVALID, "tq_quantize_append_hadamard: dtype=%d", (int)dtype);
  if (pos < 0 || n_tokens < 0)
    return fail(TQ_ERR_INVALID, "tq_quantize_append_hadamard: pos=%lld n_tokens=%lld", (long long)pos,
                (long long)n_tokens);
  if (pos + n_tokens > cache->capacity)
    return fail(TQ_ERR_CAPACITY, "tq_quantize_append_hadamard: pos %lld + n_tokens %lld > capacity %lld",
                (long long)pos, (long long)n_tokens, (long long)cache->capacity);
  if (n_tokens == 0) return TQ_OK;
  const size_t esz = dtype == TQ_FP32 ? 4 : 2;
  if (!x || !aligned(x, esz)) return fail(TQ_ERR_INVALID, "tq_quantize_append_hadamard: x NULL or misaligned");
  if (!signs || !aligned(signs, 4) || !codebook)
    return fail(TQ_ERR_INVALID, "tq_quantize_append_hadamard: signs or codebook NULL or misaligned");
  if (cache->qjl && !SPiT) return fail(TQ_ERR_INVALID, "tq_quantize_append_hadamard: key cache needs SPiT");
  if (injected(&s)) return s;
  QuantParams p{};
  p.x = x;
  p.records = cache->records;
  p.norm = cache->norm;
  p.rnorm = cache->rnorm;
  p.signs = signs;
  p.SPiT = SPiT;
  p.codebook = codebook;
  p.rows = (int64_t)cache->n_seq * cache->n_kv_heads * n_tokens;
  p.n_tokens = n_tokens;
  p.capacity = cache->capacity;
  p.pos = pos;
  p.d = d;
  p.rec_words = rec_words_of(d, cache->idx_bits, cache->qjl, cache->n_hi);
  p.idx_words = idx_words_of(d, cache->idx_bits, cache->n_hi);
  p.n_hi = cache->n_hi;
  cudaError_t e = launch_quantize_hadamard(p, cache->idx_bits, cache->qjl != 0, dtype, (cudaStream_t)stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_quantize_append_hadamard");
}

// Workspace of tq_logits: status word | Pi q | S q, and for the grouped-query
// path a 256-byte aligned table block per unit and one scale per query head.
namespace {
struct LogitsWs {
  size_t proj, tables, sigma, total;
  int qh, units;
};
LogitsWs logits_ws(const tq_cache *k, int32_t n_q_heads) {
  LogitsWs w{};
  w.proj = kWsHeader;
  w.tables = w.proj + ((2 * sizeof(float) * (size_t)k->n_seq * n_q_heads * k->d + 255) & ~(size_t)255);
  w.sigma = w.tables;
  w.total = w.tables;
  const int group = k->n_kv_heads > 0 ? n_q_heads / k->n_kv_heads : 0;
  if (k->qjl && k->n_hi == 0 && group * k->n_kv_heads == n_q_heads && gqa_supported(k->d, k->idx_bits, group)) {
    w.qh = group >= 4 ? 4 : 2;
    w.units = k->n_seq * k->n_kv_heads * (group / w.qh);
    w.sigma = w.tables + gqa_table_bytes(w.units);
    w.total = w.sigma + ((sizeof(float) * (size_t)k->n_seq * n_q_heads + 255) & ~(size_t)255);
  }
  return w;
}
}  // namespace

size_t tq_logits_workspace_size(const tq_cache *k, int32_t n_q_heads) {
  if (!k || k->n_seq <= 0 || k->d <= 0 || n_q_heads <= 0 || k->n_kv_heads <= 0) return 0;
  return logits_ws(k, n_q_heads).total;
}

tq_status tq_logits(const tq_cache *k, const float *q, int32_t n_q_heads, int64_t n_tokens, const float *Pi,
                    const float *S, const float *codebook, float *logits, void *workspace, size_t workspace_bytes,
                    tq_stream stream) {
  g_err[0] = 0;
  tq_status s = check_cache(k, "tq_logits");
  if (s != TQ_OK) return s;
  if (!k->qjl) return fail(TQ_ERR_INVALID, "tq_logits: the cache is a value cache (qjl == 0)");
  if (n_q_heads <= 0 || n_q_heads % k->n_kv_heads != 0)
    return fail(TQ_ERR_INVALID, "tq_logits: n_q_heads=%d is not a positive multiple of n_kv_heads=%d", n_q_heads,
                k->n_kv_heads);
  if (n_tokens < 0 || n_tokens > k->capacity)
    return fail(TQ_ERR_CAPACITY, "tq_logits: n_tokens=%lld outside [0, capacity=%lld]", (long long)n_tokens,
                (long long)k->capacity);
  if ((int64_t)k->n_seq * n_q_heads > 65535)
    return fail(TQ_ERR_UNSUPPORTED, "tq_logits: n_seq x n_q_heads = %lld exceeds 65535",
                (long long)k->n_seq * n_q_heads);
  if (n_tokens == 0) return TQ_OK;   // nothing to scan (logits may be an empty, NULL tensor)
  if (!q || !Pi || !S || !codebook || !logits) return fail(TQ_ERR_INVALID, "tq_logits: NULL tensor argument");
  const size_t need = tq_logits_workspace_size(k, n_q_heads);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "tq_logits: workspace needs %zu bytes, 256-byte aligned (got %zu)", need,
                workspace_bytes);
  const FastPlan fpl = plan_fast(k, n_q_heads);
  const LogitsPlan pl = plan_logits(k, n_q_heads, n_tokens);
  if (!fpl.use && pl.q_per_cta < 1)
    return fail(TQ_ERR_UNSUPPORTED, "tq_logits: lookup tables for d=%d idx_bits=%d exceed shared memory", k->d,
                k->idx_bits);
  if (injected(&s)) return s;
  uint32_t *status = static_cast<uint32_t *>(workspace);
  float *qrot = reinterpret_cast<float *>(static_cast<char *>(workspace) + kWsHeader);
  float *qsk = qrot + (size_t)k->n_seq * n_q_heads * k->d;
  LogitsWs lw = logits_ws(k, n_q_heads);
  if (!aligned(Pi, 16) || !aligned(S, 16)) lw.qh = 0;   // the table builder reads matrix rows as float4
  cudaError_t e = cudaSuccess;
  if (lw.qh == 0) {
    e = launch_qprep(q, k->n_seq * n_q_heads, k->d, Pi, S, qrot, qsk, status, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tq_logits (query projection)");
  }
  LogitsParams p{};
  p.records = k->records;
  p.norm = k->norm;
  p.rnorm = k->rnorm;
  p.qrot = qrot;
  p.qsk = qsk;
  p.codebook = codebook;
  p.logits = logits;
  p.status = status;
  p.n_tokens = n_tokens;
  p.capacity = k->capacity;
  p.chunk = pl.chunk;
  p.d = k->d;
  p.rec_words = rec_words_of(k->d, k->idx_bits, 1, k->n_hi);
  p.idx_words = idx_words_of(k->d, k->idx_bits, k->n_hi);
  p.n_hi = k->n_hi;
  p.n_kv_heads = k->n_kv_heads;
  p.n_q_heads = n_q_heads;
  p.group = n_q_heads / k->n_kv_heads;
  if (lw.qh > 0) {
    // grouped queries: fp16 tables built once per call, one CTA group per KV head block
    p.q_per_cta = lw.qh;
    p.qblocks = p.group / lw.qh;
    GqaParams g{};
    g.q = q;
    g.Pi = Pi;
    g.S = S;
    g.codebook = codebook;
    g.tables = static_cast<unsigned char *>(workspace) + lw.tables;
    g.sigma = reinterpret_cast<float *>(static_cast<char *>(workspace) + lw.sigma);
    g.status = status;
    g.n_kv_heads = k->n_kv_heads;
    g.n_q_heads = n_q_heads;
    g.group = p.group;
    g.qblocks = p.qblocks;
    e = launch_logits_gqa(p, g, k->idx_bits, k->n_seq, device_smem_optin() - 1024, (cudaStream_t)stream);
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_logits (grouped-query scan)");
  }
  if (fpl.use) {
    p.q_per_cta = fpl.q_per_cta;
    p.qblocks = (p.group + fpl.q_per_cta - 1) / fpl.q_per_cta;
    e = launch_logits_fast(p, k->idx_bits, k->n_seq, fpl.limit, (cudaStream_t)stream);
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_logits (table scan)");
  }
  p.q_per_cta = pl.q_per_cta;
  p.qblocks = pl.qblocks;
  e = launch_logits(p, k->idx_bits, k->n_seq, pl.n_chunks, pl.smem, (cudaStream_t)stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_logits (scan)");
}

size_t tq_attend_workspace_size(const tq_cache *v, int32_t n_q_heads, int64_t n_tokens) {
  if (!v || v->n_seq <= 0 || v->d <= 0 || n_q_heads <= 0 || n_tokens < 0) return 0;
  return attend_ws_bytes(v, n_q_heads, n_tokens);
}

namespace {
// tq_attend_v, or with `merged` the merged partial (M, L, A) of this token range (tq_attend_v_partial).
tq_status attend_impl(const tq_cache *v, const float *logits, float scale, int32_t n_q_heads, int64_t n_tokens,
                      const float *Pi, const float *codebook, float *out, float *merged, void *workspace,
                      size_t workspace_bytes, tq_stream stream, const char *what) {
  tq_status s = check_attend_args(v, logits, scale, n_q_heads, n_tokens, Pi, codebook, merged ? merged : out, what,
                                  merged == nullptr);
  if (s != TQ_OK) return s;
  const size_t need = tq_attend_workspace_size(v, n_q_heads, n_tokens);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "%s: workspace needs %zu bytes, 256-byte aligned (got %zu)", what, need,
                workspace_bytes);
  if (injected(&s)) return s;
  const size_t out_bytes = sizeof(float) * (size_t)v->n_seq * n_q_heads * v->d;
  if (n_tokens == 0) {
    cudaError_t e = merged ? launch_empty_partial(merged, v->n_seq * n_q_heads, v->d, (cudaStream_t)stream)
                           : cudaMemsetAsync(out, 0, out_bytes, (cudaStream_t)stream);
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, what);
  }
  if ((n_tokens + kAttendChunk - 1) / kAttendChunk > 50000)
    return fail(TQ_ERR_UNSUPPORTED, "%s: n_tokens=%lld exceeds the merge limit of %lld tokens", what,
                (long long)n_tokens, 50000LL * kAttendChunk);
  uint32_t *status = static_cast<uint32_t *>(workspace);
  float *partial = reinterpret_cast<float *>(static_cast<char *>(workspace) + kWsHeader);
  const int group = n_q_heads / v->n_kv_heads;
  AttendParams p{};
  p.records = v->records;
  p.norm = v->norm;
  p.logits = logits;
  p.codebook = codebook;
  p.partial = partial;
  p.status = status;
  p.n_tokens = n_tokens;
  p.capacity = v->capacity;
  p.chunk = kAttendChunk;
  p.n_chunks = (int)((n_tokens + kAttendChunk - 1) / kAttendChunk);
  p.scale = scale;
  p.d = v->d;
  p.rec_words = rec_words_of(v->d, v->idx_bits, 0, v->n_hi);
  p.n_hi = v->n_hi;
  p.stall_tries = debug_stall_tries();
  p.n_kv_heads = v->n_kv_heads;
  p.n_q_heads = n_q_heads;
  p.group = group;
  p.q_per_cta = group < kAttendMaxQ ? group : kAttendMaxQ;
  p.qblocks = (group + p.q_per_cta - 1) / p.q_per_cta;
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, what);
  if (attend_fast_supported(v->d, v->idx_bits, p.q_per_cta, v->records, v->n_hi, v->capacity)) {
    // d = 128: tiles streamed by bulk copies, chunks sized to whole waves (never more chunks than
    // the 512-token split the workspace is sized for)
    p.chunk = attend_fast_chunk(n_tokens, v->n_seq * v->n_kv_heads * p.qblocks);
    p.n_chunks = (int)((n_tokens + p.chunk - 1) / p.chunk);
    e = launch_attend_fast(p, v->idx_bits, v->n_seq, (cudaStream_t)stream);
  } else {
    e = launch_attend(p, v->idx_bits, v->n_seq, attend_chunk_smem(v->d, p.rec_words, kAttendChunk),
                      (cudaStream_t)stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, what);
  e = launch_combine(partial, v->n_seq * n_q_heads, p.n_chunks, v->d, Pi, out, (cudaStream_t)stream, merged);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, what);
}
}  // namespace

tq_status tq_attend_v(const tq_cache *v, const float *logits, float scale, int32_t n_q_heads, int64_t n_tokens,
                      const float *Pi, const float *codebook, float *out, void *workspace, size_t workspace_bytes,
                      tq_stream stream) {
  g_err[0] = 0;
  return attend_impl(v, logits, scale, n_q_heads, n_tokens, Pi, codebook, out, nullptr, workspace, workspace_bytes,
                     stream, "tq_attend_v");
}

tq_status tq_attend_v_partial(const tq_cache *v, const float *logits, float scale, int32_t n_q_heads,
                              int64_t n_tokens, const float *codebook, float *partial, void *workspace,
                              size_t workspace_bytes, tq_stream stream) {
  g_err[0] = 0;
  if (!partial) return fail(TQ_ERR_INVALID, "tq_attend_v_partial: partial is NULL");
  return attend_impl(v, logits, scale, n_q_heads, n_tokens, nullptr, codebook, nullptr, partial, workspace,
                     workspace_bytes, stream, "tq_attend_v_partial");
}

tq_status tq_attend_merge(const float *partials, int32_t n_parts, int32_t rows, int32_t d, const float *Pi, float *out,
                          tq_stream stream) {
  g_err[0] = 0;
  if (d < 8 || d > kMaxD || d % 8 != 0) return fail(TQ_ERR_UNSUPPORTED, "tq_attend_merge: d=%d", d);
  if (n_parts < 1 || n_parts > 50000 || rows < 0)
    return fail(TQ_ERR_INVALID, "tq_attend_merge: n_parts=%d (need 1..50000) rows=%d", n_parts, rows);
  if (rows == 0) return TQ_OK;
  if (!partials || !Pi || !out) return fail(TQ_ERR_INVALID, "tq_attend_merge: NULL tensor argument");
  tq_status s;
  if (injected(&s)) return s;
  cudaError_t e = launch_combine(partials, rows, n_parts, d, Pi, out, (cudaStream_t)stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_attend_merge");
}

tq_status tq_nn_merge(const float *part_scores, const int64_t *part_ids, int32_t n_parts, int32_t n_queries,
                      int32_t k, float *top_scores, int64_t *top_ids, tq_stream stream) {
  g_err[0] = 0;
  if (k < 1 || k > kNnMaxK) return fail(TQ_ERR_INVALID, "tq_nn_merge: k=%d (need 1..%d)", k, kNnMaxK);
  if (n_parts < 1 || n_queries < 0) return fail(TQ_ERR_INVALID, "tq_nn_merge: n_parts=%d n_queries=%d", n_parts, n_queries);
  if (n_queries == 0) return TQ_OK;
  if (!part_scores || !part_ids || !top_scores || !top_ids) return fail(TQ_ERR_INVALID, "tq_nn_merge: NULL tensor argument");
  tq_status s;
  if (injected(&s)) return s;
  cudaError_t e = launch_nn_list_merge(part_scores, part_ids, n_parts, n_queries, k, top_scores, top_ids,
                                       (cudaStream_t)stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_nn_merge");
}

// Workspace of tq_decode_attend. Fused path: status word | Pi q | S q | chunk partials.
// Otherwise: status word | logits | tq_logits workspace | tq_attend_v workspace.
namespace {

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

struct DecodeWs {
  bool fused, gqa;
  size_t qrot, qsk, partial;                  // fused (one query head per KV head); partial also grouped
  size_t tables, sigma;                       // fused grouped queries
  int qh;                                     // query heads per grouped-query unit
  size_t logits, ws_l, ws_l_bytes, ws_a, ws_a_bytes;   // two calls
  size_t total;
};

bool same_heads(const tq_cache *k, const tq_cache *v) {
  return k->d == v->d && k->n_seq == v->n_seq && k->n_kv_heads == v->n_kv_heads;
}

DecodeWs decode_ws(const tq_cache *k, const tq_cache *v, int n_q_heads, int64_t n_tokens) {
  DecodeWs w{};
  w.fused = k->n_hi == 0 && v->n_hi == 0 &&
            decode_fused_supported(k->d, k->idx_bits, v->idx_bits, n_q_heads, k->n_kv_heads, k->records,
                                   v->records, device_smem_optin() - 1024);
  const size_t rows = (size_t)k->n_seq * n_q_heads;
  const int group = n_q_heads / k->n_kv_heads;
  w.gqa = !w.fused && k->n_hi == 0 && v->n_hi == 0 && group * k->n_kv_heads == n_q_heads &&
          decode_gqa_supported(k->d, k->idx_bits, v->idx_bits, group, device_smem_optin() - 1024);
  if (w.fused) {
    const int64_t n_chunks = (n_tokens + kAttendChunk - 1) / kAttendChunk;   // at least as many as the split uses
    w.qrot = kWsHeader;
    w.qsk = w.qrot + align256(sizeof(float) * rows * k->d);
    w.partial = w.qsk + align256(sizeof(float) * rows * k->d);
    w.total = w.partial + sizeof(float) * rows * (size_t)n_chunks * (k->d + 2);
  } else {
    w.logits = kWsHeader;
    w.ws_l = w.logits + align256(sizeof(float) * rows * (size_t)n_tokens);
    w.ws_l_bytes = align256(tq_logits_workspace_size(k, n_q_heads));
    w.ws_a = w.ws_l + w.ws_l_bytes;
    w.ws_a_bytes = tq_attend_workspace_size(v, n_q_heads, n_tokens);
    w.total = w.ws_a + w.ws_a_bytes;
    if (w.gqa) {
      // status word | tables of every unit | per-head table scales | chunk partials; the two-call
      // layout (used when the matrices are not 16-byte aligned) also has to fit
      w.qh = group >= 4 ? 4 : 2;
      const int units = k->n_seq * k->n_kv_heads * (group / w.qh);
      const int64_t n_chunks = (n_tokens + kAttendChunk - 1) / kAttendChunk;   // at least as many as the split uses
      w.tables = kWsHeader;
      w.sigma = w.tables + align256(gqa_table_bytes(units));
      w.partial = w.sigma + align256(sizeof(float) * rows);
      const size_t total_gqa = w.partial + sizeof(float) * rows * (size_t)n_chunks * (k->d + 2);
      if (total_gqa > w.total) w.total = total_gqa;
    }
  }
  return w;
}

}  // namespace

size_t tq_decode_workspace_size(const tq_cache *k, const tq_cache *v, int32_t n_q_heads, int64_t n_tokens) {
  if (!k || !v || k->n_seq <= 0 || k->d <= 0 || k->n_kv_heads <= 0 || n_q_heads <= 0 || n_tokens < 0 ||
      !same_heads(k, v))
    return 0;
  return decode_ws(k, v, n_q_heads, n_tokens).total;
}

tq_status tq_decode_attend(const tq_cache *k, const tq_cache *v, const float *q, int32_t n_q_heads,
                           int64_t n_tokens, float scale, const float *Pi, const float *S,
                           const float *codebook_k, const float *codebook_v, float *out, void *workspace,
                           size_t workspace_bytes, tq_stream stream) {
  g_err[0] = 0;
  tq_status s = check_cache(k, "tq_decode_attend (keys)");
  if (s != TQ_OK) return s;
  s = check_cache(v, "tq_decode_attend (values)");
  if (s != TQ_OK) return s;
  if (!k->qjl || v->qjl) return fail(TQ_ERR_INVALID, "tq_decode_attend: k must be a key cache (qjl 1), v a value cache (qjl 0)");
  if (!same_heads(k, v))
    return fail(TQ_ERR_INVALID, "tq_decode_attend: key and value caches differ in d, n_seq or n_kv_heads");
  if (n_q_heads <= 0 || n_q_heads % k->n_kv_heads != 0)
    return fail(TQ_ERR_INVALID, "tq_decode_attend: n_q_heads=%d is not a positive multiple of n_kv_heads=%d",
                n_q_heads, k->n_kv_heads);
  if (n_tokens < 0 || n_tokens > k->capacity || n_tokens > v->capacity)
    return fail(TQ_ERR_CAPACITY, "tq_decode_attend: n_tokens=%lld outside [0, capacity]", (long long)n_tokens);
  if ((int64_t)k->n_seq * n_q_heads > 65535)
    return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attend: n_seq x n_q_heads = %lld exceeds 65535",
                (long long)k->n_seq * n_q_heads);
  if (!q || !Pi || !S || !codebook_k || !codebook_v || !out)
    return fail(TQ_ERR_INVALID, "tq_decode_attend: NULL tensor argument");
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(TQ_ERR_INVALID, "tq_decode_attend: scale is not finite");
  const DecodeWs w = decode_ws(k, v, n_q_heads, n_tokens);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.total)
    return fail(TQ_ERR_WORKSPACE, "tq_decode_attend: workspace needs %zu bytes, 256-byte aligned (got %zu)", w.total,
                workspace_bytes);
  if (injected(&s)) return s;
  if ((n_tokens + kAttendChunk - 1) / kAttendChunk > 50000)
    return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attend: n_tokens=%lld exceeds the merge limit of %lld tokens",
                (long long)n_tokens, 50000LL * kAttendChunk);
  char *ws = static_cast<char *>(workspace);
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  const size_t out_bytes = sizeof(float) * (size_t)k->n_seq * n_q_heads * k->d;
  cudaError_t e = cudaSuccess;
  if (n_tokens == 0) {
    e = cudaMemsetAsync(out, 0, out_bytes, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, sizeof(uint32_t), (cudaStream_t)stream);
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_decode_attend (empty)");
  }
  if (w.gqa && aligned(Pi, 16) && aligned(S, 16)) {
    // grouped queries: the grouped-query tables once per call (they also clear the status word),
    // then one pass over keys and values per (chunk, unit), then the merge
    const int group = n_q_heads / k->n_kv_heads;
    const int qblocks = group / w.qh;
    const int units = k->n_seq * k->n_kv_heads * qblocks;
    unsigned char *tables = reinterpret_cast<unsigned char *>(ws + w.tables);
    float *sigma = reinterpret_cast<float *>(ws + w.sigma);
    float *partial = reinterpret_cast<float *>(ws + w.partial);
    GqaParams g{};
    g.q = q;
    g.Pi = Pi;
    g.S = S;
    g.codebook = codebook_k;
    g.tables = tables;
    g.sigma = sigma;
    g.status = status;
    g.n_kv_heads = k->n_kv_heads;
    g.n_q_heads = n_q_heads;
    g.group = group;
    g.qblocks = qblocks;
    e = launch_gqa_tables(g, k->idx_bits, w.qh, units, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attend (grouped-query tables)");
    DecodeGqaArgs a{};
    a.krec = k->records;
    a.knorm = k->norm;
    a.krnorm = k->rnorm;
    a.vrec = v->records;
    a.vnorm = v->norm;
    a.tables = tables;
    a.sigma = sigma;
    a.cbv = codebook_v;
    a.partial = partial;
    a.status = status;
    a.n_tokens = n_tokens;
    a.cap_k = k->capacity;
    a.cap_v = v->capacity;
    a.chunk = attend_fast_chunk(n_tokens, units);   // the softmax.V kernel's split
    a.n_seq = k->n_seq;
    a.n_kv_heads = k->n_kv_heads;
    a.n_q_heads = n_q_heads;
    a.qblocks = qblocks;
    a.n_chunks = (int)((n_tokens + a.chunk - 1) / a.chunk);
    a.kbits = k->idx_bits;
    a.vbits = v->idx_bits;
    a.scale = scale;
    a.smem_limit = device_smem_optin() - 1024;
    e = launch_decode_gqa(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attend (grouped-query pass)");
    e = launch_combine(partial, k->n_seq * n_q_heads, a.n_chunks, k->d, Pi, out, (cudaStream_t)stream);
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_decode_attend (merge)");
  }
  if (!w.fused) {
    // other head groupings and code widths: the two calls, their status words merged into this one
    s = tq_logits(k, q, n_q_heads, n_tokens, Pi, S, codebook_k, reinterpret_cast<float *>(ws + w.logits), ws + w.ws_l,
                  w.ws_l_bytes, stream);
    if (s != TQ_OK) return s;
    s = tq_attend_v(v, reinterpret_cast<const float *>(ws + w.logits), scale, n_q_heads, n_tokens, Pi, codebook_v, out,
                    ws + w.ws_a, w.ws_a_bytes, stream);
    if (s != TQ_OK) return s;
    e = launch_status_or(status, reinterpret_cast<const uint32_t *>(ws + w.ws_l),
                         reinterpret_cast<const uint32_t *>(ws + w.ws_a), (cudaStream_t)stream);
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_decode_attend (status)");
  }
  float *qrot = reinterpret_cast<float *>(ws + w.qrot), *qsk = reinterpret_cast<float *>(ws + w.qsk);
  float *partial = reinterpret_cast<float *>(ws + w.partial);
  // the projection clears the status word and lets the fused grid start streaming tiles
  e = launch_qprep(q, k->n_seq * n_q_heads, k->d, Pi, S, qrot, qsk, status, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attend (query projection)");
  DecodeFusedArgs a{};
  a.krec = k->records;
  a.knorm = k->norm;
  a.krnorm = k->rnorm;
  a.vrec = v->records;
  a.vnorm = v->norm;
  a.qrot = qrot;
  a.qsk = qsk;
  a.cbk = codebook_k;
  a.cbv = codebook_v;
  a.partial = partial;
  a.status = status;
  a.n_tokens = n_tokens;
  a.cap_k = k->capacity;
  a.cap_v = v->capacity;
  a.chunk = attend_fast_chunk(n_tokens, k->n_seq * k->n_kv_heads);
  a.n_seq = k->n_seq;
  a.n_heads = n_q_heads;
  a.n_chunks = (int)((n_tokens + a.chunk - 1) / a.chunk);
  a.kbits = k->idx_bits;
  a.vbits = v->idx_bits;
  a.scale = scale;
  a.smem_limit = device_smem_optin() - 1024;
  e = launch_decode_fused(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode_attend (fused scan)");
  e = launch_combine(partial, k->n_seq * n_q_heads, a.n_chunks, k->d, Pi, out, (cudaStream_t)stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_decode_attend (merge)");
}

// Workspace of tq_nn_search: header | fp16 query rows | per-query scale | partial top-k lists
// (two per row for each (CTA, query block) pair a CTA's contiguous unit range touches:
// grid + blocks - 1 pairs).
struct NnWs {
  size_t qimg, sigma, part_s, part_i, total;
};

NnWs nn_ws(int d, int n_queries, int64_t n_db) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  const int64_t n_qb = (n_queries + 127) / 128, n_tiles = (n_db + 127) / 128, units = n_qb * n_tiles;
  const int64_t grid = units < kNnMaxGrid ? units : kNnMaxGrid;
  const int64_t slots = grid > 0 ? grid + n_qb - 1 : 0;
  NnWs w{};
  w.qimg = kWsHeader;
  w.sigma = w.qimg + up((size_t)n_qb * 128 * nn_kp(d) * 2);
  w.part_s = w.sigma + up((size_t)n_qb * 128 * sizeof(float));
  w.part_i = w.part_s + up((size_t)slots * 128 * 2 * kNnMaxK * sizeof(float));
  w.total = w.part_i + up((size_t)slots * 128 * 2 * kNnMaxK * sizeof(int));
  return w;
}

size_t tq_nn_workspace_size(const tq_cache *db, int32_t n_queries, int64_t n_db) {
  if (!db || db->d <= 0 || n_queries < 0 || n_db < 0) return 0;
  return nn_ws(db->d, n_queries, n_db).total;
}

tq_status tq_nn_search(const tq_cache *db, const float *queries, int32_t n_queries, int64_t n_db, const float *Pi,
                       const float *S, const float *codebook, int32_t k, float *top_scores, int64_t *top_ids,
                       void *workspace, size_t workspace_bytes, tq_stream stream) {
  g_err[0] = 0;
  tq_status s = check_cache(db, "tq_nn_search");
  if (s != TQ_OK) return s;
  if (!db->qjl) return fail(TQ_ERR_INVALID, "tq_nn_search: the database must be a key cache (qjl = 1)");
  if (db->n_seq != 1 || db->n_kv_heads != 1)
    return fail(TQ_ERR_INVALID, "tq_nn_search: the database is one stream (n_seq = n_kv_heads = 1), got %d x %d",
                db->n_seq, db->n_kv_heads);
  if (db->n_hi != 0 || !nn_supported(db->d, db->idx_bits))
    return fail(TQ_ERR_UNSUPPORTED, "tq_nn_search: d=%d idx_bits=%d (need d 128 or 200, idx_bits 1..3)", db->d,
                db->idx_bits);
  if (k < 1 || k > kNnMaxK) return fail(TQ_ERR_INVALID, "tq_nn_search: k=%d (need 1..%d)", k, kNnMaxK);
  if (n_queries < 0) return fail(TQ_ERR_INVALID, "tq_nn_search: n_queries=%d", n_queries);
  if (n_db < 0 || n_db > db->capacity)
    return fail(TQ_ERR_CAPACITY, "tq_nn_search: n_db=%lld outside [0, capacity=%lld]", (long long)n_db,
                (long long)db->capacity);
  if (n_db > 0x7fffffffLL) return fail(TQ_ERR_UNSUPPORTED, "tq_nn_search: n_db=%lld above 2^31 - 1", (long long)n_db);
  if (n_queries == 0) return TQ_OK;
  if (!queries || !Pi || !S || !codebook || !top_scores || !top_ids)
    return fail(TQ_ERR_INVALID, "tq_nn_search: NULL tensor argument");
  if (!aligned(Pi, 16) || !aligned(S, 16) || !aligned(db->norm, 16) || !aligned(db->rnorm, 16))
    return fail(TQ_ERR_INVALID, "tq_nn_search: Pi, S and the database norm and rnorm arrays must be 16-byte aligned");
  const NnWs w = nn_ws(db->d, n_queries, n_db);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.total)
    return fail(TQ_ERR_WORKSPACE, "tq_nn_search: workspace needs %zu bytes, 256-byte aligned (got %zu)", w.total,
                workspace_bytes);
  if (injected(&s)) return s;
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  NnArgs a{};
  a.records = db->records;
  a.norm = db->norm;
  a.rnorm = db->rnorm;
  a.q = queries;
  a.Pi = Pi;
  a.S = S;
  a.codebook = codebook;
  a.top_s = top_scores;
  a.top_i = top_ids;
  a.qimg = ws + w.qimg;
  a.sigma = reinterpret_cast<float *>(ws + w.sigma);
  a.part_s = reinterpret_cast<float *>(ws + w.part_s);
  a.part_i = reinterpret_cast<int *>(ws + w.part_i);
  a.status = static_cast<uint32_t *>(workspace);
  a.n_db = n_db;
  a.n_q = n_queries;
  a.d = db->d;
  a.bits = db->idx_bits;
  a.k = k;
  const int64_t units = (int64_t)((n_queries + 127) / 128) * ((n_db + 127) / 128);
  int64_t grid = device_sm_count();
  if (grid > kNnMaxGrid) grid = kNnMaxGrid;
  if (grid > units) grid = units;
  a.grid = (int)grid;
  cudaError_t e = cudaSuccess;
  if (n_db == 0) {   // no scan: the status word is cleared here, the merge writes empty lists
    e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "tq_nn_search (status)");
  }
  e = launch_nn_search(a, (cudaStream_t)stream);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_nn_search");
}

tq_status tq_workspace_status(void *workspace, tq_stream stream) {
  g_err[0] = 0;
  if (!workspace || !aligned(workspace, 256)) return fail(TQ_ERR_WORKSPACE, "tq_workspace_status: bad workspace");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_workspace_status (sync)");
  uint32_t word = 0;
  e = cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "tq_workspace_status (read)");
  if (word == 0) return TQ_OK;
  const uint32_t zero = 0;
  e = cudaMemcpy(workspace, &zero, sizeof zero, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "tq_workspace_status (clear)");
  return fail(TQ_ERR_DEVICE, "tq_workspace_status: kernel status 0x%08x%s", word,
              (word & kDevBadShape) ? " (unexpected shape)" : "");
}

const char *tq_last_error(void) { return g_err; }

void tq_debug_inject(tq_status status, int32_t count) {
  g_inject_status.store((int)status);
  g_inject_count.store(count > 0 ? count : 0);
}

void tq_debug_stall_consumers(uint32_t tries) { g_stall_tries.store(tries); }

}  // extern "C"
