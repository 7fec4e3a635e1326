/*
 * tq.h -- C ABI of the B200 (sm_100a) TurboQuant KV-cache library.
 *
 * TurboQuant stores each key/value head-vector x (dimension d) as its L2 norm,
 * the per-coordinate codes of the randomly rotated unit vector under a
 * Lloyd-Max scalar quantizer fitted to the Beta-shaped coordinate law, and,
 * for keys, a 1-bit Johnson-Lindenstrauss sketch of the residual plus the
 * residual norm. Attention logits and softmax-weighted values are computed
 * directly on that packed cache.
 *   - zubnet.ai news, "Google's TurboQuant quantizes LLM KV cache to 3.5 bits
 *     per channel", paragraph 2 (two-stage pipeline; storage = indices, sign
 *     bits, one L2-norm scalar);
 *   - winningdata.io, "TurboQuant: Google comprime KV cache para 3 bits sem
 *     perder acuracia", "Como o TurboQuant funciona" ("1. PolarQuant": random
 *     orthogonal rotation; "2. QJL Residual": one extra bit per value removes
 *     the inner-product bias);
 *   - usedby.ai, "TurboQuant: Compresion de KV Cache a 3 bits y aceleracion de
 *     inferencia en H100", "El Pitch" (logits computed on compressed keys).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller unless the
 *     comment says "host". Scratch space is a caller-provided workspace whose
 *     size a *_workspace_size call returns. The library's one allocation is
 *     8 KB of tile-schedule counters per device and CUDA context, made by the
 *     first tq_quantize_append of keys that runs on the tensor cores (a
 *     cudaMalloc: make that call before recording graphs; a call recorded
 *     before it takes its tiles in a fixed order instead, with the same
 *     result). A stream's first such call, and each such call recorded into a
 *     graph, enqueues an 8-byte memset on the stream.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous: no entry point synchronises the stream,
 *     except tq_workspace_status and tq_attend_v_noalloc_status, which say so.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check launches nothing and returns a status. Launch failures return
 *     TQ_ERR_CUDA. tq_last_error() gives a thread-local message for the last
 *     failure on the calling thread.
 *   - Nothing aborts, asserts, traps or throws across the ABI.
 *
 * Cache record layout (one record per (sequence, kv head, token)):
 *   R = index_words + sign_words little-endian uint32 words, with
 *   index_words = ceil(idx_bits*d/32) and sign_words = ceil(d/32) for keys
 *   (qjl = 1), 0 for values.
 *   Index field: a bit stream (stream bit k = bit k%32 of word k/32); the
 *   idx_bits-bit code of coordinate i sits at stream bits
 *   [idx_bits*i, idx_bits*i + idx_bits), least significant bit first.
 *   Sign field (keys): bit i = [ (S r)_i >= 0 ] at bit i%32 of word
 *   index_words + i/32. Every unused bit is 0.
 *   Records of one (sequence, head) are contiguous in token order; the array
 *   is [n_seq][n_kv_heads][capacity][R]. Norms are separate float arrays
 *   [n_seq][n_kv_heads][capacity].
 *
 * Fractional bits per channel (zubnet.ai, title and paragraph 2: 3.5 and 2.5
 * bits per channel; the pages do not say how a fractional rate is reached).
 * This library's reading: a cache with n_hi = m > 0 gives the first m rotated
 * coordinates idx_bits + 1 code bits and the other d - m coordinates idx_bits,
 * each group quantized with the Lloyd-Max codebook of the same coordinate law at
 * its own width; the average rate is idx_bits + m/d code bits per coordinate
 * (plus the sign bit for keys). Keys at 3.5 bits per channel: idx_bits 2,
 * m = d/2; values at 3.5: idx_bits 3, m = d/2. The code of coordinate i < m sits
 * at stream bits [(idx_bits+1) i, (idx_bits+1)(i+1)), the code of i >= m at
 * [(idx_bits+1) m + idx_bits (i-m), ... + idx_bits); index_words =
 * ceil(((idx_bits+1) m + idx_bits (d-m)) / 32); the sign field follows as above.
 * Every entry point that takes a codebook then takes both: 2^idx_bits floats of
 * the idx_bits codebook followed by 2^(idx_bits+1) floats of the wider one.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so that this header needs no CUDA include. */
typedef struct CUstream_st *tq_stream;

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID = 1,     /* null or misaligned pointer, negative or inconsistent size   */
  TQ_ERR_UNSUPPORTED = 2, /* d or idx_bits outside the supported range                    */
  TQ_ERR_CAPACITY = 3,    /* pos + n_tokens exceeds the cache capacity                     */
  TQ_ERR_WORKSPACE = 4,   /* workspace missing, misaligned or smaller than required        */
  TQ_ERR_CUDA = 5,        /* a CUDA runtime call or a kernel launch failed                 */
  TQ_ERR_DEVICE = 6       /* a kernel recorded a failure in the workspace status word     */
} tq_status;

typedef enum { TQ_BF16 = 0, TQ_FP16 = 1, TQ_FP32 = 2 } tq_dtype;

/* Describes one packed K or V cache. All pointers are device memory owned by
 * the caller; `records` must be 16-byte aligned, `norm`/`rnorm` 4-byte aligned. */
typedef struct {
  int32_t d;          /* head dimension: 8..256, multiple of 8                         */
  int32_t idx_bits;   /* code bits per coordinate: 1..4 (keys use b-1, values use b)   */
  int32_t qjl;        /* 1: key cache (sign field + rnorm), 0: value cache (MSE only)  */
  int32_t n_seq;      /* sequences (batch)                                             */
  int32_t n_kv_heads; /* KV heads per sequence                                         */
  int32_t n_hi;       /* mixed rate: the first n_hi rotated coordinates carry idx_bits+1 */
                      /* code bits, the others idx_bits (0 = integer rate; else a      */
                      /* multiple of 32 below d, with idx_bits + 1 <= 4)               */
  int64_t capacity;   /* token slots per (sequence, head)                              */
  uint32_t *records;  /* [n_seq][n_kv_heads][capacity][tq_record_words(d,idx_bits,qjl)] */
  float *norm;        /* [n_seq][n_kv_heads][capacity]  ||x||                          */
  float *rnorm;       /* same shape, ||r|| of the residual; NULL iff qjl == 0          */
} tq_cache;

/* Words per record for the layout above; -1 if (d, idx_bits) is unsupported. */
int32_t tq_record_words(int32_t d, int32_t idx_bits, int32_t qjl);

/* Words per record of a mixed-rate cache (n_hi coordinates at idx_bits + 1 code
 * bits, see the layout above); n_hi = 0 gives tq_record_words. -1 if unsupported
 * (n_hi not a multiple of 32 in [0, d), or idx_bits + 1 > 4 with n_hi > 0). */
int32_t tq_record_words_mixed(int32_t d, int32_t idx_bits, int32_t n_hi, int32_t qjl);

/* Lloyd-Max codebook for the coordinate law of a uniform point on the unit
 * sphere S^{d-1}, density proportional to (1 - y^2)^((d-3)/2) on [-1, 1]
 * (zubnet.ai, paragraph 2: "optimal scalar quantizer per coordinate" of the
 * Beta-distributed rotated coordinates). Fitted in double precision on the
 * HOST (setup, not the per-token path), made exactly symmetric and rounded to
 * float. `centroids_host` receives 2^idx_bits ascending values (host memory).
 * d: 3..4096; idx_bits: 1..8. */
tq_status tq_codebook_fit(int32_t d, int32_t idx_bits, float *centroids_host);

/* SPiT = S * Pi^T (d x d, row-major float). Pi: the d x d orthogonal rotation
 * (row-major), S: the d x d Gaussian sketch matrix. The key quantizer projects
 * the residual in the rotated domain, where S r = S Pi^T (y - yhat)
 * (winningdata.io, "2. QJL Residual": the sketch acts on the residual).
 * Accumulates in double on the device. d: 8..256. */
tq_status tq_sketch_rotation(int32_t d, const float *Pi, const float *S, float *SPiT, tq_stream stream);

/* Quantize n_tokens new vectors per (sequence, head) and write them into token
 * slots [pos, pos + n_tokens) of `cache` (zubnet.ai, paragraph 2: rotate, MSE
 * quantizer, 1-bit JL sketch of the residual, L2 norm).
 *   x:        [n_seq][n_kv_heads][n_tokens][d] contiguous, dtype `dtype`.
 *   Pi:       [d][d] float rotation, y = Pi x / ||x||.
 *   SPiT:     [d][d] float, S Pi^T (see tq_sketch_rotation); ignored (may be NULL)
 *             for a value cache.
 *   codebook: 2^idx_bits ascending floats; code_i = #{j : y_i > (c_j + c_{j+1})/2}
 *             (mixed rate: the two codebooks, see the layout above).
 * For each vector: norm = ||x||; y = Pi x/||x||; codes; keys also store
 * rnorm = ||y - c[code]|| and sign bits of SPiT (y - c[code]). A zero vector
 * stores norm 0, rnorm 0, codes of y = 0 and all sign bits 1.
 * Errors: TQ_ERR_CAPACITY if pos + n_tokens > capacity; n_tokens == 0 is a no-op. */
tq_status tq_quantize_append(const tq_cache *cache, const void *x, tq_dtype dtype,
                             int64_t pos, int64_t n_tokens,
                             const float *Pi, const float *SPiT, const float *codebook,
                             tq_stream stream);

/* tq_quantize_append with the structured rotation Pi = H diag(signs) / sqrt(d),
 * H the d x d Sylvester-Hadamard matrix in natural order (H_ij = (-1)^popcount(i & j)):
 * y = H (signs * x) / (sqrt(d) ||x||) by a fast Walsh-Hadamard transform, log2(d)
 * rounds of pairwise sums and differences, O(d log d) per vector instead of the
 * dense product's O(d^2) (winningdata.io, "1. PolarQuant", the rotation's cost per
 * vector). Everything else, the record layout included, is tq_quantize_append's,
 * so tq_logits / tq_attend_v / tq_decode_attend read the cache with the dense Pi of
 * the same rotation.
 *   signs: [d] device floats, each +1 or -1.
 *   SPiT:  [d][d] float, S Pi^T for that Pi (tq_sketch_rotation of the dense Pi);
 *          ignored (may be NULL) for a value cache.
 * d must be a power of two in [32, 256] (TQ_ERR_UNSUPPORTED otherwise); x of any
 * dtype; mixed-rate caches are accepted. Runs on the FP32 cores. Other errors as
 * tq_quantize_append. */
tq_status tq_quantize_append_hadamard(const tq_cache *cache, const void *x, tq_dtype dtype,
                                      int64_t pos, int64_t n_tokens,
                                      const float *signs, const float *SPiT, const float *codebook,
                                      tq_stream stream);

/* Workspace bytes tq_logits needs for this key cache and query-head count. */
size_t tq_logits_workspace_size(const tq_cache *k, int32_t n_q_heads);

/* Attention logits on the packed key cache, tokens [0, n_tokens) (usedby.ai,
 * "El Pitch": logits computed directly on the compressed keys):
 *   logits[s][h][t] = norm_t * ( <Pi q, c[code_t]> + rnorm_t * sqrt(pi/2)/d * <S q, 2 sign_t - 1> )
 * where q = q[s][h] and the key cache head is h / (n_q_heads / n_kv_heads).
 *   q:       [n_seq][n_q_heads][d] float.
 *   logits:  [n_seq][n_q_heads][n_tokens] float.
 *   Pi, S:   [d][d] float; codebook: 2^idx_bits floats (the key codebook; a
 *            mixed-rate cache takes its two codebooks, see the layout above).
 * n_q_heads must be a positive multiple of k->n_kv_heads; k->qjl must be 1.
 * workspace: >= tq_logits_workspace_size bytes, 256-byte aligned. */
tq_status tq_logits(const tq_cache *k, const float *q, int32_t n_q_heads, int64_t n_tokens,
                    const float *Pi, const float *S, const float *codebook,
                    float *logits, void *workspace, size_t workspace_bytes, tq_stream stream);

/* Workspace bytes tq_attend_v needs for this value cache, head count and length
 * (SIZE_MAX if that product does not fit a size_t; tq_attend_v then refuses the shape). */
size_t tq_attend_workspace_size(const tq_cache *v, int32_t n_q_heads, int64_t n_tokens);

/* Softmax-weighted sum of the packed values (zubnet.ai, paragraph 1: the cache
 * holds keys and values):
 *   p = softmax_t(scale * logits[s][h][t]),
 *   out[s][h] = Pi^T sum_t p_t * norm_t * c[code_t]     (rotation undone once).
 *   logits: [n_seq][n_q_heads][n_tokens] float; out: [n_seq][n_q_heads][d] float.
 *   codebook: the value codebook (two for a mixed-rate cache, see the layout above).
 *   v->qjl must be 0. n_tokens == 0 writes zeros. Shapes with n_seq x n_kv_heads x
 *   ceil(min(group, 4)-head blocks) above 65535 return TQ_ERR_UNSUPPORTED.
 * workspace: >= tq_attend_workspace_size bytes, 256-byte aligned. */
tq_status tq_attend_v(const tq_cache *v, const float *logits, float scale,
                      int32_t n_q_heads, int64_t n_tokens,
                      const float *Pi, const float *codebook, float *out,
                      void *workspace, size_t workspace_bytes, tq_stream stream);

/* The softmax.V of tq_attend_v for a range of tokens, as a partial that
 * tq_attend_merge combines with the partials of other ranges (for a cache whose
 * tokens are split over GPUs; zubnet.ai, paragraph 1: keys and values).
 * For every row r = (sequence, query head), partial[r] holds d + 2 floats
 *   M = max_t scale * logits_t,  L = sum_t e^{scale * logits_t - M},
 *   A = sum_t e^{scale * logits_t - M} * norm_t * c[code_t]   (rotated domain: no Pi^T).
 * n_tokens == 0 gives (-inf, 0, 0 ... 0). Arguments, checks and workspace
 * (tq_attend_workspace_size) as for tq_attend_v, without Pi.
 *   partial: [n_seq * n_q_heads][d + 2] float. */
tq_status tq_attend_v_partial(const tq_cache *v, const float *logits, float scale,
                              int32_t n_q_heads, int64_t n_tokens, const float *codebook,
                              float *partial, void *workspace, size_t workspace_bytes, tq_stream stream);

/* Combines partials of tq_attend_v_partial: for each row r, with the parts
 * p = 0 .. n_parts-1 of partials[r][p] = (M_p, L_p, A_p),
 *   out[r] = Pi^T (sum_p e^{M_p - M} A_p) / (sum_p e^{M_p - M} L_p),  M = max_p M_p,
 * the same result as tq_attend_v over all the ranges' tokens up to rounding;
 * zeros when every part is empty.
 *   partials: [rows][n_parts][d + 2] float; Pi: [d][d]; out: [rows][d] float.
 * d: 8..256, multiple of 8; n_parts: 1..50000. */
tq_status tq_attend_merge(const float *partials, int32_t n_parts, int32_t rows, int32_t d,
                          const float *Pi, float *out, tq_stream stream);

/* Top-k of several top-k lists per query (nearest-neighbour search over a
 * database split into shards, one tq_nn_search per shard with its ids made
 * global): for each query a, the k best entries of the n_parts lists
 * part_scores / part_ids [n_parts][n_queries][k], each sorted by decreasing
 * score (equal scores: lower id first) with id -1 (score -inf) only in places
 * past its end; ordered the same way; (-inf, -1) where fewer than k exist.
 * top_scores [n_queries][k] float, top_ids [n_queries][k] int64. k: 1..16. */
tq_status tq_nn_merge(const float *part_scores, const int64_t *part_ids, int32_t n_parts,
                      int32_t n_queries, int32_t k, float *top_scores, int64_t *top_ids,
                      tq_stream stream);

/* Workspace bytes tq_decode_attend needs for these caches, head count and length
 * (0 if the caches differ in d, n_seq or n_kv_heads). */
size_t tq_decode_workspace_size(const tq_cache *k, const tq_cache *v, int32_t n_q_heads, int64_t n_tokens);

/* One decode step on the packed caches: the logits of tq_logits, the softmax
 * and the value sum of tq_attend_v (usedby.ai, "El Pitch": attention computed
 * on the compressed cache; zubnet.ai, paragraph 1: keys and values):
 *   out[s][h] = Pi^T sum_t softmax_t(scale * l_t) * vnorm_t * cV[vcode_t],
 *   l_t = knorm_t * ( <Pi q, cK[kcode_t]> + krnorm_t * sqrt(pi/2)/d * <S q, 2 sign_t - 1> ).
 * With d = 128, 1- or 2-bit key codes and 1, 2, 4 or 8 query heads per KV head
 * (value codes of 1..4 bits for one head, 1..3 bits for grouped heads, integer
 * rates, Pi and S 16-byte aligned for grouped heads) the whole step is one pass
 * over the tokens (the logits stay on chip); other shapes run tq_logits and
 * tq_attend_v inside the workspace. Either way the result is bit-equal to
 * tq_logits followed by tq_attend_v.
 *   k: key cache (qjl = 1); v: value cache (qjl = 0), same d, n_seq, n_kv_heads.
 *   q: [n_seq][n_q_heads][d] float; out: [n_seq][n_q_heads][d] float.
 *   Pi, S: [d][d] float; codebook_k / codebook_v: 2^idx_bits floats of each cache
 *   (both codebooks of a mixed-rate cache, see the layout above; mixed-rate caches
 *   run the two calls).
 * n_q_heads must be a positive multiple of n_kv_heads; n_tokens <= both
 * capacities (n_tokens == 0 writes zeros); scale finite.
 * workspace: >= tq_decode_workspace_size bytes, 256-byte aligned; its status
 * word is read by tq_workspace_status. */
tq_status tq_decode_attend(const tq_cache *k, const tq_cache *v, const float *q, int32_t n_q_heads,
                           int64_t n_tokens, float scale, const float *Pi, const float *S,
                           const float *codebook_k, const float *codebook_v, float *out,
                           void *workspace, size_t workspace_bytes, tq_stream stream);

/* Workspace bytes tq_nn_search needs for a database of n_db vectors and n_queries
 * queries (independent of k and of the device). */
size_t tq_nn_workspace_size(const tq_cache *db, int32_t n_queries, int64_t n_db);

/* Nearest-neighbour search on a packed key stream (zubnet.ai, paragraph 3, and
 * winningdata.io, "Os numeros que importam": the quantizer also serves
 * inner-product vector search). For every query a, the k database vectors j in
 * [0, n_db) with the largest estimated inner product
 *   score(a, j) = norm_j * ( <Pi q_a, c[code_j]> + rnorm_j * sqrt(pi/2)/d * <S q_a, 2 sign_j - 1> ),
 * the key estimator of tq_logits, in order of decreasing score (equal scores:
 * lower j first).
 *   db: key cache (qjl = 1, n_hi = 0) with n_seq = n_kv_heads = 1, d 128 or 200,
 *       idx_bits 1..3, filled by tq_quantize_append; its norm and rnorm
 *       arrays 16-byte aligned (they are read by bulk copies).
 *   queries: [n_queries][d] float; Pi, S: [d][d] float, 16-byte aligned;
 *   codebook: 2^idx_bits floats.
 *   top_scores: [n_queries][k] float; top_ids: [n_queries][k] int64. A query
 *   with fewer than k candidates (n_db < k) gets score -inf and id -1 in the
 *   missing places.
 * k: 1..16; n_db <= capacity and < 2^31; n_queries == 0 does nothing.
 * Precision: the products run on the tensor core in fp16 with float32
 * accumulation (Pi q and S q scaled per query by a power of two; centroids and
 * rnorm_j sqrt(pi/2)/d rounded to fp16), so a score differs from the float64
 * value of the estimator by about 1e-4 ||q|| norm_j.
 * workspace: >= tq_nn_workspace_size bytes, 256-byte aligned; its status word
 * is read by tq_workspace_status. */
tq_status tq_nn_search(const tq_cache *db, const float *queries, int32_t n_queries, int64_t n_db,
                       const float *Pi, const float *S, const float *codebook, int32_t k,
                       float *top_scores, int64_t *top_ids,
                       void *workspace, size_t workspace_bytes, tq_stream stream);

/* Synchronises `stream`, reads the status word that the kernels of the last
 * tq_logits / tq_attend_v / tq_decode_attend / tq_nn_search call on this workspace wrote, and clears it.
 * TQ_OK if no kernel reported a failure, TQ_ERR_DEVICE otherwise (the message
 * names the failure). */
tq_status tq_workspace_status(void *workspace, tq_stream stream);

/* Thread-local text of the last failure on this thread ("" if none). */
const char *tq_last_error(void);

/* Host-side fault injection for tests: the next `count` calls that would launch
 * work return `status` instead, before any launch. count = 0 disarms. */
void tq_debug_inject(tq_status status, int32_t count);

/* Failure detection test hook: with tries > 0, the d = 128 softmax.V kernel of
 * the following tq_attend_v / tq_attend_v_partial / tq_decode_attend (two-call
 * path) calls has its consumer warps wait on an mbarrier that nothing completes,
 * for `tries` attempts, so that the wait runs out. The kernel then records a
 * timeout in the call's status word (tq_workspace_status returns TQ_ERR_DEVICE),
 * its copy thread gives up on the stages the consumers never release after as
 * many tries, every copy in flight still lands before the CTA exits, and the
 * context stays usable; the output is undefined. tries = 0 (the default)
 * restores normal operation. Not thread-safe against concurrent calls. */
void tq_debug_stall_consumers(uint32_t tries);

/* Size of the library's built-in scratch array used by tq_attend_v_noalloc:
 * 4 MiB of device memory, held on every GPU that loads this library until the
 * process exits. */
#define TQ_ATTEND_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

/* tq_attend_v without a caller workspace (the pages have no counterpart: this
 * is a deployment convenience of this library).
 *
 * For callers that cannot allocate device memory themselves: code that runs
 * inside a host framework which owns every byte of device memory through its
 * own pool and hands plugins no scratch buffer, or a latency-critical decode
 * loop that must not call cudaMalloc (which can synchronise the device).
 * Arguments and results are those of tq_attend_v; the scratch space comes from
 * a fixed array compiled into the library (TQ_ATTEND_NOALLOC_SCRATCH_BYTES).
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   - The array's device address is looked up (cudaGetSymbolAddress, with the
 *     device current) by the first call in each CUDA context of a device, and
 *     again after the context changes (a cudaDeviceReset loads the library's
 *     device code anew). Make the first call on a device before any stream
 *     capture.
 *   - Arguments are checked exactly as tq_attend_v checks them, with the same
 *     statuses; then TQ_ERR_WORKSPACE, before any launch, when
 *     tq_attend_workspace_size(v, n_q_heads, n_tokens) exceeds the array.
 *   - The kernels' status word sits at the start of the array: read it with
 *     tq_attend_v_noalloc_status, not tq_workspace_status (the caller does not
 *     hold the array's address). The next call clears it.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents: two calls whose work can overlap on the GPU (different
 *     streams, or different host threads) race and corrupt each other's
 *     results. Serialise them on one stream. */
tq_status tq_attend_v_noalloc(const tq_cache *v, const float *logits, float scale,
                              int32_t n_q_heads, int64_t n_tokens,
                              const float *Pi, const float *codebook, float *out,
                              tq_stream stream);

/* tq_workspace_status for the built-in array of tq_attend_v_noalloc on the
 * current device: synchronises `stream`, reads the status word that the kernels
 * of the last tq_attend_v_noalloc call on this device wrote, and clears it.
 * TQ_OK if no kernel reported a failure, TQ_ERR_DEVICE otherwise. Allocates
 * nothing. (No counterpart in the pages.) */
tq_status tq_attend_v_noalloc_status(tq_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
