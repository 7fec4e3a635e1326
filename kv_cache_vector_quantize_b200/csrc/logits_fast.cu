// Logit scan for d = 128 keys (1..3 code bits + the QJL sign field), staged by
// bulk copies and read through bank-conflict-free lookup tables.
//
// Estimator (usedby.ai, "TurboQuant: Compresion de KV Cache a 3 bits y
// aceleracion de inferencia en H100", "El Pitch"; winningdata.io, "TurboQuant:
// Google comprime KV cache para 3 bits sem perder acuracia", "2. QJL
// Residual"):
//   l_t = n_t ( <Pi q, c[code_t]> + rho_t sqrt(pi/2)/d <S q, 2 sign_t - 1> ).
//
// Work split. The key tiles of all (sequence, KV head, query block) units form
// one list. With at least as many units as SMs each CTA (one per SM) takes a
// contiguous slice of it and rebuilds its tables only when its slice crosses
// into the next unit; with fewer, every unit gets the same number of CTAs and
// each CTA a slice of one unit, so it builds its tables once. One
// producer thread streams 512-key tiles of records (and, when aligned, norms)
// with cp.async.bulk into a ring of shared-memory stages guarded by mbarriers;
// 16 consumer warps take 32 keys each per tile (one key per lane). Every wait
// is bounded and reports a timeout through the workspace status word.
//
// Shared-memory layout. The tables of query head q start at the 64 KB-aligned
// shared address T0 + q * 64 KB; the stage slots fill the space below T0 and
// after the last table. With the table base aligned, a lookup address is
// formed by bit operations alone (no add), and the per-query offset is the
// load's immediate.
//
// Tables. An index key is the codes of g consecutive coordinates as they sit
// in the code stream (g = 8, 4, 2 for 1, 2, 3 code bits: 8, 8 and 6 key
// bits); a d = 128 key has 16, 32 or 64 of them plus 16 sign bytes. Each table
// entry is the partial dot product of the query with that group.
//
// Byte keys (1 and 2 code bits): one table row per key value holds 64 words,
// positions 0..31 for the index tables and 32..63 for the sign tables (a
// 16-table set sits twice, at p and p + 16). At step s lane l reads position
// p = s XOR l, so the 32 lanes hit 32 different banks whatever the key values.
// The lane first permutes its record words by XOR with l/4 (a few selects,
// shared by every query head of the group); the byte of key p is then picked
// by one byte-permute whose selector depends only on l mod 4 and s mod 4, and
// lands already shifted into the row field, merged with the table base's high
// bytes. A lookup is one byte-permute, one three-input logic op
// (row | (lane ^ step)), one shared load and one add.
//
// 6-bit keys (3 code bits): 64 tables of 64 entries in two groups of 32 (row
// stride 32 words), and the 16 sign tables in their own rows (twice, rows of
// 32 words). At step s lane l reads position (s + l) mod 32 after rotating its
// record so that key (s + l) sits at static position s.
#include "common.cuh"

namespace tq {

namespace {

constexpr int kFD = 128;                       // head dimension of this kernel
constexpr int kFConsumers = 16;                // consumer warps
constexpr int kFThreads = 32 * (kFConsumers + 1);
constexpr int kFTile = 32 * kFConsumers;       // keys per stage
constexpr int kFMaxStages = 8;
constexpr uint32_t kTabStride = 0x10000;       // shared bytes per query head's tables (64 KB)
constexpr uint32_t kBarBytes = 2 * kFMaxStages * 8;
constexpr uint32_t kQStage = 2048;                     // shared bytes for the staged Pi q and S q of 2 query heads
static_assert(kFTile % 64 == 0, "table builds walk key values with a stride of kFTile / 64");

template <int BETA>
struct FastKeys {
  static constexpr int IW = BETA * kFD / 32;               // code-stream words
  static constexpr int RW = IW + kFD / 32;                 // record words
  static constexpr int NI = BETA == 1 ? 16 : BETA == 2 ? 32 : 64;   // index keys per record
  static constexpr int G = BETA == 3 ? 2 : 8 / BETA;       // coordinates per index key
  static constexpr uint32_t kStageBytes = kFTile * (RW + 2) * 4;
};

struct FastParams {
  LogitsParams p;
  int tiles_per_unit;
  int ctas_per_unit;       // > 0: CTA b scans part b % ctas_per_unit of unit b / ctas_per_unit
  int64_t total_tiles;
  uint32_t dyn_bytes;      // dynamic shared memory of the launch
};


template <uint32_t OFF>
__device__ __forceinline__ float lds_at(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(OFF));
  return v;
}

// Rotate an n-word cyclic bit stream right by `rb` bits (0 <= rb < 32 n):
// out bit k = in bit (k + rb) mod 32n.
template <int N>
__device__ __forceinline__ void rotate_stream(uint32_t (&w)[N], int rb) {
  const int wofs = rb >> 5, boff = rb & 31;
#pragma unroll
  for (int bit = 1; bit < N; bit <<= 1) {
    uint32_t t[N];
    const bool take = (wofs & bit) != 0;
#pragma unroll
    for (int j = 0; j < N; ++j) t[j] = take ? w[(j + bit) % N] : w[j];
#pragma unroll
    for (int j = 0; j < N; ++j) w[j] = t[j];
  }
  uint32_t t[N];
#pragma unroll
  for (int j = 0; j < N; ++j) t[j] = __funnelshift_r(w[j], w[(j + 1) % N], boff);
#pragma unroll
  for (int j = 0; j < N; ++j) w[j] = t[j];
}

// Permute N words by XOR of their index with c (N a power of two, c < N).
template <int N>
__device__ __forceinline__ void xor_permute(uint32_t (&w)[N], int c) {
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

// Key of KB bits at bit `pos` of a rotated stream, shifted to bit 7 (rows of 32
// words) and merged with `bank` (table base | position offset).
template <int KB, int N>
__device__ __forceinline__ uint32_t key_addr7(const uint32_t (&r)[N], int pos, uint32_t bank) {
  const int w = pos >> 5, b = pos & 31;
  uint32_t v;
  int at;
  if (b + KB <= 32) {
    v = r[w];
    at = b;
  } else {
    v = __funnelshift_r(r[w], r[(w + 1) % N], b);
    at = 0;
  }
  const uint32_t shifted = at >= 7 ? (v >> (at - 7)) : (v << (7 - at));
  constexpr uint32_t mask = ((1u << KB) - 1u) << 7;
  return (shifted & mask) | bank;
}

// One query head's logit for a byte-key record (1 or 2 code bits), tables at
// T0 + QQ * 64 KB. xi[m] / xs[m] hold, per lane, the table-base bytes 2..3 and
// the row positions (l ^ s) * 4 of steps s = 2m and 2m + 1 in bytes 0 and 1, so
// one byte-permute yields the whole address T0 | key << 8 | position.
template <int BETA, int QQ>
__device__ __forceinline__ float scan_bytes(const uint32_t (&wi)[BETA * 4], const uint32_t (&wsg)[4],
                                            const uint32_t (&sel)[4], const uint32_t (&xi)[BETA * 8],
                                            const uint32_t (&xs)[8], float nrm, float rho) {
  constexpr int NI = BETA == 1 ? 16 : 32;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
  for (int st = 0; st < NI; ++st) {
    const float v = lds_at<QQ * kTabStride>(__byte_perm(wi[st >> 2], xi[st >> 1], sel[st & 3]));
    if ((st & 3) == 0) a0 += v;
    else if ((st & 3) == 1) a1 += v;
    else if ((st & 3) == 2) a2 += v;
    else a3 += v;
  }
#pragma unroll
  for (int st = 0; st < 16; ++st) {
    const float v = lds_at<QQ * kTabStride>(__byte_perm(wsg[st >> 2], xs[st >> 1], sel[st & 3]));
    if (st & 1) b1 += v;
    else b0 += v;
  }
  return nrm * fmaf(rho, b0 + b1, (a0 + a1) + (a2 + a3));
}

// One query head's logit for a 3-bit-code record (rotated halves lo/hi and sign stream rs).
template <int QQ>
__device__ __forceinline__ float scan_six(const uint32_t (&lo)[6], const uint32_t (&hi)[6], const uint32_t (&rs)[4],
                                          const uint32_t (&bank)[32], float nrm, float rho) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
  for (int st = 0; st < 32; ++st) {
    const float v = lds_at<QQ * kTabStride>(key_addr7<6>(lo, 6 * st, bank[st]));
    if (st & 1) a1 += v;
    else a0 += v;
  }
#pragma unroll
  for (int st = 0; st < 32; ++st) {
    const float v = lds_at<QQ * kTabStride + 8192>(key_addr7<6>(hi, 6 * st, bank[st]));
    if (st & 1) a3 += v;
    else a2 += v;
  }
#pragma unroll
  for (int st = 0; st < 16; ++st) {
    const float v = lds_at<QQ * kTabStride + 32768>(key_addr7<8>(rs, 8 * st, bank[st]));
    if (st & 1) b1 += v;
    else b0 += v;
  }
  return nrm * fmaf(rho, b0 + b1, (a0 + a1) + (a2 + a3));
}

template <int BETA, int QMAX>
__global__ void __launch_bounds__(kFThreads, 1) logits_fast_kernel(const FastParams fp) {
  using K = FastKeys<BETA>;
  constexpr int RW = K::RW, IW = K::IW;
  constexpr uint32_t SB = K::kStageBytes;
  const LogitsParams &p = fp.p;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float cbs[8];

  // ---- layout in the shared window ----
  const uint32_t dyn0 = smem_u32(smem);
  const uint32_t dyn_end = dyn0 + fp.dyn_bytes;
  const uint32_t T0 = (dyn0 + kBarBytes + kTabStride - 1) & ~(kTabStride - 1);
  const uint32_t a0 = dyn0 + kBarBytes;                  // first stage slot below the tables
  const uint32_t qst = T0 - kQStage;                     // staged query projections, just below the tables
  const int n_a = (int)((qst - a0) / SB);
  const uint32_t b0 = T0 + QMAX * kTabStride;            // slots after the tables
  const int n_b = b0 < dyn_end ? (int)((dyn_end - b0) / SB) : 0;
  const int stages = min(kFMaxStages, n_a + n_b);
  auto slot = [&](int s) -> uint32_t { return s < n_a ? a0 + (uint32_t)s * SB : b0 + (uint32_t)(s - n_a) * SB; };
  const uint32_t bar0 = dyn0;                            // full[8], empty[8]
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kFMaxStages + s); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (stages < 2 || T0 + QMAX * kTabStride > dyn_end) {
    if (tid == 0) {
      pdl_wait();   // the query projection clears the status word first
      atomicOr(p.status, kDevBadShape);   // the launch's shared memory cannot hold this layout
    }
    return;
  }
  int64_t g0, g1;
  if (fp.ctas_per_unit > 0) {
    const int unit = blockIdx.x / fp.ctas_per_unit, part = blockIdx.x - unit * fp.ctas_per_unit;
    const int64_t base = (int64_t)unit * fp.tiles_per_unit;
    g0 = base + (int64_t)part * fp.tiles_per_unit / fp.ctas_per_unit;
    g1 = base + (int64_t)(part + 1) * fp.tiles_per_unit / fp.ctas_per_unit;
  } else {
    const int64_t per_cta = (fp.total_tiles + gridDim.x - 1) / gridDim.x;
    g0 = (int64_t)blockIdx.x * per_cta;
    g1 = min(fp.total_tiles, g0 + per_cta);
  }
  if (g0 >= g1) return;
  const int n_my = (int)(g1 - g0);
  const int unit0 = (int)(g0 / fp.tiles_per_unit);
  const int tile0 = (int)(g0 - (int64_t)unit0 * fp.tiles_per_unit);

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kFConsumers);
    }
    mbar_fence_init();
  }
  if (tid < (1 << BETA)) cbs[tid] = p.codebook[tid];
  __syncthreads();

  auto norms_by_copy = [&](size_t first, int n) {
    return (n % 4 == 0) && (((uintptr_t)(p.norm + first)) % 16 == 0) && (((uintptr_t)(p.rnorm + first)) % 16 == 0);
  };

  if (warp == kFConsumers) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      int issued = 0, vunit = unit0, tile = tile0, s = 0;
      uint32_t phase = 1u;   // parity of the empty-barrier phase a stage's reuse waits for
      size_t unit_first = (size_t)(vunit / p.qblocks) * p.capacity;
      for (int i = 0; i < n_my; ++i) {
        if (i >= stages && !mbar_wait(empty_bar(s), phase)) {
          pdl_wait();
          atomicOr(p.status, kDevTimeout);
          break;
        }
        const int64_t t0 = (int64_t)tile * kFTile;
        const int n = (int)min((int64_t)kFTile, p.n_tokens - t0);
        const size_t first = unit_first + t0;
        const uint32_t rec_bytes = (uint32_t)n * RW * 4;
        const bool nc = norms_by_copy(first, n);
        mbar_arrive_expect_tx(full_bar(s), rec_bytes + (nc ? 8u * n : 0u));
        const uint32_t st = slot(s);
        bulk_g2s(st, p.records + first * RW, rec_bytes, full_bar(s));
        if (nc) {
          bulk_g2s(st + kFTile * RW * 4, p.norm + first, 4u * n, full_bar(s));
          bulk_g2s(st + kFTile * RW * 4 + kFTile * 4, p.rnorm + first, 4u * n, full_bar(s));
        }
        ++issued;
        if (++s == stages) {
          s = 0;
          phase ^= 1u;
        }
        if (++tile == fp.tiles_per_unit) {
          tile = 0;
          ++vunit;
          unit_first = (size_t)(vunit / p.qblocks) * p.capacity;
        }
      }
      // drain: every issued copy must land before the CTA exits
      for (int i = max(0, issued - stages); i < issued; ++i)
        if (!mbar_wait(full_bar(i % stages), (i / stages) & 1)) {
          pdl_wait();
          atomicOr(p.status, kDevTimeout);
          break;
        }
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  pdl_wait();   // the query projections (and a clean status word) come from the previous grid
  const float kappa = 1.2533141373155003f / (float)kFD;   // sqrt(pi/2)/d
  int vunit = unit0, tile = tile0, cur_unit = -1;
  int nq = 0, seq = 0, h0 = 0;
  size_t unit_first = 0;
  float *tables = reinterpret_cast<float *>(smem + (T0 - dyn0));
  // per-unit values, set at each table build: this unit's logits row, norm and rnorm
  // pointers, and whether its norms come with the tiles (tiles start 512 keys apart)
  float *lg_row = nullptr;
  const float *nrm_p = nullptr, *rho_p = nullptr;
  bool unit_nc = false;
  const int k = warp * 32 + lane;   // this lane's key in a tile
  int s = 0;                        // stage of key tile i, and its phase parity
  uint32_t phase = 0;

  for (int i = 0; i < n_my; ++i) {
    if (vunit != cur_unit) {
      // (re)build this unit's tables; all consumer warps take part
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kFConsumers) : "memory");
      cur_unit = vunit;
      const int qb = vunit % p.qblocks, sk = vunit / p.qblocks;
      unit_first = (size_t)sk * p.capacity;
      seq = sk / p.n_kv_heads;
      const int kvh = sk - seq * p.n_kv_heads;
      h0 = kvh * p.group + qb * p.q_per_cta;
      nq = min(p.q_per_cta, p.group - qb * p.q_per_cta);
      lg_row = p.logits + ((size_t)seq * p.n_q_heads + h0) * p.n_tokens;
      nrm_p = p.norm + unit_first;
      rho_p = p.rnorm + unit_first;
      unit_nc = (reinterpret_cast<uintptr_t>(nrm_p) % 16 == 0) && (reinterpret_cast<uintptr_t>(rho_p) % 16 == 0);
      float *qv = reinterpret_cast<float *>(smem + (qst - dyn0));   // [qq][Pi q | S q][128]
      for (int e = tid; e < nq * 2 * kFD; e += 32 * kFConsumers) {
        const int qq = e / (2 * kFD), r = e - qq * 2 * kFD;
        const size_t qrow = ((size_t)seq * p.n_q_heads + h0 + qq) * kFD;
        qv[e] = r < kFD ? p.qrot[qrow + r] : p.qsk[qrow + r - kFD];
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kFConsumers) : "memory");
      // Each thread keeps one table position (and so its few query values) in
      // registers and walks the key values with a stride of kFTile / width, so a
      // warp shares one key: codebook reads broadcast and stores hit 32 banks.
      for (int qq = 0; qq < nq; ++qq) {
        const float *qr = qv + qq * 2 * kFD, *qs = qr + kFD;
        float *tq_ = tables + (size_t)qq * (kTabStride / 4);
        if constexpr (BETA != 3) {
          // 256 rows of 64 words: [0, 32) index positions, [32, 64) sign positions
          const int pos = tid & 63;
          if (pos < 32) {
            const int t = pos & (K::NI - 1);
            float qc[K::G];
#pragma unroll
            for (int c = 0; c < K::G; ++c) qc[c] = qr[t * K::G + c];
            for (int key = tid >> 6; key < 256; key += kFTile / 64) {
              float v = 0.f;
#pragma unroll
              for (int c = 0; c < K::G; ++c) v = fmaf(qc[c], cbs[(key >> (BETA * c)) & ((1 << BETA) - 1)], v);
              tq_[key * 64 + pos] = v;
            }
          } else {
            const int t = pos & 15;
            float sv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) sv[c] = kappa * qs[8 * t + c];
            for (int key = tid >> 6; key < 256; key += kFTile / 64) {
              float v = 0.f;
#pragma unroll
              for (int c = 0; c < 8; ++c) v += ((key >> c) & 1) ? sv[c] : -sv[c];
              tq_[key * 64 + pos] = v;
            }
          }
        } else {
          // index: 2 groups x 64 rows x 32 words at +0; sign: 256 rows x 32 words at +32 KB
          {
            const int t = tid & 63;
            const float q0 = qr[2 * t], q1 = qr[2 * t + 1];
            float *row = tq_ + (t >> 5) * 64 * 32 + (t & 31);
            for (int key = tid >> 6; key < 64; key += kFTile / 64)
              row[key * 32] = fmaf(q1, cbs[(key >> 3) & 7], q0 * cbs[key & 7]);
          }
          {
            const int pos = tid & 31, t = pos & 15;
            float sv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) sv[c] = kappa * qs[8 * t + c];
            float *ts = tq_ + 8192;
            for (int key = tid >> 5; key < 256; key += kFTile / 32) {
              float v = 0.f;
#pragma unroll
              for (int c = 0; c < 8; ++c) v += ((key >> c) & 1) ? sv[c] : -sv[c];
              ts[key * 32 + pos] = v;
            }
          }
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kFConsumers) : "memory");
    }

    if (!mbar_wait(full_bar(s), phase)) {
      atomicOr(p.status, kDevTimeout);
      return;
    }
    const int64_t t0 = (int64_t)tile * kFTile;
    const int n = (int)min((int64_t)kFTile, p.n_tokens - t0);
    const bool valid = k < n;
    const unsigned char *st = smem + (slot(s) - dyn0);
    uint32_t w[RW];
    if (valid) {
      const uint4 *src = reinterpret_cast<const uint4 *>(st + (size_t)k * RW * 4);
#pragma unroll
      for (int j = 0; j < RW / 4; ++j) {
        const uint4 v = src[j];
        w[4 * j] = v.x;
        w[4 * j + 1] = v.y;
        w[4 * j + 2] = v.z;
        w[4 * j + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < RW; ++j) w[j] = 0u;
    }
    float nrm = 0.f, rho = 0.f;
    if (valid) {
      if (unit_nc && (n & 3) == 0) {   // the producer's condition (norms_by_copy) for this tile
        nrm = reinterpret_cast<const float *>(st + kFTile * RW * 4)[k];
        rho = reinterpret_cast<const float *>(st + kFTile * RW * 4 + kFTile * 4)[k];
      } else {
        nrm = __ldg(nrm_p + t0 + k);
        rho = __ldg(rho_p + t0 + k);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));   // this warp is done with the stage
    if (++s == stages) {
      s = 0;
      phase ^= 1u;
    }

    float out[QMAX];
#pragma unroll
    for (int qq = 0; qq < QMAX; ++qq) out[qq] = 0.f;
    if constexpr (BETA != 3) {
      // byte-permute selectors for step s (j = s mod 4): result byte 0 = position byte
      // (s mod 2) of the x register, byte 1 = key byte (j ^ (l & 3)) of the record
      // word, bytes 2..3 = table-base bytes 2..3 of the x register
      uint32_t sel[4];
      const uint32_t sel0 = 0x7604u | ((uint32_t)(lane & 3) << 4);
#pragma unroll
      for (int j = 0; j < 4; ++j) sel[j] = sel0 ^ ((uint32_t)(j & 1) | ((uint32_t)j << 4));
      const uint32_t xi0 = (T0 & 0xFFFF0000u) | ((uint32_t)lane << 2) | ((uint32_t)(lane ^ 1) << 10);
      const uint32_t xs0 = xi0 | 0x8080u;
      uint32_t xi[BETA * 8], xs[8];
#pragma unroll
      for (int m = 0; m < BETA * 8; ++m) xi[m] = xi0 ^ ((uint32_t)m * 0x808u);
#pragma unroll
      for (int m = 0; m < 8; ++m) xs[m] = xs0 ^ ((uint32_t)m * 0x808u);
      uint32_t wi[IW], wsg[4];
#pragma unroll
      for (int j = 0; j < IW; ++j) wi[j] = w[j];
#pragma unroll
      for (int j = 0; j < 4; ++j) wsg[j] = w[IW + j];
      xor_permute<IW>(wi, (lane >> 2) & (IW - 1));
      xor_permute<4>(wsg, (lane >> 2) & 3);
      out[0] = scan_bytes<BETA, 0>(wi, wsg, sel, xi, xs, nrm, rho);
      if constexpr (QMAX > 1)
        if (nq > 1) out[1] = scan_bytes<BETA, 1>(wi, wsg, sel, xi, xs, nrm, rho);
    } else {
      uint32_t bank[32];   // T0 | position offset ((s + l) mod 32, times 4)
#pragma unroll
      for (int s2 = 0; s2 < 32; ++s2) bank[s2] = T0 | (uint32_t)(((s2 + lane) & 31) << 2);
      uint32_t lo[6], hi[6], rs[4];
#pragma unroll
      for (int j = 0; j < 6; ++j) { lo[j] = w[j]; hi[j] = w[6 + j]; }
#pragma unroll
      for (int j = 0; j < 4; ++j) rs[j] = w[12 + j];
      rotate_stream<6>(lo, 6 * lane);
      rotate_stream<6>(hi, 6 * lane);
      rotate_stream<4>(rs, 8 * (lane & 15));
      out[0] = scan_six<0>(lo, hi, rs, bank, nrm, rho);
      if constexpr (QMAX > 1)
        if (nq > 1) out[1] = scan_six<1>(lo, hi, rs, bank, nrm, rho);
    }
    if (valid) {
#pragma unroll
      for (int qq = 0; qq < QMAX; ++qq)
        if (qq < nq) lg_row[qq * p.n_tokens + t0 + k] = out[qq];
    }
    if (++tile == fp.tiles_per_unit) {
      tile = 0;
      ++vunit;
    }
  }
}

// Dynamic shared memory for QMAX query heads' tables with dynamic smem starting
// at `dyn0` (the reserved region below it): the aligned table block plus as many
// stage slots as fit, capped by the opt-in limit.
template <int BETA>
uint32_t fast_dyn_bytes(int qmax, uint32_t limit, int *stages_out) {
  using K = FastKeys<BETA>;
  const uint32_t dyn0 = 1024;   // reserved shared memory below the dynamic window on sm_100
  const uint32_t T0 = (dyn0 + kBarBytes + kTabStride - 1) & ~(kTabStride - 1);
  const uint32_t n_a = (T0 - kQStage - dyn0 - kBarBytes) / K::kStageBytes;
  const uint32_t b0 = T0 + qmax * kTabStride;
  const uint32_t dyn_end = dyn0 + limit;
  const uint32_t n_b = b0 < dyn_end ? (dyn_end - b0) / K::kStageBytes : 0;
  int stages = (int)(n_a + n_b);
  if (stages > kFMaxStages) stages = kFMaxStages;
  *stages_out = stages;
  // bytes up to the end of the last slot used
  uint32_t end = b0;
  if ((uint32_t)stages > n_a) end = b0 + (stages - n_a) * K::kStageBytes;
  return end - dyn0;
}

template <int BETA, int QMAX>
cudaError_t launch_fast(const LogitsParams &p, int n_seq, uint32_t limit, cudaStream_t st) {
  FastParams fp{};
  fp.p = p;
  fp.tiles_per_unit = (int)((p.n_tokens + kFTile - 1) / kFTile);
  fp.total_tiles = (int64_t)n_seq * p.n_kv_heads * p.qblocks * fp.tiles_per_unit;
  int stages = 0;
  fp.dyn_bytes = fast_dyn_bytes<BETA>(QMAX, limit, &stages);
  auto kern = logits_fast_kernel<BETA, QMAX>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), fp.dyn_bytes);
  if (e != cudaSuccess) return e;
  // Two splits over one CTA per SM, costed in tiles of the busiest CTA, a table
  // build counting as kTableTiles: contiguous slices of the tile list (a slice
  // may cross into a second unit and build twice), or, with fewer units than
  // SMs, the same whole number of CTAs per unit (one build each, but some SMs
  // may idle).
  constexpr int64_t kTableTiles = 3;
  if (fp.total_tiles <= 0) return cudaSuccess;
  const int64_t slots = device_sm_count();
  const int64_t units = fp.tiles_per_unit > 0 ? fp.total_tiles / fp.tiles_per_unit : 0;
  const int64_t cpu = units > 0 ? (slots / units < fp.tiles_per_unit ? slots / units : fp.tiles_per_unit) : 0;
  const int64_t cost_aligned = cpu > 0 ? (fp.tiles_per_unit + cpu - 1) / cpu + kTableTiles : INT64_MAX;
  const int64_t per_slice = (fp.total_tiles + slots - 1) / slots;
  const int64_t cost_slices = per_slice + (per_slice < fp.tiles_per_unit ? 2 : 1 + per_slice / fp.tiles_per_unit) * kTableTiles;
  int64_t grid;
  if (units > 0 && units < slots && cost_aligned < cost_slices) {
    fp.ctas_per_unit = (int)cpu;
    grid = units * cpu;
  } else {
    fp.ctas_per_unit = 0;
    grid = fp.total_tiles < slots ? fp.total_tiles : slots;
  }
  // Launched as a programmatic dependent of the query projection: the producer
  // starts streaming keys (written by earlier grids, not by that one) while the
  // projection runs; consumers wait for it before building tables.
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = fp.dyn_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, fp);
}

}  // namespace

// Stage slots the d = 128 scan gets for `q` query heads per CTA within `limit`
// bytes of dynamic shared memory (0 if the tables do not fit).
int logits_fast_stages(int bits, int q, size_t limit) {
  int stages = 0;
  const uint32_t lim = (uint32_t)limit;
  switch (bits) {
    case 1: fast_dyn_bytes<1>(q, lim, &stages); break;
    case 2: fast_dyn_bytes<2>(q, lim, &stages); break;
    default: fast_dyn_bytes<3>(q, lim, &stages); break;
  }
  const uint32_t need = 65536 * (uint32_t)(q + 1);   // aligned table block inside the window
  return need <= lim + 1024 ? stages : 0;
}

cudaError_t launch_logits_fast(const LogitsParams &p, int bits, int n_seq, size_t limit, cudaStream_t st) {
  const int q = p.q_per_cta;
  const uint32_t lim = (uint32_t)limit;
  switch (bits) {
    case 1: return q == 1 ? launch_fast<1, 1>(p, n_seq, lim, st) : launch_fast<1, 2>(p, n_seq, lim, st);
    case 2: return q == 1 ? launch_fast<2, 1>(p, n_seq, lim, st) : launch_fast<2, 2>(p, n_seq, lim, st);
    default: return q == 1 ? launch_fast<3, 1>(p, n_seq, lim, st) : launch_fast<3, 2>(p, n_seq, lim, st);
  }
}

}  // namespace tq
