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
// after the last table. The tables, their layout and the per-key lookups are
// those of scan_core.cuh.
#include "scan_core.cuh"

namespace tq {

namespace {

using scan::kFD;
using scan::kTabStride;
constexpr int kFConsumers = 16;                // consumer warps
constexpr int kFThreads = 32 * (kFConsumers + 1);
constexpr int kFTile = 32 * kFConsumers;       // keys per stage
constexpr int kFMaxStages = 8;
constexpr uint32_t kBarBytes = 2 * kFMaxStages * 8;
constexpr uint32_t kQStage = 2048;                     // shared bytes for the staged Pi q and S q of 2 query heads

// Record words and stage bytes; MIXED: the mixed-rate record (scan::MixedKeys), whose 40 or 56 bytes
// are not a multiple of 16: a tile with an odd number of keys gets its last record by plain loads.
template <int BETA, bool MIXED = false>
struct FastKeys {
  static constexpr int RW = MIXED ? scan::MixedKeys<BETA>::RW : scan::FastKeys<BETA>::RW;
  static constexpr uint32_t kStageBytes = kFTile * (RW + 2) * 4;
};

struct FastParams {
  LogitsParams p;
  int tiles_per_unit;
  int ctas_per_unit;       // > 0: CTA b scans part b % ctas_per_unit of unit b / ctas_per_unit
  int64_t total_tiles;
  uint32_t dyn_bytes;      // dynamic shared memory of the launch
};


template <int BETA, int QMAX, bool MIXED>
__global__ void __launch_bounds__(kFThreads, 1) logits_fast_kernel(const FastParams fp) {
  using K = FastKeys<BETA, MIXED>;
  constexpr int RW = K::RW;
  constexpr uint32_t SB = K::kStageBytes;
  const LogitsParams &p = fp.p;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float cbs[24];   // the codebook (mixed: the narrow one, then the wide one)

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
  if (tid < (1 << BETA) + (MIXED ? 2 << BETA : 0)) cbs[tid] = p.codebook[tid];
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
        const uint32_t st = slot(s);
        int ncopy = n;
        if (MIXED && (n & 1)) {
          // the last record by plain loads (before the arrival that completes the stage), the rest by copy
          --ncopy;
          const uint32_t *src = p.records + (first + ncopy) * RW;
          uint32_t *dst = reinterpret_cast<uint32_t *>(smem + (st - dyn0)) + (size_t)ncopy * RW;
#pragma unroll
          for (int w = 0; w < RW; ++w) dst[w] = __ldg(src + w);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // ordered with the copy engine's writes
        }
        const uint32_t rec_bytes = (uint32_t)ncopy * RW * 4;
        const bool nc = norms_by_copy(first, n);
        mbar_arrive_expect_tx(full_bar(s), rec_bytes + (nc ? 8u * n : 0u));
        if (rec_bytes > 0) bulk_g2s(st, p.records + first * RW, rec_bytes, full_bar(s));
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
      for (int qq = 0; qq < nq; ++qq) {
        const float *qr = qv + qq * 2 * kFD;
        if constexpr (MIXED)
          scan::build_tables_mixed<BETA, kFTile>(qr, qr + kFD, tables + (size_t)qq * (kTabStride / 4), cbs,
                                                 cbs + (1 << BETA), tid, kappa);
        else
          scan::build_tables<BETA, kFTile>(qr, qr + kFD, tables + (size_t)qq * (kTabStride / 4), cbs, tid, kappa);
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
    // this lane's record, read whether or not the key exists: slots past n hold stale words whose
    // logits are never stored, so the load needs no branch
    uint32_t w[RW];
    if constexpr (RW % 4 == 0) {
      const uint4 *src = reinterpret_cast<const uint4 *>(st + (size_t)k * RW * 4);
#pragma unroll
      for (int j = 0; j < RW / 4; ++j) {
        const uint4 v = src[j];
        w[4 * j] = v.x;
        w[4 * j + 1] = v.y;
        w[4 * j + 2] = v.z;
        w[4 * j + 3] = v.w;
      }
    } else {   // mixed records: 8-byte aligned
      const uint2 *src = reinterpret_cast<const uint2 *>(st + (size_t)k * RW * 4);
#pragma unroll
      for (int j = 0; j < RW / 2; ++j) {
        const uint2 v = src[j];
        w[2 * j] = v.x;
        w[2 * j + 1] = v.y;
      }
    }
    float nrm, rho;
    if (unit_nc && (n & 3) == 0) {   // the producer's condition (norms_by_copy) for this tile
      nrm = reinterpret_cast<const float *>(st + kFTile * RW * 4)[k];
      rho = reinterpret_cast<const float *>(st + kFTile * RW * 4 + kFTile * 4)[k];
    } else {
      nrm = valid ? __ldg(nrm_p + t0 + k) : 0.f;
      rho = valid ? __ldg(rho_p + t0 + k) : 0.f;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));   // this warp is done with the stage
    if (++s == stages) {
      s = 0;
      phase ^= 1u;
    }

    float out[QMAX];
    if constexpr (MIXED) scan::key_logits_mixed<BETA, QMAX>(w, lane, T0, nq, nrm, rho, out);
    else scan::key_logits<BETA, QMAX>(w, lane, T0, nq, nrm, rho, out);
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
template <int BETA, bool MIXED = false>
uint32_t fast_dyn_bytes(int qmax, uint32_t limit, int *stages_out) {
  using K = FastKeys<BETA, MIXED>;
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

template <int BETA, int QMAX, bool MIXED = false>
cudaError_t launch_fast(const LogitsParams &p, int n_seq, uint32_t limit, cudaStream_t st) {
  FastParams fp{};
  fp.p = p;
  fp.tiles_per_unit = (int)((p.n_tokens + kFTile - 1) / kFTile);
  fp.total_tiles = (int64_t)n_seq * p.n_kv_heads * p.qblocks * fp.tiles_per_unit;
  int stages = 0;
  fp.dyn_bytes = fast_dyn_bytes<BETA, MIXED>(QMAX, limit, &stages);
  auto kern = logits_fast_kernel<BETA, QMAX, MIXED>;
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
// bytes of dynamic shared memory (0 if the tables do not fit); n_hi = 64: the
// mixed-rate records (bits 1 or 2).
int logits_fast_stages(int bits, int q, size_t limit, int n_hi) {
  int stages = 0;
  const uint32_t lim = (uint32_t)limit;
  if (n_hi == 64) {
    if (bits == 1) fast_dyn_bytes<1, true>(q, lim, &stages);
    else fast_dyn_bytes<2, true>(q, lim, &stages);
  } else {
    switch (bits) {
      case 1: fast_dyn_bytes<1>(q, lim, &stages); break;
      case 2: fast_dyn_bytes<2>(q, lim, &stages); break;
      default: fast_dyn_bytes<3>(q, lim, &stages); break;
    }
  }
  const uint32_t need = 65536 * (uint32_t)(q + 1);   // aligned table block inside the window
  return need <= lim + 1024 ? stages : 0;
}

cudaError_t launch_logits_fast(const LogitsParams &p, int bits, int n_seq, size_t limit, cudaStream_t st) {
  const int q = p.q_per_cta;
  const uint32_t lim = (uint32_t)limit;
  if (p.n_hi == 64) {
    if (bits == 1) return q == 1 ? launch_fast<1, 1, true>(p, n_seq, lim, st) : launch_fast<1, 2, true>(p, n_seq, lim, st);
    return q == 1 ? launch_fast<2, 1, true>(p, n_seq, lim, st) : launch_fast<2, 2, true>(p, n_seq, lim, st);
  }
  switch (bits) {
    case 1: return q == 1 ? launch_fast<1, 1>(p, n_seq, lim, st) : launch_fast<1, 2>(p, n_seq, lim, st);
    case 2: return q == 1 ? launch_fast<2, 1>(p, n_seq, lim, st) : launch_fast<2, 2>(p, n_seq, lim, st);
    default: return q == 1 ? launch_fast<3, 1>(p, n_seq, lim, st) : launch_fast<3, 2>(p, n_seq, lim, st);
  }
}

}  // namespace tq
