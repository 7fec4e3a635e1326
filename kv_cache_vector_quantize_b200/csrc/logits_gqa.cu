// Logit scan for grouped-query attention on d = 128 keys with 1 or 2 code bits
// per coordinate (byte-wide lookup keys) and 2, 4 or 8 query heads per KV head.
//
// Estimator (usedby.ai, "TurboQuant: Compresion de KV Cache a 3 bits y
// aceleracion de inferencia en H100", "El Pitch"; winningdata.io, "TurboQuant:
// Google comprime KV cache para 3 bits sem perder acuracia", "2. QJL
// Residual"):
//   l_t = n_t ( <Pi q, c[code_t]> + rho_t sqrt(pi/2)/d <S q, 2 sign_t - 1> ).
//
// A KV head's keys are shared by its query heads, so one CTA scans them for up
// to four heads at once (QH heads; a "unit" is a sequence, a KV head and a
// block of QH of its query heads). Both inner products are sums over byte-wide
// groups of the record (the codes of 8/bits coordinates, or 8 sign bits), so
// each head's query becomes lookup tables with one entry per (byte position,
// byte value), and a key costs one table read per record byte.
//
// Tables. Entries are float16, divided by a per-head scale sigma = ||q|| (1 for
// a zero query) so that they are O(1/sqrt(d)); the entries of the QH heads of
// a unit for one (position, byte) sit side by side (8 bytes for four heads), so
// one 64-bit shared load serves all four heads. Partial sums run in float16
// pairs over at most 16 reads and are then added into float32 (the rounding of
// both stays about 40 standard deviations below the 2e-3 |q| |k| tolerance on
// Gaussian data). A unit's block is 128 KB: an index half (row = byte value,
// 32 positions of 8 bytes; 1-bit codes have 16 byte positions, stored twice)
// and a sign half (16 sign bytes, stored twice). It is built once per call by
// gqa_tables_kernel in the workspace and copied into shared memory by each CTA
// of the unit with bulk copies.
//
// Scan. As in the single-head scan: one producer thread streams 512-key tiles
// of records (and norms) into a ring of shared-memory stages; 16 consumer
// warps take 32 keys each (one key per lane). At step s lane l reads position
// s XOR l, so a half-warp's 16 loads hit 16 different bank pairs whatever the
// byte values; the address is one byte-permute of the (XOR-permuted) record
// word with a per-lane constant that holds the 64 KB-aligned table base and
// the position.
#include <cuda_fp16.h>

#include "common.cuh"
#include "gqa_core.cuh"

namespace tq {

namespace {

using namespace gqa;

constexpr int kGConsumers = 16;
constexpr int kGThreads = 32 * (kGConsumers + 1);
constexpr int kGTile = 32 * kGConsumers;        // keys per stage
constexpr int kGMaxStages = 6;
constexpr uint32_t kGBarBytes = 128;             // full[6], empty[6], table barrier; keeps the stage ring 16-byte aligned
static_assert(kGBarBytes >= 8 * (2 * kGMaxStages + 1) && kGBarBytes % 16 == 0, "stage slots must start 16-byte aligned");

// bytes of one scan stage: a tile's records, then its norms and residual norms
template <int BETA>
struct GStage {
  static constexpr uint32_t kBytes = kGTile * (GKeys<BETA>::RW + 2) * 4;
  static_assert(kBytes % 16 == 0 && (kGTile * GKeys<BETA>::RW * 4) % 16 == 0, "bulk copies need 16-byte offsets");
};

// ------------------------------------------------------------------------
// tables: grid (units, 2 halves, 4 parts); part k fills byte positions
// [8k, 8k + 8) of its half for all 256 byte values and all QH heads. A byte's
// entry is the sum of two 16-entry nibble tables, so an entry costs one add.
// ------------------------------------------------------------------------
template <int BETA, int QH>
__global__ void __launch_bounds__(256) gqa_tables_kernel(GqaParams g) {
  using K = GKeys<BETA>;
  constexpr int L = 1 << BETA;
  __shared__ __align__(16) float qs[QH][kGD];   // the unit's queries (read as float4)
  __shared__ float proj[QH][64];                 // projections of the coordinates this part needs, / sigma
  __shared__ float nib[8][2][QH][16];            // per position: sums over the low / high nibble of a byte
  __shared__ float sig[QH];
  __shared__ float cbs[16];
  const int unit = blockIdx.x, half = blockIdx.y, part = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int qb = unit % g.qblocks, sk = unit / g.qblocks;
  const int seq = sk / g.n_kv_heads, kvh = sk - seq * g.n_kv_heads;
  const int h0 = kvh * g.group + qb * QH;
  pdl_wait();   // launched as a dependent of the previous work: it must be finished first
  if (unit == 0 && half == 0 && part == 0 && tid == 0) *g.status = 0u;   // this call reports into a clean word
  pdl_launch_dependents();   // the scan may start streaming keys; it waits for this grid before its tables
  // coordinates of byte positions [8 part, 8 part + 8): index bytes of 1-bit codes and sign bytes
  // repeat every 16 positions, so a part covers 32 or 64 coordinates starting at c0
  const int per_byte = half == 0 ? K::G : 8;
  const int nbytes = half == 0 ? K::NI : 16;
  const int c0 = ((8 * part) % nbytes) * per_byte;
  const int ncoord = 8 * per_byte;
  const float *M = half == 0 ? g.Pi : g.S;
  const float scale = half == 0 ? 1.f : 1.2533141373155003f / (float)kGD;   // sqrt(pi/2)/d on the sign half
  // matrix rows first (one warp per row, a coalesced 512-byte read each), so their latency overlaps the query loads
  constexpr int kRowsPerWarp = 8;   // 64 rows / 8 warps
  float4 mv[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int cl = warp * kRowsPerWarp + r;
    mv[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (cl < ncoord)   // volatile: issued here, ahead of the query loads and the barriers
      asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                   : "=f"(mv[r].x), "=f"(mv[r].y), "=f"(mv[r].z), "=f"(mv[r].w)
                   : "l"(reinterpret_cast<const float4 *>(M + (size_t)(c0 + cl) * kGD) + lane));
  }
  for (int e = tid; e < QH * kGD; e += 256) qs[e / kGD][e % kGD] = g.q[((size_t)seq * g.n_q_heads + h0) * kGD + e];
  if (tid < L) cbs[tid] = g.codebook[tid];
  __syncthreads();
  // sigma = ||q|| in a fixed order (warp h: lane sums 4 consecutive values, then a butterfly)
  if (warp < QH) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) s = fmaf(qs[warp][4 * lane + c], qs[warp][4 * lane + c], s);
    s = warp_sum(s);
    if (lane == 0) {
      const float n = sqrtf(s);
      sig[warp] = n > 0.f ? n : 1.f;
      if (half == 0 && part == 0) g.sigma[(size_t)seq * g.n_q_heads + h0 + warp] = sig[warp];
    }
  }
  __syncthreads();
  {
    // partial dot products of this warp's 8 rows with the QH queries (lane: 4 coordinates), then a
    // reduce-scatter butterfly: after it lane l holds the full sum of (row l / QH, head l % QH)
    float4 qv[QH];
#pragma unroll
    for (int h = 0; h < QH; ++h) qv[h] = *reinterpret_cast<const float4 *>(&qs[h][4 * lane]);
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int r = i / QH, h = i % QH;
      v[i] = r < kRowsPerWarp
                 ? fmaf(mv[r].x, qv[h].x, fmaf(mv[r].y, qv[h].y, fmaf(mv[r].z, qv[h].z, mv[r].w * qv[h].w)))
                 : 0.f;
    }
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
      const bool up = (lane & k) != 0;
#pragma unroll
      for (int i = 0; i < k; ++i) {
        const float send = up ? v[i] : v[i + k];
        const float keep = up ? v[i + k] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
      }
    }
    const int r = lane / QH, h = lane % QH, cl = warp * kRowsPerWarp + r;
    if (r < kRowsPerWarp && cl < ncoord) proj[h][cl] = scale * v[0] / sig[h];
  }
  __syncthreads();
  // nibble sums: a byte's entry is the sum over its low nibble plus the sum over its high nibble
  // (index bytes: 4/BETA coordinates per nibble, their codes; sign bytes: 4 bits, +-)
  for (int e = tid; e < 8 * 2 * QH * 16; e += 256) {
    const int v = e & 15, h = (e >> 4) % QH, hi = (e / (16 * QH)) & 1, pp = e / (32 * QH);
    const int p = 8 * part + pp;
    const int cb0 = (p % nbytes) * per_byte - c0 + hi * (per_byte / 2);   // first coordinate of the nibble
    float s = 0.f;
    if (half == 0) {
      constexpr int kPer = 4 / BETA;   // coordinates per nibble
#pragma unroll
      for (int c = 0; c < kPer; ++c) s = fmaf(proj[h][cb0 + c], cbs[(v >> (BETA * c)) & (L - 1)], s);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) s += ((v >> c) & 1) ? proj[h][cb0 + c] : -proj[h][cb0 + c];
    }
    nib[pp][hi][h][v] = s;
  }
  __syncthreads();
  // entries: thread -> (byte value b, position p); 8 positions x 256 values
  unsigned char *blk = g.tables + (size_t)unit * (2 * kGHalf) + (size_t)half * kGHalf;
  for (int e = tid; e < 8 * 256; e += 256) {
    const int b = e >> 3, pp = e & 7, p = 8 * part + pp;
    __half hv[QH];
#pragma unroll
    for (int h = 0; h < QH; ++h) hv[h] = __float2half_rn(nib[pp][0][h][b & 15] + nib[pp][1][h][b >> 4]);
    // row b: 256 bytes; 4-head entries are 8 bytes at 8 p, 2-head entries 4 bytes at 4 p
    unsigned char *dst = blk + (size_t)b * 256 + (size_t)p * (2 * QH);
    if constexpr (QH == 4) {
      *reinterpret_cast<uint2 *>(dst) = make_uint2(
          (uint32_t)__half_as_ushort(hv[0]) | ((uint32_t)__half_as_ushort(hv[1]) << 16),
          (uint32_t)__half_as_ushort(hv[2]) | ((uint32_t)__half_as_ushort(hv[3]) << 16));
    } else {
      *reinterpret_cast<uint32_t *>(dst) = (uint32_t)__half_as_ushort(hv[0]) | ((uint32_t)__half_as_ushort(hv[1]) << 16);
    }
  }
}

// ------------------------------------------------------------------------
// scan
// ------------------------------------------------------------------------
struct GScan {
  LogitsParams p;
  const unsigned char *tables;   // units x 128 KB
  const float *sigma;            // [n_seq][n_q_heads]
  int tiles_per_unit;
  int ctas_per_unit;
  uint32_t dyn_bytes;
};

template <int BETA, int QH>
__global__ void __launch_bounds__(kGThreads, 1) logits_gqa_kernel(const GScan gs) {
  using K = GKeys<BETA>;
  constexpr int RW = K::RW, IW = K::IW;
  constexpr uint32_t SB = GStage<BETA>::kBytes;
  constexpr uint32_t ESZ = 2 * QH;                 // bytes per table entry
  const LogitsParams &p = gs.p;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float sig_s[QH];

  const uint32_t dyn0 = smem_u32(smem);
  const uint32_t dyn_end = dyn0 + gs.dyn_bytes;
  const uint32_t T0 = (dyn0 + kGBarBytes + kGHalf - 1) & ~(kGHalf - 1);
  const uint32_t a0 = dyn0 + kGBarBytes;
  const int n_a = (int)((T0 - a0) / SB);
  const uint32_t b0 = T0 + 2 * kGHalf;
  const int n_b = b0 < dyn_end ? (int)((dyn_end - b0) / SB) : 0;
  const int stages = min(kGMaxStages, n_a + n_b);
  auto slot = [&](int s) -> uint32_t { return s < n_a ? a0 + (uint32_t)s * SB : b0 + (uint32_t)(s - n_a) * SB; };
  auto full_bar = [&](int s) { return dyn0 + 8u * s; };
  auto empty_bar = [&](int s) { return dyn0 + 8u * (kGMaxStages + s); };
  const uint32_t tab_bar = dyn0 + 8u * (2 * kGMaxStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (stages < 2 || b0 > dyn_end) {
    if (tid == 0) {
      pdl_wait();
      atomicOr(p.status, kDevBadShape);
    }
    return;
  }
  const int unit = blockIdx.x / gs.ctas_per_unit, part = blockIdx.x - unit * gs.ctas_per_unit;
  const int g0 = part * gs.tiles_per_unit / gs.ctas_per_unit, g1 = (part + 1) * gs.tiles_per_unit / gs.ctas_per_unit;
  if (g0 >= g1) return;
  const int n_my = g1 - g0;
  const int qb = unit % p.qblocks, sk = unit / p.qblocks;
  const size_t unit_first = (size_t)sk * p.capacity;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kGConsumers);
    }
    mbar_init(tab_bar, 1);
    mbar_fence_init();
  }
  __syncthreads();

  auto norms_by_copy = [&](size_t first, int n) {
    return (n % 4 == 0) && (((uintptr_t)(p.norm + first)) % 16 == 0) && (((uintptr_t)(p.rnorm + first)) % 16 == 0);
  };

  if (warp == kGConsumers) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      int issued = 0, s = 0;
      uint32_t phase = 1u;   // parity of the empty-barrier phase a stage's reuse waits for
      for (int i = 0; i < n_my; ++i) {
        if (i >= stages && !mbar_wait(empty_bar(s), phase)) {
          pdl_wait();
          atomicOr(p.status, kDevTimeout);
          break;
        }
        const int64_t t0 = (int64_t)(g0 + i) * kGTile;
        const int n = (int)min((int64_t)kGTile, p.n_tokens - t0);
        const size_t first = unit_first + t0;
        const uint32_t rec_bytes = (uint32_t)n * RW * 4;
        const bool nc = norms_by_copy(first, n);
        mbar_arrive_expect_tx(full_bar(s), rec_bytes + (nc ? 8u * n : 0u));
        const uint32_t st = slot(s);
        bulk_g2s(st, p.records + first * RW, rec_bytes, full_bar(s));
        if (nc) {
          bulk_g2s(st + kGTile * RW * 4, p.norm + first, 4u * n, full_bar(s));
          bulk_g2s(st + kGTile * RW * 4 + kGTile * 4, p.rnorm + first, 4u * n, full_bar(s));
        }
        ++issued;
        if (++s == stages) {
          s = 0;
          phase ^= 1u;
        }
      }
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
  pdl_wait();   // the tables (and a clean status word) come from the previous grid
  const int seq = sk / p.n_kv_heads, kvh = sk - seq * p.n_kv_heads;
  const int h0 = kvh * p.group + qb * QH;
  if (tid == 0) {
    constexpr uint32_t kChunk = 16384;
    mbar_arrive_expect_tx(tab_bar, 2 * kGHalf);
    const unsigned char *src = gs.tables + (size_t)unit * (2 * kGHalf);
    for (uint32_t o = 0; o < 2 * kGHalf; o += kChunk) bulk_g2s(T0 + o, src + o, kChunk, tab_bar);
  }
  if (tid < QH) sig_s[tid] = gs.sigma[(size_t)seq * p.n_q_heads + h0 + tid];
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kGConsumers) : "memory");
  float sg[QH];
#pragma unroll
  for (int h = 0; h < QH; ++h) sg[h] = sig_s[h];
  if (!mbar_wait(tab_bar, 0)) {
    atomicOr(p.status, kDevTimeout);
    return;
  }

  // per-lane address constants: byte 0 / byte 1 = entry offset of position (l ^ s) for steps
  // s = 2m / 2m + 1, bytes 2..3 = table base bytes 2..3 (T0 is 64 KB aligned)
  uint32_t sel[4];
  const uint32_t sel0 = 0x7604u | ((uint32_t)(lane & 3) << 4);
#pragma unroll
  for (int j = 0; j < 4; ++j) sel[j] = sel0 ^ ((uint32_t)(j & 1) | ((uint32_t)j << 4));
  constexpr int PSH = QH == 4 ? 3 : 2;   // log2 of the entry size
  const uint32_t x0 = (T0 & 0xFFFF0000u) | ((uint32_t)lane << PSH) | ((uint32_t)(lane ^ 1) << (8 + PSH));
  uint32_t xv[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) xv[m] = x0 ^ ((uint32_t)m * (0x202u << PSH));
  // the unit's logits rows and norm pointers; its norms come with the tiles when aligned (tiles
  // start 512 keys apart, so one check per unit decides it with the tile's length)
  float *lg_row = p.logits + ((size_t)seq * p.n_q_heads + h0) * p.n_tokens;
  const float *nrm_p = p.norm + unit_first, *rho_p = p.rnorm + unit_first;
  const bool unit_nc = (reinterpret_cast<uintptr_t>(nrm_p) % 16 == 0) && (reinterpret_cast<uintptr_t>(rho_p) % 16 == 0);
  const int k = warp * 32 + lane;
  int s = 0;
  uint32_t phase = 0;

  for (int i = 0; i < n_my; ++i) {
    if (!mbar_wait(full_bar(s), phase)) {
      atomicOr(p.status, kDevTimeout);
      return;
    }
    const int64_t t0 = (int64_t)(g0 + i) * kGTile;
    const int n = (int)min((int64_t)kGTile, p.n_tokens - t0);
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
        nrm = reinterpret_cast<const float *>(st + kGTile * RW * 4)[k];
        rho = reinterpret_cast<const float *>(st + kGTile * RW * 4 + kGTile * 4)[k];
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

    uint32_t wi[IW], wsg[4];
#pragma unroll
    for (int j = 0; j < IW; ++j) wi[j] = w[j];
#pragma unroll
    for (int j = 0; j < 4; ++j) wsg[j] = w[IW + j];
    xor_perm<IW>(wi, (lane >> 2) & (IW - 1));
    xor_perm<4>(wsg, (lane >> 2) & 3);
    float fi[QH], fs[QH];
#pragma unroll
    for (int h = 0; h < QH; ++h) fi[h] = fs[h] = 0.f;
    gqa_sum<QH, K::NI, 0u>(wi, sel, xv, fi);
    gqa_sum<QH, 16, kGHalf>(wsg, sel, xv, fs);
    if (valid) {
#pragma unroll
      for (int h = 0; h < QH; ++h)
        lg_row[h * p.n_tokens + t0 + k] = nrm * sg[h] * fmaf(rho, fs[h], fi[h]);
    }
  }
}

template <int BETA, int QH>
cudaError_t launch_gqa_t(const LogitsParams &p, const GqaParams &g, int n_seq, size_t limit, cudaStream_t st) {
  using K = GKeys<BETA>;
  const int units = n_seq * p.n_kv_heads * p.qblocks;
  // tables: one small grid, then the scan as its programmatic dependent
  cudaError_t e = launch_after(gqa_tables_kernel<BETA, QH>, dim3(units, 2, 4), dim3(256), 0, st, g);
  if (e != cudaSuccess) return e;
  GScan gs{};
  gs.p = p;
  gs.tables = g.tables;
  gs.sigma = g.sigma;
  gs.tiles_per_unit = (int)((p.n_tokens + kGTile - 1) / kGTile);
  // dynamic shared memory: barriers, the 64 KB-aligned 128 KB table block, stage slots around it
  const uint32_t dyn0 = 1024;
  const uint32_t T0 = (dyn0 + kGBarBytes + kGHalf - 1) & ~(kGHalf - 1);
  const uint32_t n_a = (T0 - dyn0 - kGBarBytes) / GStage<BETA>::kBytes;
  const uint32_t b0 = T0 + 2 * kGHalf;
  const uint32_t end = dyn0 + (uint32_t)limit;
  uint32_t n_b = b0 < end ? (end - b0) / GStage<BETA>::kBytes : 0;
  if (n_a + n_b > (uint32_t)kGMaxStages) n_b = kGMaxStages > (int)n_a ? kGMaxStages - n_a : 0;
  gs.dyn_bytes = (b0 + n_b * GStage<BETA>::kBytes) - dyn0;
  auto kern = logits_gqa_kernel<BETA, QH>;
  e = set_smem_once(reinterpret_cast<const void *>(kern), gs.dyn_bytes);
  if (e != cudaSuccess) return e;
  const int slots = device_sm_count();
  int cpu = slots / units;
  if (cpu < 1) cpu = 1;
  if (cpu > gs.tiles_per_unit) cpu = gs.tiles_per_unit;
  gs.ctas_per_unit = cpu;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(units * cpu));
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = gs.dyn_bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, gs);
}

}  // namespace

bool gqa_supported(int d, int bits, int group) {
  return d == kGD && (bits == 1 || bits == 2) && (group == 2 || group == 4 || group == 8);
}

size_t gqa_table_bytes(int units) { return (size_t)units * 2 * kGHalf; }

cudaError_t launch_gqa_tables(const GqaParams &g, int bits, int qh, int units, cudaStream_t st) {
  const dim3 grid(units, 2, 4), block(256);
  if (bits == 1) return qh == 4 ? launch_after(gqa_tables_kernel<1, 4>, grid, block, 0, st, g)
                                : launch_after(gqa_tables_kernel<1, 2>, grid, block, 0, st, g);
  return qh == 4 ? launch_after(gqa_tables_kernel<2, 4>, grid, block, 0, st, g)
                 : launch_after(gqa_tables_kernel<2, 2>, grid, block, 0, st, g);
}

cudaError_t launch_logits_gqa(const LogitsParams &p, const GqaParams &g, int bits, int n_seq, size_t limit,
                              cudaStream_t st) {
  const int qh = p.q_per_cta;
  if (bits == 1) return qh == 4 ? launch_gqa_t<1, 4>(p, g, n_seq, limit, st) : launch_gqa_t<1, 2>(p, g, n_seq, limit, st);
  return qh == 4 ? launch_gqa_t<2, 4>(p, g, n_seq, limit, st) : launch_gqa_t<2, 2>(p, g, n_seq, limit, st);
}

}  // namespace tq
