// Nearest-neighbour inner-product search over a packed key stream: for every query, the k
// database vectors with the largest estimated inner product. The pages also present the
// quantizer as a nearest-neighbour search method (zubnet.ai news, "Google's TurboQuant quantizes
// LLM KV cache to 3.5 bits per channel", paragraph 3; winningdata.io, "TurboQuant: Google
// comprime KV cache para 3 bits sem perder acuracia", "Os numeros que importam", recall on an
// inner-product search benchmark). The score of database vector j for query q is the key
// estimator of the logit scan,
//   score(q, j) = n_j ( <Pi q, c[idx_j]> + rho_j sqrt(pi/2)/d <S q, 2 sign_j - 1> ).
//
// With thousands of queries the scan is a dense contraction, so it runs on the tensor core:
//   A[q] = [Pi q | S q] / sigma_q                      fp16, sigma_q a power of two
//   B[j] = [c[idx_j] | rho_j sqrt(pi/2)/d (2 sign_j - 1)]   fp16, decoded on chip
//   score(q, j) = sigma_q n_j (A B^T)[q, j]
// One persistent CTA per SM walks a contiguous range of (query block, database tile) units:
//   * the 128 queries of the current block sit in tensor memory as the MMA's A operand;
//   * a copy warp streams each 128-vector tile's records and norms into shared memory;
//   * eight decode warps turn them into B, one 64-element K chunk at a time, in a ring of
//     128-byte-swizzled shared-memory chunks;
//   * one thread issues tcgen05 MMAs (M = 128 queries, N = 128 vectors, K = 16) into one of
//     two tensor-memory accumulators;
//   * four epilogue warps (one per lane quadrant) keep a running top-k per query row in
//     registers and write it to a per-CTA partial list when the query block changes.
// A merge kernel then combines the partial lists of every CTA that covered a query block.
#include <type_traits>

#include "common.cuh"
#include "tc.cuh"

namespace tq {
namespace {

constexpr int kQB = 128;                 // queries per block: MMA M, one tensor-memory lane each
constexpr int kNT = 128;                 // database vectors per tile: MMA N
constexpr int kDecWarps = 8;             // two groups of four (even and odd K chunks); a thread owns a row
constexpr int kEpiWarps = 4;             // one per lane quadrant
constexpr int kLists = kEpiWarps / 4;   // partial top-k lists per query row and CTA
constexpr int kNnThreads = 32 * (2 + kDecWarps + kEpiWarps);   // + MMA warp + copy warp
constexpr int kRStages = 4;              // ring of database tiles (records, norms, rnorms) in shared memory
constexpr uint32_t kChunk = kNT * 128;   // one 64-element K block of a tile: 16 KB
constexpr uint32_t kAcc0 = 256;          // first accumulator column; two buffers of kNT columns
constexpr int kNrmRing = 4;              // tiles of database norms staged for the epilogue
constexpr int kPrepQ = 16;               // queries per CTA of the projection kernel
constexpr int kPrepThreads = 256;

template <int D>
struct NnDim {
  static constexpr int NCH = (2 * D + 63) / 64;   // 64-element K chunks of a row
  static constexpr int KP = 64 * NCH;             // padded K
  static constexpr int ACOLS = KP / 2;            // tensor-memory columns of the query block
  static_assert(D % 8 == 0 && ACOLS <= (int)kAcc0 && ACOLS % 8 == 0, "unsupported d");
};

// Lookup of the centroids of several consecutive coordinates from their packed codes.
template <int BETA>
struct NnLut {
  static constexpr int CPL = BETA == 1 ? 8 : 4;   // coordinates per lookup
  static constexpr int LB = BETA * CPL;           // code bits per lookup
  static constexpr int ENTRIES = 1 << LB;
  static constexpr int EB = 2 * CPL;              // bytes per entry (fp16 centroids)
  // copies of each entry side by side, one per lane of a shared-memory phase (8 lanes of 16-byte
  // loads, 16 lanes of 8-byte loads): lane l reads copy l mod REP, so a phase never conflicts
  static constexpr int REP = BETA == 1 ? 8 : BETA == 2 ? 16 : 1;
  static constexpr uint32_t STRIDE = REP * EB;    // bytes from one entry to the next
  static constexpr uint32_t BYTES = ENTRIES * STRIDE;
};

template <int D, int BETA>
struct NnRec {
  static constexpr int IW = (BETA * D + 31) / 32;   // code-stream words
  static constexpr int SW = (D + 31) / 32;          // sign words
  static constexpr int RW = IW + SW;
  static_assert(RW % 2 == 0, "records are read as 8-byte pairs");
};

template <int D, int BETA>
struct NnSmem {
  static constexpr uint32_t kBFull = 0, kBEmpty = 96, kDFull = 192, kDEmpty = 208, kAFull = 224, kNFull = 232,
                            kNEmpty = 264, kRFull = 296, kREmpty = 328, kTslot = 360;
  static constexpr uint32_t kRecBytes = kNT * NnRec<D, BETA>::RW * 4;
  static constexpr uint32_t kStage = kRecBytes + 2 * kNT * 4;   // records, norms, rnorms
  static constexpr uint32_t kFixed = 1024 + NnLut<BETA>::BYTES + kNrmRing * kNT * 4 + kRStages * kStage;
  // B chunks: as many as the opt-in shared memory (227 KB) leaves, at most 12
  static constexpr int kSlots = (232448 - kFixed) / kChunk > 12 ? 12 : (int)((232448 - kFixed) / kChunk);
  static_assert(kSlots >= 4, "B ring");
  static constexpr uint32_t kRing = 1024;   // 1024-byte aligned for the 128-byte swizzle
  static constexpr uint32_t kLut = kRing + kSlots * kChunk;
  static constexpr uint32_t kNrm = kLut + NnLut<BETA>::BYTES;   // [kNrmRing][kNT] database norms
  static constexpr uint32_t kRec = kNrm + kNrmRing * kNT * 4;   // [kRStages] tile stages
  static constexpr uint32_t kBytes = kRec + kRStages * kStage;
};

struct NnParams {
  const uint32_t *records;
  const float *norm, *rnorm;
  const __half *qimg;     // [n_qb * 128][KP]
  const float *sigma;     // [n_qb * 128]
  const float *codebook;
  float *part_s;          // [slots][128][2][kNnMaxK] (the first kLists of each row used)
  int *part_i;
  uint32_t *status;
  int64_t n_db;
  int64_t units;          // query blocks x database tiles
  int n_tiles, k;
  float kappa;            // sqrt(pi/2) / d
};

__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

// B values of 8 consecutive K elements (one 16-byte unit) of a database row whose record is held
// in registers (`uk` a compile-time constant after unrolling, so every word index is too).
//   * Units [0, D/8): centroids c[idx] of coordinates 8 uk .. 8 uk + 7, by one lookup of 8 or two
//     of 4 consecutive codes (`lut` points at this lane's copy of the table).
//   * Units [D/8, D/4): the signed sketch weights rho kappa (2 sign - 1). Half p of word w takes
//     sign bit 2 w + p into its own sign bit: the product places bit 2w at bit 15 and bit 2w + 1 at
//     bit 31 without overlapping terms; `nb` = fp16x2 of -rho kappa.
//   * The rest: zero padding.
template <int D, int BETA>
__device__ __forceinline__ uint4 nn_unit_reg(const uint32_t *rec, int uk, uint32_t lut, uint32_t nb) {
  using R = NnRec<D, BETA>;
  constexpr int U8 = D / 8;
  if (uk < U8) {
    const int bit = 8 * BETA * uk, w = bit >> 5, sh = bit & 31;
    if constexpr (BETA == 1) {
      return lds_u128(lut + NnLut<1>::STRIDE * ((rec[w] >> sh) & 0xFFu));
    } else if constexpr (BETA == 2) {
      const uint32_t f = (rec[w] >> sh) & 0xFFFFu;
      const uint2 a = lds64(lut + NnLut<2>::STRIDE * (f & 0xFFu)), b = lds64(lut + NnLut<2>::STRIDE * (f >> 8));
      return make_uint4(a.x, a.y, b.x, b.y);
    } else {
      const uint32_t f = (sh > 8 ? __funnelshift_r(rec[w], rec[w + 1], sh) : rec[w] >> sh) & 0xFFFFFFu;
      const uint2 a = lds64(lut + NnLut<3>::STRIDE * (f & 0xFFFu)), b = lds64(lut + NnLut<3>::STRIDE * (f >> 12));
      return make_uint4(a.x, a.y, b.x, b.y);
    }
  } else if (uk < 2 * U8) {
    const int j = uk - U8;
    const uint32_t b = (rec[R::IW + (j >> 2)] >> (8 * (j & 3))) & 0xFFu;
    uint4 o;
    o.x = ((b * 0x40008000u) & 0x80008000u) ^ nb;
    o.y = ((b * 0x10002000u) & 0x80008000u) ^ nb;
    o.z = ((b * 0x04000800u) & 0x80008000u) ^ nb;
    o.w = ((b * 0x01000200u) & 0x80008000u) ^ nb;
    return o;
  }
  return make_uint4(0u, 0u, 0u, 0u);
}

// Sorted (descending score, then ascending index) top-k of one thread's stream in the last k of
// kNnMaxK slots; the first kNnMaxK - k slots hold +inf and never move, so the k-th score is always
// the last slot. A new score goes behind equal ones (within one stream the indices increase); an
// entry that an insertion pushes down keeps its place ahead of equal scores with higher indices,
// so an equal-scored entry of a higher index is the one that falls off the end.
__device__ __forceinline__ void topk_insert(float (&sv)[kNnMaxK], int (&si)[kNnMaxK], float v, int id) {
  bool moved = false;   // once the new entry is placed, the entries behind it shift down one slot each
#pragma unroll
  for (int j = 0; j < kNnMaxK; ++j) {
    if (moved || v > sv[j]) {
      moved = true;
      const float tv = sv[j];
      const int ti = si[j];
      sv[j] = v;
      si[j] = id;
      v = tv;
      id = ti;
    }
  }
}

template <int D, int BETA>
__global__ void __launch_bounds__(kNnThreads, 1) nn_scan_kernel(const NnParams p) {
  using Dm = NnDim<D>;
  using R = NnRec<D, BETA>;
  using L = NnSmem<D, BETA>;
  using Lu = NnLut<BETA>;
  constexpr int NCH = Dm::NCH, RW = R::RW, kSlots = L::kSlots;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sb = smem_u32(smem);
  auto b_full = [&](int s) { return sb + L::kBFull + 8u * s; };
  auto b_empty = [&](int s) { return sb + L::kBEmpty + 8u * s; };
  auto d_full = [&](int b) { return sb + L::kDFull + 8u * b; };
  auto d_empty = [&](int b) { return sb + L::kDEmpty + 8u * b; };
  const uint32_t a_full = sb + L::kAFull;
  auto n_full = [&](int e) { return sb + L::kNFull + 8u * e; };
  auto n_empty = [&](int e) { return sb + L::kNEmpty + 8u * e; };
  auto r_full = [&](int e) { return sb + L::kRFull + 8u * e; };
  auto r_empty = [&](int e) { return sb + L::kREmpty + 8u * e; };
  const uint32_t ring = sb + L::kRing, lut = sb + L::kLut, stages = sb + L::kRec;
  float *nrm_s = reinterpret_cast<float *>(smem + L::kNrm);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t u0 = p.units * blockIdx.x / gridDim.x, u1 = p.units * (blockIdx.x + 1) / gridDim.x;
  const int n_my = (int)(u1 - u0);

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(b_full(s), kDecWarps / 2);   // the decode group that wrote the chunk
      mbar_init(b_empty(s), 1);  // the MMAs' commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(d_full(b), 1);
      mbar_init(d_empty(b), kEpiWarps);
    }
    mbar_init(a_full, kEpiWarps);
    for (int e = 0; e < kNrmRing; ++e) {
      mbar_init(n_full(e), kDecWarps / 2);   // decode group 0 (all 128 rows)
      mbar_init(n_empty(e), kEpiWarps);
    }
    for (int e = 0; e < kRStages; ++e) {
      mbar_init(r_full(e), 1);   // the copy thread's expect_tx
      mbar_init(r_empty(e), kDecWarps);
    }
    mbar_fence_init();
  }
  if (warp == 0) {
    tc::alloc(sb + L::kTslot, 512);
    tc::relinquish();
  }
  pdl_wait();                 // the query rows come from the projection kernel
  pdl_launch_dependents();    // the merge may become resident meanwhile
  // centroid lookup: entry e -> fp16 c[code] of CPL consecutive coordinates
  for (int e = tid; e < Lu::ENTRIES; e += kNnThreads) {
    uint32_t wv[4];
#pragma unroll
    for (int c2 = 0; c2 < Lu::CPL / 2; ++c2) {
      const float lo = __ldg(p.codebook + ((e >> (BETA * 2 * c2)) & ((1 << BETA) - 1)));
      const float hi = __ldg(p.codebook + ((e >> (BETA * (2 * c2 + 1))) & ((1 << BETA) - 1)));
      wv[c2] = (uint32_t)__half_as_ushort(__float2half_rn(lo)) | ((uint32_t)__half_as_ushort(__float2half_rn(hi)) << 16);
    }
#pragma unroll 1
    for (int c = 0; c < Lu::REP; ++c) {
      if constexpr (Lu::CPL == 8)
        *reinterpret_cast<uint4 *>(smem + L::kLut + Lu::STRIDE * e + 16 * c) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      else
        *reinterpret_cast<uint2 *>(smem + L::kLut + Lu::STRIDE * e + 8 * c) = make_uint2(wv[0], wv[1]);
    }
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + L::kTslot);
  bool ok = true;

  if (warp == 0) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(kQB, kNT, false);
      int64_t prev_qb = -1;
      int seg = -1, last = -1;
      for (int i = 0; i < n_my && ok; ++i) {
        const int64_t qb = (u0 + i) / p.n_tiles;
        if (qb != prev_qb) {
          prev_qb = qb;
          ++seg;
          if (!mbar_wait(a_full, seg & 1)) { ok = false; break; }
        }
        const int b = i & 1;
        if (i >= 2 && !mbar_wait(d_empty(b), ((i >> 1) - 1) & 1)) { ok = false; break; }
        tc::fence_after();
        const uint32_t dt = tmem + kAcc0 + kNT * b;
#pragma unroll 1
        for (int kc = 0; kc < NCH && ok; ++kc) {
          const int g = NCH * i + kc, s = g % kSlots;
          if (!mbar_wait(b_full(s), (g / kSlots) & 1)) { ok = false; break; }
          tc::fence_after();
          const uint32_t base = ring + (uint32_t)s * kChunk;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            tc::mma_ts(dt, tmem + 8 * (4 * kc + ks), tc::smem_desc_sw128(base + 32 * ks), idesc, (kc | ks) ? 1u : 0u);
          tc::commit(b_empty(s));
        }
        if (!ok) break;
        tc::commit(d_full(b));
        last = i;
      }
      if (!ok) atomicOr(p.status, kDevTimeout);
      // nothing may still write tensor memory when it is freed
      if (last >= 0) mbar_wait(d_full(last & 1), (last >> 1) & 1);
    }
  } else if (warp == 1 + kDecWarps + kEpiWarps) {
    // ------------------------------ tile copies ------------------------------
    // records, norms and rnorms of each 128-vector tile; the bytes past the last 16-byte
    // boundary of a ragged last tile are copied with plain loads before the stage is armed
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n_my; ++i) {
        const int e = i % kRStages;
        if (i >= kRStages && !mbar_wait(r_empty(e), ((i / kRStages) - 1) & 1)) {
          ok = false;
          break;
        }
        const int64_t j0 = ((u0 + i) % p.n_tiles) * kNT;
        const uint32_t nv = (uint32_t)min((int64_t)kNT, p.n_db - j0);
        const uint32_t st = stages + (uint32_t)e * L::kStage;
        const uint32_t rb = nv * RW * 4, rb16 = rb & ~15u, nb = nv * 4, nb16 = nb & ~15u;
        const uint32_t *rsrc = p.records + (size_t)j0 * RW;
        for (uint32_t o = rb16; o < rb; o += 4) asm volatile("st.shared.u32 [%0], %1;" ::"r"(st + o), "r"(__ldg(rsrc + o / 4)) : "memory");
        for (uint32_t o = nb16; o < nb; o += 4) {
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(st + L::kRecBytes + o), "f"(__ldg(p.norm + j0 + o / 4)) : "memory");
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(st + L::kRecBytes + kNT * 4 + o), "f"(__ldg(p.rnorm + j0 + o / 4))
                       : "memory");
        }
        if (rb16 < rb || nb16 < nb) tc::fence_proxy_async();   // plain stores before later bulk writes here
        mbar_arrive_expect_tx(r_full(e), rb16 + 2 * nb16);
        if (rb16) bulk_g2s(st, rsrc, rb16, r_full(e));
        if (nb16) {
          bulk_g2s(st + L::kRecBytes, p.norm + j0, nb16, r_full(e));
          bulk_g2s(st + L::kRecBytes + kNT * 4, p.rnorm + j0, nb16, r_full(e));
        }
        ++issued;
      }
      // no copy may still be landing when the CTA exits
      for (int i = max(0, issued - kRStages); i < issued; ++i) mbar_wait(r_full(i % kRStages), (i / kRStages) & 1);
      if (!ok) atomicOr(p.status, kDevTimeout);
    }
  } else if (warp <= kDecWarps) {
    // -------------------------------- decode --------------------------------
    // group 0 (warps 1-4) writes the even K chunks, group 1 the odd ones; a thread owns one row
    // and holds its record in registers while it writes its group's chunks
    const int dw = warp - 1, grp = dw >> 2, r = 32 * (dw & 3) + lane;
    const uint32_t row_ofs = (uint32_t)r * 128u;
    const int rsw = r & 7;
    const uint32_t lut_l = lut + (uint32_t)(lane & (Lu::REP - 1)) * Lu::EB;   // this lane's copy of the table
    uint32_t rec[RW];
    auto chunks = [&](auto G, int i, uint32_t nbh) {
      constexpr int kc0 = decltype(G)::value;
#pragma unroll
      for (int kc = kc0; kc < NCH; kc += 2) {
        const int g = NCH * i + kc, s = g % kSlots;
        if (g >= kSlots && !mbar_wait(b_empty(s), ((g / kSlots) - 1) & 1)) {
          ok = false;
          return;
        }
        const uint32_t dst = ring + (uint32_t)s * kChunk + row_ofs;
#pragma unroll
        for (int uu = 0; uu < 8; ++uu)
          sts128(dst + (uint32_t)((uu ^ rsw) << 4), nn_unit_reg<D, BETA>(rec, 8 * kc + uu, lut_l, nbh));
        tc::fence_proxy_async();   // generic stores -> tensor-core reads
        __syncwarp();
        if (lane == 0) mbar_arrive(b_full(s));
      }
    };
    for (int i = 0; i < n_my && ok; ++i) {
      const int e = i % kRStages;
      if (!mbar_wait(r_full(e), (i / kRStages) & 1)) {
        ok = false;
        break;
      }
      const uint32_t st = stages + (uint32_t)e * L::kStage;
      const uint32_t rs = st + (uint32_t)r * RW * 4;
#pragma unroll
      for (int w = 0; w < RW / 2; ++w) {
        const uint2 v = lds64(rs + 8u * w);
        rec[2 * w] = v.x;
        rec[2 * w + 1] = v.y;
      }
      const bool valid = ((u0 + i) % p.n_tiles) * kNT + r < p.n_db;   // rows past the database: ignored columns
      const float nrm = valid ? lds_f32(st + L::kRecBytes + 4u * r) : __int_as_float(0x7fc00000);
      const float rho = valid ? lds_f32(st + L::kRecBytes + kNT * 4 + 4u * r) : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(r_empty(e));   // the stage is in registers: the copy may refill it
      if (grp == 0) {
        // the tile's norms for the epilogue (its entry of the ring is free once tile i - 4 is scored)
        const int ne = i % kNrmRing;
        if (i >= kNrmRing && !mbar_wait(n_empty(ne), ((i / kNrmRing) - 1) & 1)) {
          ok = false;
          break;
        }
        nrm_s[ne * kNT + r] = nrm;
        __syncwarp();
        if (lane == 0) mbar_arrive(n_full(ne));
      }
      const uint32_t nbh = (uint32_t)__half_as_ushort(__float2half_rn(-rho * p.kappa)) * 0x00010001u;
      if (grp == 0)
        chunks(std::integral_constant<int, 0>{}, i, nbh);
      else
        chunks(std::integral_constant<int, 1>{}, i, nbh);
    }
    if (!ok) atomicOr(p.status, kDevTimeout);
  } else {
    // ------------------------------- epilogue -------------------------------
    const int ew = warp - 1 - kDecWarps, q4 = warp & 3, hh = ew >> 2, r = 32 * q4 + lane;
    constexpr int kCols = kNT / kLists;   // columns of each tile this warp scores
    const uint32_t lane_ofs = (uint32_t)(32 * q4) << 16;
    float sv[kNnMaxK], sig = 1.f;
    int si[kNnMaxK];
    auto reset = [&]() {
#pragma unroll
      for (int j = 0; j < kNnMaxK; ++j) {
        sv[j] = j < kNnMaxK - p.k ? INFINITY : -INFINITY;
        si[j] = -1;
      }
    };
    auto flush = [&](int64_t qb) {
      const size_t base = (((size_t)(blockIdx.x + qb) * kQB + r) * 2 + hh) * kNnMaxK;
#pragma unroll
      for (int j = 0; j < kNnMaxK; ++j)
        if (j >= kNnMaxK - p.k) {
          p.part_s[base + j - (kNnMaxK - p.k)] = sv[j] * sig;
          p.part_i[base + j - (kNnMaxK - p.k)] = si[j];
        }
    };
    // score 16 columns (accumulators in `acc`, norms from the staged tile) against the running list
    auto score16 = [&](uint32_t (&acc)[16], const float4 *nr4, int jc) {
      const float thr = sv[kNnMaxK - 1];
      float mx = -INFINITY;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const float4 n4 = nr4[c4];   // same address in every lane: one broadcast
        const float nn[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float v = __uint_as_float(acc[4 * c4 + c]) * nn[c];
          acc[4 * c4 + c] = __float_as_uint(v);   // the score replaces the accumulator
          mx = fmaxf(mx, v);                       // NaN (past the database) is dropped
        }
      }
      if (!(mx > thr)) return;   // the common case once the list has filled
      uint32_t hit = 0;
#pragma unroll
      for (int c = 0; c < 16; ++c) hit |= (__uint_as_float(acc[c]) > thr ? 1u : 0u) << c;
      // columns above the running k-th score, inserted in column order
      while (hit) {
        const int c = __ffs(hit) - 1;
        hit &= hit - 1;
        uint32_t vb = acc[0];
#pragma unroll
        for (int m = 1; m < 16; ++m)
          if (m == c) vb = acc[m];
        const float v = __uint_as_float(vb);
        if (v > sv[kNnMaxK - 1]) topk_insert(sv, si, v, jc + c);
      }
    };
    reset();
    int64_t prev_qb = -1;
    for (int i = 0; i < n_my; ++i) {
      const int64_t u = u0 + i, qb = u / p.n_tiles, t = u - qb * p.n_tiles;
      if (qb != prev_qb) {
        // every MMA of the previous block is complete (its last accumulator was read below)
        if (prev_qb >= 0) {
          flush(prev_qb);
          reset();
        }
        prev_qb = qb;
        const size_t row = (size_t)qb * kQB + r;
        sig = __ldg(p.sigma + row);
        // this warp's share of the row: columns [hh ACOLS / kLists, (hh + 1) ACOLS / kLists)
        constexpr int kAc = Dm::ACOLS / kLists;
        const uint4 *src = reinterpret_cast<const uint4 *>(p.qimg + row * Dm::KP + hh * 2 * kAc);
#pragma unroll 2
        for (int c = 0; c < kAc; c += 8) {
          const uint4 a = __ldg(src + c / 4), b = __ldg(src + c / 4 + 1);
          const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
          tc::st8(tmem + lane_ofs + hh * kAc + c, v);
        }
        tc::wait_st();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_full);
      }
      const int b = i & 1, ne = i % kNrmRing;
      if (!mbar_wait(d_full(b), (i >> 1) & 1) || !mbar_wait(n_full(ne), (i / kNrmRing) & 1)) {
        ok = false;
        break;
      }
      tc::fence_after();
      const int j0 = (int)(t * kNT) + kCols * hh;
      const uint32_t ta = tmem + lane_ofs + kAcc0 + kNT * b + kCols * hh;
      const float4 *nr4 = reinterpret_cast<const float4 *>(nrm_s + ne * kNT + kCols * hh);
      // two 16-column groups per pass: the second is loaded from tensor memory while the first is scored
      uint32_t acc0[16], acc1[16];
      tc::ld16(ta, acc0);
      tc::wait_ld();
#pragma unroll 1
      for (int g = 0; g < kCols / 16; g += 2) {
        tc::ld16(ta + 16 * (g + 1), acc1);
        score16(acc0, nr4 + 4 * g, j0 + 16 * g);
        __syncwarp();
        tc::wait_ld();
        if (g + 2 < kCols / 16) tc::ld16(ta + 16 * (g + 2), acc0);
        score16(acc1, nr4 + 4 * (g + 1), j0 + 16 * (g + 1));
        __syncwarp();
        if (g + 2 < kCols / 16) tc::wait_ld();
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(d_empty(b));    // the accumulator has been read
        mbar_arrive(n_empty(ne));   // and the norms
      }
    }
    if (ok && prev_qb >= 0) flush(prev_qb);
    if (!ok) atomicOr(p.status, kDevTimeout);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  if (warp == 0) {
    __syncwarp();
    tc::dealloc(tmem, 512);
  }
}

// Query rows of the A operand: [Pi q | S q | 0] / sigma in fp16, sigma = 2^e >= max |.| of the
// row (exact scaling), for every row of every query block (rows past n_q are zero).
template <int D>
__global__ void __launch_bounds__(kPrepThreads) nn_qprep_kernel(const float *__restrict__ q, int n_q,
                                                                const float *__restrict__ Pi,
                                                                const float *__restrict__ S, __half *qimg,
                                                                float *sigma, uint32_t *status) {
  constexpr int KP = NnDim<D>::KP;
  __shared__ float qs[kPrepQ][D];
  __shared__ float os[kPrepQ][2 * D];
  __shared__ unsigned int mx[kPrepQ];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, q0 = blockIdx.x * kPrepQ;
  if (blockIdx.x == 0 && tid == 0) *status = 0u;
  for (int e = tid; e < kPrepQ * D; e += kPrepThreads) {
    const int a = e / D, i = e - a * D;
    qs[a][i] = q0 + a < n_q ? __ldg(q + (size_t)(q0 + a) * D + i) : 0.f;
  }
  if (tid < kPrepQ) mx[tid] = 0u;
  __syncthreads();
  for (int o = tid; o < 2 * D; o += kPrepThreads) {
    const float4 *row = reinterpret_cast<const float4 *>(o < D ? Pi + (size_t)o * D : S + (size_t)(o - D) * D);
    float acc[kPrepQ];
#pragma unroll
    for (int a = 0; a < kPrepQ; ++a) acc[a] = 0.f;
    for (int i4 = 0; i4 < D / 4; ++i4) {
      const float4 m = __ldg(row + i4);
#pragma unroll
      for (int a = 0; a < kPrepQ; ++a) {
        acc[a] = fmaf(m.x, qs[a][4 * i4], acc[a]);
        acc[a] = fmaf(m.y, qs[a][4 * i4 + 1], acc[a]);
        acc[a] = fmaf(m.z, qs[a][4 * i4 + 2], acc[a]);
        acc[a] = fmaf(m.w, qs[a][4 * i4 + 3], acc[a]);
      }
    }
#pragma unroll
    for (int a = 0; a < kPrepQ; ++a) {
      os[a][o] = acc[a];
      atomicMax(&mx[a], __float_as_uint(fabsf(acc[a])));   // non-negative floats order as integers
    }
  }
  __syncthreads();
  for (int e = tid; e < kPrepQ * (KP / 2); e += kPrepThreads) {
    const int a = e / (KP / 2), c = e - a * (KP / 2);
    const float m = __uint_as_float(mx[a]);
    int ex = 0;
    const bool scaled = m > 0.f && isfinite(m);
    if (scaled) frexpf(m, &ex);
    const float inv = scaled ? ldexpf(1.f, -ex) : 1.f;
    const float v0 = 2 * c < 2 * D ? os[a][2 * c] * inv : 0.f;
    const float v1 = 2 * c + 1 < 2 * D ? os[a][2 * c + 1] * inv : 0.f;
    reinterpret_cast<__half2 *>(qimg + (size_t)(q0 + a) * KP)[c] = __floats2half2_rn(v0, v1);
    if (c == 0) sigma[q0 + a] = scaled ? ldexpf(1.f, ex) : 1.f;
  }
}

// Per query: the k best of every partial list of the CTAs that covered its block, in
// (score descending, index ascending) order; missing entries are (-inf, -1).
__global__ void __launch_bounds__(128) nn_merge_kernel(const float *__restrict__ part_s,
                                                       const int *__restrict__ part_i, int n_q, int64_t units,
                                                       int n_tiles, int grid, int k, float *top_s,
                                                       int64_t *top_i) {
  pdl_wait();
  const int qi = blockIdx.x * blockDim.x + threadIdx.x;
  if (qi >= n_q) return;
  const int qb = qi / kQB, r = qi - qb * kQB;
  float sv[kNnMaxK];
  int si[kNnMaxK];
#pragma unroll
  for (int j = 0; j < kNnMaxK; ++j) {
    sv[j] = -INFINITY;
    si[j] = -1;
  }
  const int64_t lo = (int64_t)qb * n_tiles, hi = lo + n_tiles;
  for (int c = 0; c < grid; ++c) {
    const int64_t c0 = units * c / grid, c1 = units * (c + 1) / grid;
    if (c0 >= hi) break;
    if (c1 <= lo || c0 == c1) continue;
    for (int hh = 0; hh < kLists; ++hh) {
      const size_t base = (((size_t)(c + qb) * kQB + r) * 2 + hh) * kNnMaxK;
      for (int j = 0; j < k; ++j) {
        float v = part_s[base + j];
        int id = part_i[base + j];
        if (id < 0) break;   // lists are filled from the front
#pragma unroll
        for (int m = 0; m < kNnMaxK; ++m) {
          if (m < k && (v > sv[m] || (v == sv[m] && id < si[m]) || si[m] < 0)) {
            const float tv = sv[m];
            const int ti = si[m];
            sv[m] = v;
            si[m] = id;
            v = tv;
            id = ti;
          }
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kNnMaxK; ++j)
    if (j < k) {
      top_s[(size_t)qi * k + j] = sv[j];
      top_i[(size_t)qi * k + j] = si[j];
    }
}

template <int D, int BETA>
cudaError_t launch_scan(const NnParams &p, int grid, cudaStream_t st) {
  auto kern = nn_scan_kernel<D, BETA>;
  const size_t smem = NnSmem<D, BETA>::kBytes;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  return launch_after(kern, dim3((unsigned)grid), dim3(kNnThreads), smem, st, p);
}

template <int D>
cudaError_t launch_d(const NnArgs &a, cudaStream_t st) {
  const int n_qb = (a.n_q + kQB - 1) / kQB;
  cudaError_t e = launch_after(nn_qprep_kernel<D>, dim3((unsigned)(n_qb * kQB / kPrepQ)), dim3(kPrepThreads), 0, st,
                               a.q, a.n_q, a.Pi, a.S, reinterpret_cast<__half *>(a.qimg), a.sigma, a.status);
  if (e != cudaSuccess) return e;
  const int n_tiles = (int)((a.n_db + kNT - 1) / kNT);
  NnParams p{};
  p.records = a.records;
  p.norm = a.norm;
  p.rnorm = a.rnorm;
  p.qimg = reinterpret_cast<const __half *>(a.qimg);
  p.sigma = a.sigma;
  p.codebook = a.codebook;
  p.part_s = a.part_s;
  p.part_i = a.part_i;
  p.status = a.status;
  p.n_db = a.n_db;
  p.units = (int64_t)n_qb * n_tiles;
  p.n_tiles = n_tiles;
  p.k = a.k;
  p.kappa = (float)(1.2533141373155002512 / D);   // sqrt(pi / 2) / d
  switch (a.bits) {
    case 1: e = launch_scan<D, 1>(p, a.grid, st); break;
    case 2: e = launch_scan<D, 2>(p, a.grid, st); break;
    default: e = launch_scan<D, 3>(p, a.grid, st); break;
  }
  if (e != cudaSuccess) return e;
  return launch_after(nn_merge_kernel, dim3((unsigned)((a.n_q + 127) / 128)), dim3(128), 0, st,
                      (const float *)a.part_s, (const int *)a.part_i, a.n_q, p.units, n_tiles, a.grid, a.k, a.top_s,
                      a.top_i);
}

}  // namespace

namespace {
// Top-k of n_parts sorted lists per query (score descending, then id ascending; id -1 marks an
// empty place, only at a list's end): the same insertion order as nn_merge_kernel.
__global__ void __launch_bounds__(128) nn_list_merge_kernel(const float *__restrict__ ps, const int64_t *__restrict__ pi,
                                                            int n_parts, int n_q, int k, float *top_s,
                                                            int64_t *top_i) {
  const int qi = blockIdx.x * blockDim.x + threadIdx.x;
  if (qi >= n_q) return;
  float sv[kNnMaxK];
  int64_t si[kNnMaxK];
#pragma unroll
  for (int j = 0; j < kNnMaxK; ++j) {
    sv[j] = -INFINITY;
    si[j] = -1;
  }
  for (int c = 0; c < n_parts; ++c) {
    const size_t base = ((size_t)c * n_q + qi) * k;
    for (int j = 0; j < k; ++j) {
      float v = ps[base + j];
      int64_t id = pi[base + j];
      if (id < 0) break;
#pragma unroll
      for (int m = 0; m < kNnMaxK; ++m) {
        if (m < k && (v > sv[m] || (v == sv[m] && id < si[m]) || si[m] < 0)) {
          const float tv = sv[m];
          const int64_t ti = si[m];
          sv[m] = v;
          si[m] = id;
          v = tv;
          id = ti;
        }
      }
    }
  }
  for (int j = 0; j < k; ++j) {
    top_s[(size_t)qi * k + j] = sv[j];
    top_i[(size_t)qi * k + j] = si[j];
  }
}
}  // namespace

cudaError_t launch_nn_list_merge(const float *ps, const int64_t *pi, int n_parts, int n_q, int k, float *top_s,
                                 int64_t *top_i, cudaStream_t st) {
  nn_list_merge_kernel<<<(n_q + 127) / 128, 128, 0, st>>>(ps, pi, n_parts, n_q, k, top_s, top_i);
  return cudaGetLastError();
}

bool nn_supported(int d, int bits) { return (d == 128 || d == 200) && bits >= 1 && bits <= 3; }

int nn_kp(int d) { return 64 * ((2 * d + 63) / 64); }

// n_db == 0 launches only the merge (every list empty); grid == 0 then.
cudaError_t launch_nn_search(const NnArgs &a, cudaStream_t st) {
  if (a.n_db == 0)
    return launch_after(nn_merge_kernel, dim3((unsigned)((a.n_q + 127) / 128)), dim3(128), 0, st,
                        (const float *)a.part_s, (const int *)a.part_i, a.n_q, (int64_t)0, 0, 0, a.k, a.top_s,
                        a.top_i);
  return a.d == 128 ? launch_d<128>(a, st) : launch_d<200>(a, st);
}

}  // namespace tq
