// Lookup-table logit machinery for d = 128 key records (1..3 code bits + the
// QJL sign field), shared by the logit scan (logits_fast.cu) and the fused
// decode attention (decode_fused.cu).
//
// Estimator (usedby.ai, "TurboQuant: Compresion de KV Cache a 3 bits y
// aceleracion de inferencia en H100", "El Pitch"; winningdata.io, "TurboQuant:
// Google comprime KV cache para 3 bits sem perder acuracia", "2. QJL
// Residual"):
//   l_t = n_t ( <Pi q, c[code_t]> + rho_t sqrt(pi/2)/d <S q, 2 sign_t - 1> ).
//
// Tables. The tables of query head q start at a 64 KB-aligned shared address
// T0 + q * 64 KB, so a lookup address is formed by bit operations alone and the
// per-query offset is the load's immediate. An index key is the codes of g
// consecutive coordinates as they sit in the code stream (g = 8, 4, 2 for 1, 2,
// 3 code bits: 8, 8 and 6 key bits); a d = 128 key has 16, 32 or 64 of them plus
// 16 sign bytes. Each table entry is the partial dot product of the query with
// that group.
//
// Byte keys (1 and 2 code bits): one table row per key value holds 64 words,
// positions 0..31 for the index tables and 32..63 for the sign tables (a
// 16-table set sits twice, at p and p + 16). At step s lane l reads position
// p = s XOR l, so the 32 lanes hit 32 different banks whatever the key values.
// The lane first permutes its record words by XOR with l/4 (a few selects,
// shared by every query head of the group); the byte of key p is then picked
// by one byte-permute whose selector depends only on l mod 4 and s mod 4, and
// lands already shifted into the row field, merged with the table base's high
// bytes. A lookup is one byte-permute, one shared load and one add.
//
// 6-bit keys (3 code bits): 64 tables of 64 entries in two groups of 32 (row
// stride 32 words), and the 16 sign tables in their own rows (twice, rows of
// 32 words). At step s lane l reads position (s + l) mod 32 after rotating its
// record so that key (s + l) sits at static position s.
#pragma once

#include "common.cuh"

namespace tq {
namespace scan {

constexpr int kFD = 128;                       // head dimension
constexpr uint32_t kTabStride = 0x10000;       // shared bytes per query head's tables (64 KB)

template <int BETA>
struct FastKeys {
  static constexpr int IW = BETA * kFD / 32;               // code-stream words
  static constexpr int RW = IW + kFD / 32;                 // record words
  static constexpr int NI = BETA == 1 ? 16 : BETA == 2 ? 32 : 64;   // index keys per record
  static constexpr int G = BETA == 3 ? 2 : 8 / BETA;       // coordinates per index key
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
  float a[4], b[2];   // each chain starts at its first lookup (no zeroing, no add to zero)
#pragma unroll
  for (int st = 0; st < NI; ++st) {
    const float v = lds_at<QQ * kTabStride>(__byte_perm(wi[st >> 2], xi[st >> 1], sel[st & 3]));
    a[st & 3] = st < 4 ? v : a[st & 3] + v;
  }
#pragma unroll
  for (int st = 0; st < 16; ++st) {
    const float v = lds_at<QQ * kTabStride>(__byte_perm(wsg[st >> 2], xs[st >> 1], sel[st & 3]));
    b[st & 1] = st < 2 ? v : b[st & 1] + v;
  }
  const float a0 = a[0], a1 = a[1], a2 = a[2], a3 = a[3], b0 = b[0], b1 = b[1];
  return nrm * fmaf(rho, b0 + b1, (a0 + a1) + (a2 + a3));
}

// One query head's logit for a 3-bit-code record (rotated halves lo/hi and sign stream rs).
template <int QQ>
__device__ __forceinline__ float scan_six(const uint32_t (&lo)[6], const uint32_t (&hi)[6], const uint32_t (&rs)[4],
                                          const uint32_t (&bank)[32], float nrm, float rho) {
  float a[4], b[2];   // each chain starts at its first lookup (no zeroing, no add to zero)
#pragma unroll
  for (int st = 0; st < 32; ++st) {
    const float v = lds_at<QQ * kTabStride>(key_addr7<6>(lo, 6 * st, bank[st]));
    a[st & 1] = st < 2 ? v : a[st & 1] + v;
  }
#pragma unroll
  for (int st = 0; st < 32; ++st) {
    const float v = lds_at<QQ * kTabStride + 8192>(key_addr7<6>(hi, 6 * st, bank[st]));
    a[2 + (st & 1)] = st < 2 ? v : a[2 + (st & 1)] + v;
  }
#pragma unroll
  for (int st = 0; st < 16; ++st) {
    const float v = lds_at<QQ * kTabStride + 32768>(key_addr7<8>(rs, 8 * st, bank[st]));
    b[st & 1] = st < 2 ? v : b[st & 1] + v;
  }
  const float a0 = a[0], a1 = a[1], a2 = a[2], a3 = a[3], b0 = b[0], b1 = b[1];
  return nrm * fmaf(rho, b0 + b1, (a0 + a1) + (a2 + a3));
}

// The logits of one key record for QMAX query heads (tables at T0 + qq * 64 KB;
// heads past nq are left at 0). w: the record words of this lane's key.
template <int BETA, int QMAX>
__device__ __forceinline__ void key_logits(const uint32_t (&w)[FastKeys<BETA>::RW], int lane, uint32_t T0, int nq,
                                           float nrm, float rho, float (&out)[QMAX]) {
  constexpr int IW = FastKeys<BETA>::IW;
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
}

// The lookup tables of one query head at tq_ (its 64 KB block), from qr = Pi q
// and qs = S q, with kappa = sqrt(pi/2)/d folded into the sign tables. Called
// by NTHR threads (tid < NTHR).
//
// Byte keys (1 and 2 code bits; NTHR = 512, 16 warps): an entry is the sum of a
// part over its low nibble and a part over its high nibble. Lane l of warp w
// owns table column l (warps 0-7: index positions) or 32 + l (warps 8-15: sign
// positions) and the 32 keys whose high nibble is 2 (w mod 8) or 2 (w mod 8) + 1:
// it forms the 16 low-nibble parts and its 2 high-nibble parts in registers,
// and then each entry is one add and one store, a warp storing 32 consecutive
// words of one row.
//
// 6-bit keys (3 code bits): each thread keeps one table position (and so its
// few query values) in registers and walks the key values with a stride of
// NTHR / width, so a warp shares one key: codebook reads broadcast and stores
// hit 32 banks.
template <int BETA, int NTHR>
__device__ __forceinline__ void build_tables(const float *qr, const float *qs, float *tq_, const float *cbs, int tid,
                                             float kappa) {
  using K = FastKeys<BETA>;
  if constexpr (BETA != 3) {
    static_assert(NTHR == 512, "byte-key tables: 16 warps, 2 high nibbles each");
    constexpr int L = 1 << BETA, GH = K::G / 2;   // codes per nibble
    const int warp = tid >> 5, lane = tid & 31, hn0 = 2 * (warp & 7);
    const bool sign = warp >= 8;
    float lo[16], hi[2];
    if (!sign) {
      // index position t: the G codes of one byte of the code stream
      const int t = lane & (K::NI - 1);
      float qc[K::G], cv[L];
#pragma unroll
      for (int c = 0; c < K::G; ++c) qc[c] = qr[t * K::G + c];
#pragma unroll
      for (int c = 0; c < L; ++c) cv[c] = cbs[c];
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        float v = qc[0] * cv[n & (L - 1)];
#pragma unroll
        for (int c = 1; c < GH; ++c) v = fmaf(qc[c], cv[(n >> (BETA * c)) & (L - 1)], v);
        lo[n] = v;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int n = hn0 + j;
        float v = qc[GH] * cv[n & (L - 1)];
#pragma unroll
        for (int c = 1; c < GH; ++c) v = fmaf(qc[GH + c], cv[(n >> (BETA * c)) & (L - 1)], v);
        hi[j] = v;
      }
    } else {
      // sign position t: 8 sign bits, +-kappa (S q)_i
      const int t = lane & 15;
      float sv[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) sv[c] = kappa * qs[8 * t + c];
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        float v = (n & 1) ? sv[0] : -sv[0];
#pragma unroll
        for (int c = 1; c < 4; ++c) v += ((n >> c) & 1) ? sv[c] : -sv[c];
        lo[n] = v;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int n = hn0 + j;
        float v = (n & 1) ? sv[4] : -sv[4];
#pragma unroll
        for (int c = 1; c < 4; ++c) v += ((n >> c) & 1) ? sv[4 + c] : -sv[4 + c];
        hi[j] = v;
      }
    }
    float *col = tq_ + (sign ? 32 : 0) + lane;   // 256 rows of 64 words: [0, 32) index, [32, 64) sign positions
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int n = 0; n < 16; ++n) col[((hn0 + j) * 16 + n) * 64] = lo[n] + hi[j];
  } else {
    // index: 2 groups x 64 rows x 32 words at +0; sign: 256 rows x 32 words at +32 KB
    {
      const int t = tid & 63;
      const float q0 = qr[2 * t], q1 = qr[2 * t + 1];
      float *row = tq_ + (t >> 5) * 64 * 32 + (t & 31);
      for (int key = tid >> 6; key < 64; key += NTHR / 64)
        row[key * 32] = fmaf(q1, cbs[(key >> 3) & 7], q0 * cbs[key & 7]);
    }
    {
      const int pos = tid & 31, t = pos & 15;
      float sv[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) sv[c] = kappa * qs[8 * t + c];
      float *ts = tq_ + 8192;
      for (int key = tid >> 5; key < 256; key += NTHR / 32) {
        float v = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) v += ((key >> c) & 1) ? sv[c] : -sv[c];
        ts[key * 32 + pos] = v;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Mixed rate (fractional bits per channel): the first 64 rotated coordinates at
// BETA + 1 code bits, the other 64 at BETA (BETA = 1: 2.5 bits per channel with
// the sign bit, BETA = 2: 3.5). The record holds the 64 wide codes, the 64
// narrow codes and the 16 sign bytes back to back. Keys are taken two wide
// coordinates at a time (32 keys of 2 (BETA + 1) bits) and 8 / BETA narrow bits
// at a time (4-bit keys: 32 of them for BETA = 2, 16 for BETA = 1), plus the 16
// sign bytes; every table has rows of 32 words (a key shifted to bit 7) and one
// column per key position, read at position (s + l) mod 32 after the lane's
// streams are rotated, as for the 6-bit keys above. Sets of 16 positions sit
// twice (p and p + 16). Per query head: wide tables at +0 (2^(2 BETA + 2) rows),
// narrow at +8 KB (16 rows), signs at +32 KB (256 rows).
template <int BETA>
struct MixedKeys {
  static constexpr int WW = 2 * (BETA + 1);      // wide code words (64 codes of BETA + 1 bits)
  static constexpr int NW = 2 * BETA;            // narrow code words
  static constexpr int IW = WW + NW;
  static constexpr int RW = IW + kFD / 32;       // + the sign words
  static constexpr int KW = 2 * (BETA + 1);      // wide key bits (two coordinates)
  static constexpr int NKN = BETA == 2 ? 32 : 16;   // narrow 4-bit keys
  static constexpr int CN = 4 / BETA;            // coordinates per narrow key
  static constexpr uint32_t kNarrow = 8192, kSign = 32768;   // byte offsets in a query head's tables
};

template <int BETA, int QQ>
__device__ __forceinline__ float scan_mixed(const uint32_t (&wr)[MixedKeys<BETA>::WW],
                                            const uint32_t (&nr)[MixedKeys<BETA>::NW], const uint32_t (&rs)[4],
                                            const uint32_t (&bank)[32], float nrm, float rho) {
  using M = MixedKeys<BETA>;
  float a[4], b[2];   // each chain starts at its first lookup
#pragma unroll
  for (int st = 0; st < 32; ++st) {
    const float v = lds_at<QQ * kTabStride>(key_addr7<M::KW>(wr, M::KW * st, bank[st]));
    a[st & 1] = st < 2 ? v : a[st & 1] + v;
  }
#pragma unroll
  for (int st = 0; st < M::NKN; ++st) {
    const float v = lds_at<QQ * kTabStride + M::kNarrow>(key_addr7<4>(nr, 4 * st, bank[st]));
    a[2 + (st & 1)] = st < 2 ? v : a[2 + (st & 1)] + v;
  }
#pragma unroll
  for (int st = 0; st < 16; ++st) {
    const float v = lds_at<QQ * kTabStride + M::kSign>(key_addr7<8>(rs, 8 * st, bank[st]));
    b[st & 1] = st < 2 ? v : b[st & 1] + v;
  }
  const float a0 = a[0], a1 = a[1], a2 = a[2], a3 = a[3], b0 = b[0], b1 = b[1];
  return nrm * fmaf(rho, b0 + b1, (a0 + a1) + (a2 + a3));
}

// The logits of one mixed-rate key record for QMAX query heads (as key_logits).
template <int BETA, int QMAX>
__device__ __forceinline__ void key_logits_mixed(const uint32_t (&w)[MixedKeys<BETA>::RW], int lane, uint32_t T0,
                                                 int nq, float nrm, float rho, float (&out)[QMAX]) {
  using M = MixedKeys<BETA>;
#pragma unroll
  for (int qq = 0; qq < QMAX; ++qq) out[qq] = 0.f;
  uint32_t bank[32];
#pragma unroll
  for (int s2 = 0; s2 < 32; ++s2) bank[s2] = T0 | (uint32_t)(((s2 + lane) & 31) << 2);
  uint32_t wr[M::WW], nr[M::NW], rs[4];
#pragma unroll
  for (int j = 0; j < M::WW; ++j) wr[j] = w[j];
#pragma unroll
  for (int j = 0; j < M::NW; ++j) nr[j] = w[M::WW + j];
#pragma unroll
  for (int j = 0; j < 4; ++j) rs[j] = w[M::IW + j];
  rotate_stream<M::WW>(wr, M::KW * lane);
  rotate_stream<M::NW>(nr, 4 * (lane & (M::NKN - 1)));
  rotate_stream<4>(rs, 8 * (lane & 15));
  out[0] = scan_mixed<BETA, 0>(wr, nr, rs, bank, nrm, rho);
  if constexpr (QMAX > 1)
    if (nq > 1) out[1] = scan_mixed<BETA, 1>(wr, nr, rs, bank, nrm, rho);
}

// The mixed-rate tables of one query head at tq_, from qr = Pi q and qs = S q;
// cbn / cbw: the narrow (2^BETA) and wide (2^(BETA+1)) codebooks. Each thread
// keeps one table position and walks the key values with a stride of NTHR / 32,
// so a warp shares one key: codebook reads broadcast and stores hit 32 banks.
template <int BETA, int NTHR>
__device__ __forceinline__ void build_tables_mixed(const float *qr, const float *qs, float *tq_, const float *cbn,
                                                   const float *cbw, int tid, float kappa) {
  using M = MixedKeys<BETA>;
  constexpr int LW = 1 << (BETA + 1), LN = 1 << BETA;
  const int pos = tid & 31, k0 = tid >> 5;
  constexpr int KS = NTHR / 32;
  {   // wide: position pos = coordinates 2 pos, 2 pos + 1
    const float q0 = qr[2 * pos], q1 = qr[2 * pos + 1];
    for (int key = k0; key < (1 << M::KW); key += KS)
      tq_[key * 32 + pos] = fmaf(q1, cbw[key >> (BETA + 1)], q0 * cbw[key & (LW - 1)]);
  }
  {   // narrow: position pos (mod the key count) = coordinates 64 + CN p .. 64 + CN p + CN - 1
    const int pn = pos & (M::NKN - 1);
    float qn[M::CN];
#pragma unroll
    for (int c = 0; c < M::CN; ++c) qn[c] = qr[64 + M::CN * pn + c];
    float *tn = tq_ + M::kNarrow / 4;
    for (int key = k0; key < 16; key += KS) {
      float v = qn[0] * cbn[key & (LN - 1)];
#pragma unroll
      for (int c = 1; c < M::CN; ++c) v = fmaf(qn[c], cbn[(key >> (BETA * c)) & (LN - 1)], v);
      tn[key * 32 + pos] = v;
    }
  }
  {   // signs: position pos (mod 16) = 8 sign bits, +-kappa (S q)_i
    const int t = pos & 15;
    float sv[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) sv[c] = kappa * qs[8 * t + c];
    float *ts = tq_ + M::kSign / 4;
    for (int key = k0; key < 256; key += KS) {
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) v += ((key >> c) & 1) ? sv[c] : -sv[c];
      ts[key * 32 + pos] = v;
    }
  }
}

}  // namespace scan
}  // namespace tq
