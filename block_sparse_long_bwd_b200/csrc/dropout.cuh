// Seeded attention dropout: the keep decisions of the attended probabilities.
//
// The pages ask for stateless, seeded dropout so that a recomputed pass
// draws the same noise ([gitcode page] "梯度检查点的实现方式"; the rate is the
// encoder's attention_dropout_rate, "BigBirdEncoder 的关键参数").  Every pass
// regenerates the decisions from (seed, b, h, t, u): nothing is stored.
//
// Keep rule of element (b, h, query token t, key token u): Philox4x32-10 with
// counter words (u >> 4, t, h, b) and key words (seed lo, seed hi) yields 16
// bytes (little-endian, words in order) for the key tokens
// 16 (u >> 4) .. 16 (u >> 4) + 15; byte u & 15 keeps the element when it is
// >= thr (Problem::drop_thr, the rate times 256 rounded).
//
// One call thus covers 16 consecutive keys of one query row: the forward
// and dQ softmax threads (one query row each) need four calls per 64-key
// tile.  The dK/dV threads own key rows; a warp there draws, per 64-query
// tile, the rows of its 32 keys (four calls a lane) and transposes the
// 32 x 32 bit blocks with shuffles.
//
// Optionally (Problem::keep_bits, a caller buffer) the forward also stores
// the decisions it draws, one bit per attended element, and the two
// backward passes load them instead of drawing them again: the same bits,
// so the same results, for a word load where three Philox calls were.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace bb {

// Philox4x32 with 10 rounds (J. K. Salmon, M. A. Moraes, R. O. Dror and
// D. E. Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011).  A
// round forms the 64-bit products M0 c0 and M1 c2 and outputs
// (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)); the key
// advances by the Weyl increments between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)c.x * kM0;
    const uint64_t p1 = (uint64_t)c.z * kM1;
    c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1,
                   (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
    k0 += kW0;
    k1 += kW1;
  }
  return c;
}

// Bit i (i < 4) set when byte i of w is >= the byte threshold (thr4 holds
// the threshold in each byte).
__device__ __forceinline__ uint32_t keep4(uint32_t w, uint32_t thr4) {
  const uint32_t ge = __vcmpgeu4(w, thr4) & 0x01010101u;  // 1 per kept byte
  // Gather the bytes' low bits (positions 0, 8, 16, 24) into bits 24..27.
  return (ge * 0x01020408u) >> 24;
}

// 16 keep bits of one Philox call: bit j for byte j (key 16 g + j).
__device__ __forceinline__ uint32_t keep16(uint4 w, uint32_t thr4) {
  return keep4(w.x, thr4) | (keep4(w.y, thr4) << 4) | (keep4(w.z, thr4) << 8) |
         (keep4(w.w, thr4) << 12);
}

__device__ __forceinline__ uint32_t keep_thr4(const Problem& p) {
  return p.drop_thr * 0x01010101u;
}

// Keep bits of query token t over the 16 key tokens of group g.
__device__ __forceinline__ uint32_t keep_group(const Problem& p, int b, int h, int t, int g,
                                               uint32_t thr4) {
  return keep16(philox4x32_10(make_uint4((uint32_t)g, (uint32_t)t, (uint32_t)h, (uint32_t)b),
                              (uint32_t)p.drop_seed, (uint32_t)(p.drop_seed >> 32)),
                thr4);
}

// 64 keep bits of query token t over key tile kt (64 tokens: bit e is key
// 64 kt + e).
__device__ __forceinline__ uint64_t keep_row64(const Problem& p, int b, int h, int t, int kt) {
  const uint32_t thr4 = keep_thr4(p);
  const uint32_t lo = keep_group(p, b, h, t, 4 * kt, thr4) |
                      (keep_group(p, b, h, t, 4 * kt + 1, thr4) << 16);
  const uint32_t hi = keep_group(p, b, h, t, 4 * kt + 2, thr4) |
                      (keep_group(p, b, h, t, 4 * kt + 3, thr4) << 16);
  return ((uint64_t)hi << 32) | lo;
}

// 32 keep bits of query token t over the keys of column half hc of key tile
// kt (bit e is key 64 kt + 32 hc + e): the half of keep_row64 a warp that
// owns one column half needs.
__device__ __forceinline__ uint32_t keep_row32(const Problem& p, int b, int h, int t, int kt,
                                               int hc) {
  const uint32_t thr4 = keep_thr4(p);
  return keep_group(p, b, h, t, 4 * kt + 2 * hc, thr4) |
         (keep_group(p, b, h, t, 4 * kt + 2 * hc + 1, thr4) << 16);
}

// One element's decision (the CUDA-core kernels).
__device__ __forceinline__ bool keep_one(const Problem& p, int b, int h, int t, int u) {
  return (keep_group(p, b, h, t, u >> 4, keep_thr4(p)) >> (u & 15)) & 1u;
}

// Transpose of a 32 x 32 bit matrix held one row per lane (bit j of lane i is
// element (i, j)): afterwards bit j of lane i is element (j, i).  Each stage
// swaps the off-diagonal s x s blocks of every 2s x 2s block.  All 32 lanes
// must call it.
__device__ __forceinline__ uint32_t transpose32(uint32_t x, int lane) {
  const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const int s = 16 >> k;
    const uint32_t m = masks[k];
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, s);
    x = (lane & s) ? ((x & ~m) | ((y >> s) & m)) : ((x & m) | ((y & m) << s));
  }
  return x;
}

// dK/dV: keep bits of the warp's 32 key tokens u0 .. u0 + 31 (u0 a multiple
// of 32) against the 32 query tokens t0 .. t0 + 31: bit j of the result is
// this lane's key u0 + lane against query t0 + j.  All 32 lanes must call it.
__device__ __forceinline__ uint32_t keep_cols32(const Problem& p, int b, int h, int u0, int t0,
                                                int lane) {
  const uint32_t thr4 = keep_thr4(p);
  const int g = u0 >> 4;
  const uint32_t r = keep_group(p, b, h, t0 + lane, g, thr4) |
                     (keep_group(p, b, h, t0 + lane, g + 1, thr4) << 16);
  return transpose32(r, lane);
}

// dK/dV: keep bits of the warp's 32 key tokens u0 .. u0 + 31 (u0 a multiple
// of 32) against the 64 query tokens t0 .. t0 + 63.  Returns, for this lane's
// key u0 + lane, bit j of lo = query t0 + j and bit j of hi = query
// t0 + 32 + j.  All 32 lanes must call it.
__device__ __forceinline__ void keep_cols64(const Problem& p, int b, int h, int u0, int t0,
                                            int lane, uint32_t& lo, uint32_t& hi) {
  const uint32_t thr4 = keep_thr4(p);
  const int g = u0 >> 4;
  const uint32_t ra = keep_group(p, b, h, t0 + lane, g, thr4) |
                      (keep_group(p, b, h, t0 + lane, g + 1, thr4) << 16);
  const uint32_t rb = keep_group(p, b, h, t0 + 32 + lane, g, thr4) |
                      (keep_group(p, b, h, t0 + 32 + lane, g + 1, thr4) << 16);
  lo = transpose32(ra, lane);
  hi = transpose32(rb, lane);
}

// ---- stored keep decisions ------------------------------------------------

// Slot of the attended pair (query block i, key block u) among the
// keep_slots slots of one (b, h).  Query blocks 0 and nb - 1 attend every
// key block: slots u and nb + u.  A middle block i has 5 + r slots from
// 2 nb + (i - 1)(5 + r); its pair takes the count of members of
// {0, i - 1 (if >= 2), i, i + 1 (if <= nb - 2)} and of table entries of row i
// in [0, nb) below u.  Every attended block below u is counted, so distinct
// attended blocks get distinct slots, and the count is at most 4 + r, so
// it stays inside the row's stride (for any table, corrupt ones included).
__device__ __forceinline__ int keep_slot(const Problem& p, int h, int i, int u) {
  const int nb = p.nb;
  if (i == 0) return u;
  if (i == nb - 1) return nb + u;
  int c = (u > 0) + (i >= 2 && i - 1 < u) + (i < u) + (i + 1 <= nb - 2 && i + 1 < u);
  const int32_t* row = p.rand_idx + ((size_t)h * nb + i) * p.r;
  // Four independent loads per round, so their latencies overlap.
  for (int a = 0; a < p.r; a += 4) {
    int j[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) j[x] = a + x < p.r ? __ldg(row + a + x) : -1;
#pragma unroll
    for (int x = 0; x < 4; ++x) c += (j[x] >= 0 && j[x] < u);
  }
  return 2 * nb + (i - 1) * (5 + p.r) + c;
}

__device__ __forceinline__ int keep_log2_bs(const Problem& p) {
  return p.bs == 32 ? 5 : (p.bs == 64 ? 6 : 7);
}

// Slot of query token tq against the block of key token k0.
__device__ __forceinline__ int keep_slot_of(const Problem& p, int h, int tq, int k0) {
  const int sh = keep_log2_bs(p);
  return keep_slot(p, h, tq >> sh, k0 >> sh);
}

// Word of the stored bits holding query token tq against the 32 key tokens
// k0 .. k0 + 31 (k0 a multiple of 32) in slot `slot` of (b, h) = bh: a slot
// is bs x bs bits, query row major, bs / 32 words per row.
__device__ __forceinline__ uint32_t* keep_at(const Problem& p, int bh, int slot, int tq, int k0) {
  const int wpr = p.bs >> 5;  // words per row
  const int q = tq & (p.bs - 1), w = (k0 & (p.bs - 1)) >> 5;
  return p.keep_bits + ((size_t)bh * p.keep_slots + slot) * (size_t)(wpr * p.bs) + q * wpr + w;
}

__device__ __forceinline__ uint32_t* keep_ptr(const Problem& p, int bh, int h, int tq, int k0) {
  return keep_at(p, bh, keep_slot_of(p, h, tq, k0), tq, k0);
}

// The table row of one query block held in registers (up to four random
// blocks per row, the common case), so that the slots of a row's tiles cost
// no loads: a softmax thread's query block is the same on every tile of an
// item.  With r > 4 the slots are looked up in the table.
struct KeepRow {
  int i;       // query block
  int id[4];   // table row i (-1 past r, or for the global blocks)
};

__device__ __forceinline__ KeepRow keep_row(const Problem& p, int h, int tq) {
  KeepRow kr;
  kr.i = tq >> keep_log2_bs(p);
  const bool mid = kr.i > 0 && kr.i < p.nb - 1 && p.r <= 4;
  const int32_t* row = p.rand_idx + ((size_t)h * p.nb + (mid ? kr.i : 0)) * p.r;
#pragma unroll
  for (int x = 0; x < 4; ++x) kr.id[x] = (mid && x < p.r) ? __ldg(row + x) : -1;
  return kr;
}

// keep_slot(p, h, kr.i, u).
__device__ __forceinline__ int keep_slot_row(const Problem& p, int h, const KeepRow& kr,
                                             int u) {
  const int nb = p.nb, i = kr.i;
  if (i == 0) return u;
  if (i == nb - 1) return nb + u;
  if (p.r > 4) return keep_slot(p, h, i, u);
  int c = (u > 0) + (i >= 2 && i - 1 < u) + (i < u) + (i + 1 <= nb - 2 && i + 1 < u);
#pragma unroll
  for (int x = 0; x < 4; ++x) c += (unsigned)kr.id[x] < (unsigned)u;  // -1 never counts
  return 2 * nb + (i - 1) * (5 + p.r) + c;
}

// The slots of a row's attended column halves m2 of key tile kt (one block
// for both halves when the block size is 64 or more; -1 for an unattended
// half).
__device__ __forceinline__ void keep_slots64(const Problem& p, int h, const KeepRow& kr, int kt,
                                             int m2, int& s0, int& s1) {
  const int sh = keep_log2_bs(p);
  s0 = (m2 & 1) ? keep_slot_row(p, h, kr, (kt * 64) >> sh) : -1;
  s1 = (m2 & 2) ? ((p.bs >= 64 && (m2 & 1)) ? s0 : keep_slot_row(p, h, kr, (kt * 64 + 32) >> sh))
                : -1;
}

// Forward: store the decisions of query token tq over key tile kt (bit e of
// bits: key 64 kt + e) into the slots keep_slots64 gave.  With both halves
// in one block the two words are adjacent: one 8-byte store.
__device__ __forceinline__ void keep_store64(const Problem& p, int bh, int tq, int kt, int s0,
                                             int s1, uint64_t bits) {
  const int k0 = kt * 64;
  if (s0 >= 0 && s1 >= 0 && p.bs >= 64) {
    *reinterpret_cast<uint2*>(keep_at(p, bh, s0, tq, k0)) =
        make_uint2((uint32_t)bits, (uint32_t)(bits >> 32));
  } else {
    if (s0 >= 0) *keep_at(p, bh, s0, tq, k0) = (uint32_t)bits;
    if (s1 >= 0) *keep_at(p, bh, s1, tq, k0 + 32) = (uint32_t)(bits >> 32);
  }
}

// Multiplier of a probability under the keep bit e of `keep`: 1 / keep
// probability (sc) where kept, 0 where dropped.
__device__ __forceinline__ float keep_factor(uint32_t keep, int e, float sc) {
  return ((keep >> e) & 1u) ? sc : 0.f;
}

// dQ: the stored counterpart of keep_row64 for the attended halves m2
// (unattended halves read as 0).
__device__ __forceinline__ uint64_t keep_load64(const Problem& p, int bh, int h,
                                                const KeepRow& kr, int tq, int kt, int m2) {
  int s0, s1;
  keep_slots64(p, h, kr, kt, m2, s0, s1);
  const int k0 = kt * 64;
  if (s0 >= 0 && s1 >= 0 && p.bs >= 64) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(keep_at(p, bh, s0, tq, k0)));
    return ((uint64_t)w.y << 32) | w.x;
  }
  const uint32_t lo = s0 >= 0 ? __ldg(keep_at(p, bh, s0, tq, k0)) : 0u;
  const uint32_t hi = s1 >= 0 ? __ldg(keep_at(p, bh, s1, tq, k0 + 32)) : 0u;
  return ((uint64_t)hi << 32) | lo;
}

}  // namespace bb
