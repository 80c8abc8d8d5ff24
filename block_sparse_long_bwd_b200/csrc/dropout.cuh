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

}  // namespace bb
