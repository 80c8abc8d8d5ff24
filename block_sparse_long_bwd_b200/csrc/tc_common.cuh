// Work-item description shared by the tensor-core kernels.
//
// A query-side item pairs two query blocks of one (b, h) in one 128-row MMA
// tile (rows 0-63: half 0, rows 64-127: half 1):
//  * middle pair (i, i+1), i = 1, 3, 5, ...: the key blocks visited are the
//    union of the two attended sets A(i), A(i+1) ({0, i-1, i, i+1, nb-1} and
//    the row's random blocks); each carries a 2-bit mask of the halves that
//    attend it.  The last pair has an empty half when nb - 2 is odd.
//  * global chunk c: query blocks 0 and nb-1, which attend every key block,
//    over key blocks [c * kChunk, (c + 1) * kChunk); the kernels write
//    per-chunk partials that a second kernel merges.
#pragma once

#include "sm100.cuh"

namespace bb {

constexpr int kBS = 64;                               // block size (tokens)
constexpr int kMaxT = 32;                             // key blocks per item
constexpr int kChunk = 8;                             // key blocks per chunk
constexpr uint32_t kTileBytes = kBS * kHeadDim * 2;   // one 64 x 64 bf16 tile
constexpr int kPartStride = 68;                       // floats per partial row

struct ItemList {
  int n;
  int global;   // 1 = global chunk
  int bh, b;
  int blk[2];   // query block of half 0 / half 1 (-1: half unused)
  int chunk;
  int16_t tile[kMaxT];
  uint8_t mask[kMaxT];
};

struct PairArgs {
  Problem p;
  int npairs, nchunks, items;
};

inline PairArgs make_pair_args(const Problem& p) {
  PairArgs a;
  a.p = p;
  a.nchunks = (p.nb + kChunk - 1) / kChunk;
  a.npairs = p.nb > 2 ? (p.nb - 1) / 2 : 0;
  a.items = p.B * p.H * (a.npairs + a.nchunks);
  return a;
}

__device__ __forceinline__ void list_add(ItemList& L, int j, int bit) {
  for (int c = 0; c < L.n; ++c)
    if (L.tile[c] == j) {
      L.mask[c] |= (uint8_t)bit;
      return;
    }
  L.tile[L.n] = (int16_t)j;
  L.mask[L.n] = (uint8_t)bit;
  ++L.n;
}

// Fills L for query-side item `item` (items are (b, h)-major; within one
// (b, h) the global chunks come first, then the middle pairs).
__device__ inline void build_pair_item(const PairArgs& a, int item,
                                       ItemList& L) {
  const Problem& p = a.p;
  const int nb = p.nb;
  const int per = a.npairs + a.nchunks;
  const int bh = item / per, loc = item % per;
  L.n = 0;
  L.bh = bh;
  L.b = bh / p.H;
  const int h = bh % p.H;
  if (loc < a.nchunks) {
    L.global = 1;
    L.chunk = loc;
    L.blk[0] = 0;
    L.blk[1] = nb > 1 ? nb - 1 : -1;
    const int bits = nb > 1 ? 3 : 1;
    const int j1 = min(nb, (loc + 1) * kChunk);
    for (int j = loc * kChunk; j < j1; ++j) {
      L.tile[L.n] = (int16_t)j;
      L.mask[L.n] = (uint8_t)bits;
      ++L.n;
    }
    return;
  }
  L.global = 0;
  L.chunk = 0;
  const int i0 = 1 + 2 * (loc - a.nchunks);
  L.blk[0] = i0;
  L.blk[1] = (i0 + 1 <= nb - 2) ? i0 + 1 : -1;
  for (int half = 0; half < 2; ++half) {
    const int i = L.blk[half];
    if (i < 0) continue;
    const int bit = 1 << half;
    list_add(L, 0, bit);
    list_add(L, i - 1, bit);
    list_add(L, i, bit);
    list_add(L, i + 1, bit);
    list_add(L, nb - 1, bit);
    const int32_t* row = p.rand_idx + ((size_t)h * nb + i) * p.r;
    for (int c = 0; c < p.r; ++c) {
      const int j = row[c];
      if (j == -1) continue;
      if (j < 0 || j >= nb) {
        set_status(p.status, BB_ERR_BAD_TABLE);
        continue;
      }
      list_add(L, j, bit);
    }
  }
}

// Validity bitmap of the 64 keys of key block j (bit k set = attend).
__device__ __forceinline__ uint64_t key_bits(const Problem& p, int b, int j) {
  const uint4* m4 = reinterpret_cast<const uint4*>(
      p.key_mask + (size_t)b * p.L + (size_t)j * kBS);
  uint64_t bits = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 w = __ldg(m4 + c);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int by = 0; by < 4; ++by)
        if ((ws[e] >> (8 * by)) & 0xFFu) bits |= 1ull << (16 * c + 4 * e + by);
  }
  return bits;
}

// TMA/tcgen05 path conditions shared by forward and backward.
inline bool tc_shape_ok(const Problem& p) {
  return p.dtype == BB_BF16 && p.bs == kBS && p.d == kHeadDim &&
         10 + 2 * p.r <= kMaxT && (size_t)p.B * p.H * p.L < (1ull << 31);
}

}  // namespace bb
