// Work items shared by the tensor-core kernels.
//
// The kernels work in 64-token tiles (one 64 x 64 bf16 TMA box) whatever the
// block size (32, 64 or 128).  An item is one 128-row MMA tile made of two
// 64-row tiles ("halves"), split into four 32-row groups g = 0..3 (group g =
// TMEM lane quarter g, so each softmax warp owns one group).  A group lies in
// a single block of the pattern (blocks are >= 32 tokens).  Each tile an
// item visits (a key tile on the query side, a query tile on the key side)
// carries an 8-bit mask: bit 2g + c says "row group g attends the 32
// columns c of this tile" (c = 0: columns 0-31, c = 1: columns 32-63).
//
// Query-side items (forward and dQ):
//  * middle window w: rows [128 w, 128 w + 128) (query tiles 2w, 2w + 1);
//    every group whose block is a middle block (1 .. nb - 2) visits the key
//    tiles of its attended set A(i) = {0, i-1, i, i+1, nb-1} U rand(i);
//    groups of the global blocks, or past L, are masked off.  Only windows
//    that hold a middle block are items.
//  * global item gi, chunk c: the 64-row tiles holding the global blocks 0
//    and nb-1 (at most four, paired two per item) over key tiles
//    [8c, 8c + 8); those rows attend every key, so the kernels write
//    per-chunk partials that a second kernel merges.
// Key-side items (dK / dV) mirror this with key and query swapped: a middle
// window walks the merged transposed-adjacency lists of its key blocks; the
// global key blocks are split over chunks of query tiles.
#pragma once

#include "sm100.cuh"

namespace bb {

constexpr int kTile = 64;                             // tokens per tile
// From this length on, the global key blocks' P^T and dS^T carry a bf16
// low part in the dK/dV pass (they sum over every query row).
constexpr int kSplitMinL = 16384;
constexpr int kMaxT = 64;                             // tiles per item
constexpr int kChunk = 8;                             // tiles per chunk (split rows)
// CTAs the balance rule below plans for: two per SM of a B200 (148 SMs).
constexpr int kBalanceCtas = 2 * 148;
constexpr uint32_t kTileBytes = kTile * kHeadDim * 2; // one 64 x 64 bf16 tile
constexpr int kPartStride = 68;                       // floats per fwd partial row

// Geometry of the tiled problem (host and device).
struct Geom {
  int bs, nb, nt;       // block size, blocks, 64-token tiles
  int bs_shift;         // log2(bs): bs is 32, 64 or 128 on this path
  int w_first, n_mid;   // middle windows
  int ngt;              // tiles holding global blocks (ascending in gt)
  int gt[4];
  int n_git;            // global items = ceil(ngt / 2)
  int chunk;            // tiles per chunk of a global item
  int nchunks;          // chunks of the tile range [0, nt)
  int per_bh;           // items per (b, h): n_mid + n_git * nchunks
};

// Geometry for L tokens in blocks of bs; chunk = tiles per chunk of a global
// item (0: kChunk).
__host__ __device__ inline Geom make_geom(int L, int bs, int chunk = 0) {
  Geom g;
  g.bs = bs;
  g.bs_shift = bs == 32 ? 5 : bs == 64 ? 6 : 7;
  g.nb = L / bs;
  g.nt = L / kTile;
  // Windows intersecting the middle tokens [bs, L - bs).
  if (g.nb >= 3) {
    g.w_first = bs / 128;
    const int w_last = (L - bs - 1) / 128;
    g.n_mid = w_last - g.w_first + 1;
  } else {
    g.w_first = 0;
    g.n_mid = 0;
  }
  // Tiles holding rows of blocks 0 and nb - 1.
  g.ngt = 0;
  const int tpb = bs >= kTile ? bs / kTile : 1;  // tiles per block
  for (int t = 0; t < tpb; ++t) g.gt[g.ngt++] = t;
  for (int t = g.nt - tpb; t < g.nt; ++t) {
    bool dup = false;
    for (int c = 0; c < g.ngt; ++c) dup |= (g.gt[c] == t);
    if (!dup && t >= 0) g.gt[g.ngt++] = t;
  }
  g.n_git = (g.ngt + 1) / 2;
  g.chunk = chunk > 0 ? chunk : kChunk;
  g.nchunks = (g.nt + g.chunk - 1) / g.chunk;
  g.per_bh = g.n_mid + g.n_git * g.nchunks;
  return g;
}

// Tiles per chunk of a global item for problem p.  A global row visits every
// key tile (a global key block every query tile).  Long chunks mean fewer
// partials to write and merge, but an item must stay shorter than the work
// each CTA of the launch gets (middle windows estimated at 8 + r tiles).
//  - One tile list holds the whole row (nt <= kMaxT) and it balances: the
//    item runs whole, writes its rows directly, and nothing is merged.
//  - Else chunks of kMaxT tiles when they balance, of kChunk otherwise.
// Chunk partials are merged in a fixed order by a launch of their own.
__host__ __device__ inline int global_chunk_tiles(const Problem& p) {
  const Geom g = make_geom(p.L, p.bs);
  const long long work = (long long)p.B * p.H *
                         ((long long)g.n_mid * (8 + p.r) + (long long)g.n_git * g.nt);
  if (g.nt <= kMaxT && work >= (long long)kBalanceCtas * g.nt) return g.nt;
  if (g.nt > kMaxT && work >= (long long)kBalanceCtas * kMaxT) return kMaxT;
  return kChunk;
}

// Query-side geometry (forward, dQ).
__host__ __device__ inline Geom make_geom(const Problem& p) {
  return make_geom(p.L, p.bs, global_chunk_tiles(p));
}

// Key-side geometry (dK/dV): the same items, except that from the length
// where the global key blocks run in a launch of their own their chunks are
// kChunk query tiles (that launch holds only them and needs many items).
__host__ __device__ inline Geom make_kgeom(const Problem& p) {
  return make_geom(p.L, p.bs, p.L >= kSplitMinL ? kChunk : global_chunk_tiles(p));
}

// Block of token row `tok`.
__host__ __device__ inline int block_of(const Geom& g, int tok) {
  return tok >> g.bs_shift;
}

// Tiles covering block j and the column halves of each it spans:
// bs 32 -> one tile, one half; 64 -> one tile, both halves; 128 -> two tiles.
template <typename F>
__host__ __device__ __forceinline__ void for_block_tiles(const Geom& g, int j, F f) {
  if (g.bs == 32) {
    f(j >> 1, 1 << (j & 1));
  } else if (g.bs == 64) {
    f(j, 3);
  } else {
    f(2 * j, 3);
    f(2 * j + 1, 3);
  }
}

// The tiles an item visits, planned once per call (one per (head, item):
// lists do not depend on the batch index) and copied into shared memory by
// the producer with one bulk copy.  208 bytes, a multiple of 16.
struct __align__(16) TileList {
  int n;
  int pad[3];
  int16_t tile[kMaxT];
  uint8_t mask[kMaxT];
};
static_assert(sizeof(TileList) % 16 == 0, "bulk-copy size");

// What an item covers, computable from its index alone.
struct ItemMeta {
  int bh, b, h, loc;
  int global;   // 1 = global item
  int t[2];     // row tile of half 0 / 1 (-1: absent)
  int gvalid;   // 4-bit: groups whose rows this item produces
  int gi, chunk;
};

struct PairArgs {
  Problem p;
  Geom geo;
  int items;
};

inline PairArgs make_pair_args(const Problem& p) {
  PairArgs a;
  a.p = p;
  a.geo = make_geom(p);
  a.items = p.B * p.H * a.geo.per_bh;
  return a;
}

__host__ __device__ __forceinline__ void list_add(TileList& L, int tile, int bits) {
  for (int c = 0; c < L.n; ++c)
    if (L.tile[c] == tile) {
      L.mask[c] |= (uint8_t)bits;
      return;
    }
  if (L.n >= kMaxT) return;  // host validation keeps lists within kMaxT
  L.tile[L.n] = (int16_t)tile;
  L.mask[L.n] = (uint8_t)bits;
  ++L.n;
}

// Row tiles and valid groups of a window / global item.
__host__ __device__ __forceinline__ void item_rows(const Geom& g, bool global, int w_or_gi,
                                          int (&t)[2], int& gvalid) {
  if (!global) {
    t[0] = 2 * w_or_gi;
    t[1] = 2 * w_or_gi + 1 < g.nt ? 2 * w_or_gi + 1 : -1;
  } else {
    t[0] = g.gt[2 * w_or_gi];
    t[1] = 2 * w_or_gi + 1 < g.ngt ? g.gt[2 * w_or_gi + 1] : -1;
  }
  gvalid = 0;
  for (int gr = 0; gr < 4; ++gr) {
    const int tt = t[gr >> 1];
    if (tt < 0) continue;
    const int blk = block_of(g, tt * kTile + 32 * (gr & 1));
    const bool is_global = (blk == 0 || blk == g.nb - 1);
    if (global == is_global) gvalid |= 1 << gr;
  }
}

// Expand a 4-bit group set into mask bits for column halves `halves`.
__host__ __device__ __forceinline__ int expand_groups(int groups, int halves) {
  int m = 0;
  for (int gr = 0; gr < 4; ++gr)
    if (groups & (1 << gr)) m |= halves << (2 * gr);
  return m;
}

// Metadata of item `item` ((b, h)-major; within one (b, h) the global items'
// chunks come first, then the middle windows).  Same decoding on both sides.
// Item at (b, h, loc): no divisions (at most two global items per (b, h)).
__host__ __device__ __forceinline__ ItemMeta item_meta_at(const Geom& g, int b, int h,
                                                          int H, int loc) {
  ItemMeta m;
  m.b = b;
  m.h = h;
  m.bh = b * H + h;
  m.loc = loc;
  const int nglob = g.n_git * g.nchunks;
  if (loc < nglob) {
    m.global = 1;
    m.gi = loc >= g.nchunks ? 1 : 0;
    m.chunk = loc - m.gi * g.nchunks;
    item_rows(g, true, m.gi, m.t, m.gvalid);
  } else {
    m.global = 0;
    m.gi = 0;
    m.chunk = 0;
    item_rows(g, false, g.w_first + (loc - nglob), m.t, m.gvalid);
  }
  return m;
}

__host__ __device__ __forceinline__ ItemMeta item_meta(const Geom& g, int H, int item) {
  const int bh = item / g.per_bh;
  return item_meta_at(g, bh / H, bh % H, H, item % g.per_bh);
}

// Next work item of a launch, taken from its counter: the locs [loc0, loc0 +
// nloc) of every (b, h), longest items first so the short ones fill the end
// of the launch: middle windows, then short global chunks; global items of
// more than kChunk tiles, which are longer than a window, before the
// windows.  False when none is left.
__device__ __forceinline__ bool next_work(const Geom& g, int B, int H, int loc0, int nloc,
                                          int* ctr, int& b, int& h, int& loc) {
  const int nglob = g.n_git * g.nchunks;
  const int mlo = max(loc0, nglob);
  const int nmid = max(0, loc0 + nloc - mlo);
  const int ngl = nloc - nmid;
  const int BH = B * H;
  const int w = atomicAdd(ctr, 1);
  if (w >= BH * nloc) return false;
  int bh;
  const bool glob_first = g.chunk > kChunk;
  const int nfirst = glob_first ? ngl : nmid;
  if (w < BH * nfirst) {
    bh = w / nfirst;
    loc = (glob_first ? loc0 : mlo) + w % nfirst;
  } else {
    const int w2 = w - BH * nfirst;
    const int nsecond = glob_first ? nmid : ngl;
    bh = w2 / nsecond;
    loc = (glob_first ? mlo : loc0) + w2 % nsecond;
  }
  b = bh / H;
  h = bh % H;
  return true;
}

// Plans the key tiles of query-side item (h, loc) into L.  Returns false if
// the random table held an entry outside [-1, nb) (ignored).
__host__ __device__ inline bool build_tile_list(const Problem& p, const Geom& g,
                                                int h, int loc, TileList& L) {
  ItemMeta m = item_meta(g, p.H, h * g.per_bh + loc);  // b = 0: lists ignore b
  L.n = 0;
  bool table_ok = true;
  if (m.global) {
    const int bits = expand_groups(m.gvalid, 3);
    const int j1 = g.nt < (m.chunk + 1) * g.chunk ? g.nt : (m.chunk + 1) * g.chunk;
    for (int j = m.chunk * g.chunk; j < j1; ++j) {
      L.tile[L.n] = (int16_t)j;
      L.mask[L.n] = (uint8_t)bits;
      ++L.n;
    }
    return true;
  }
  const int nb = g.nb;
  for (int gr = 0; gr < 4; ++gr) {
    if (!(m.gvalid & (1 << gr))) continue;
    const int i = block_of(g, m.t[gr >> 1] * kTile + 32 * (gr & 1));
    const int gbits = 1 << (2 * gr);
    auto add_block = [&](int j) {
      for_block_tiles(g, j, [&](int tile, int halves) {
        list_add(L, tile, halves * gbits);
      });
    };
    add_block(0);
    add_block(i - 1);
    add_block(i);
    add_block(i + 1);
    add_block(nb - 1);
    const int32_t* row = p.rand_idx + ((size_t)h * nb + i) * p.r;
    for (int c = 0; c < p.r; ++c) {
      const int j = row[c];
      if (j == -1) continue;
      if (j < 0 || j >= nb) {
        table_ok = false;
        continue;
      }
      add_block(j);
    }
  }
  return table_ok;
}

// Key-side walk entries: query tile in the low 16 bits, mask in bits 16-23.
__host__ __device__ __forceinline__ uint32_t kentry(int tile, int mask) {
  return (uint32_t)tile | ((uint32_t)mask << 16);
}

// Walk of one key-side item over the query tiles that attend it, with the
// 8-bit mask (bit 2g + c: key group g is attended by query rows of column
// half c of the query tile).  Every role of the dK/dV kernel runs its own
// copy; all copies see the same sequence.
struct KeyWalk {
  int bh, b;
  int t[2];       // key tile of half 0 / 1 (-1: absent)
  int gvalid;
  int global, gi, chunk;
  // global: query tiles [cur, end)
  int cur, end, gmask;
  // middle: up to four sorted CSR lists (one per distinct key block)
  int nl;
  const int* lp[4];
  int ln[4], li[4], lg[4];
  int bs;
  int pend_tile, pend_mask;  // block 128: second tile of a query block

  __host__ __device__ void init(const Geom& g, int H, const int* csr_offs,
                                const int* csr_list, int csr_cap, int item) {
    const int h = item_meta(g, H, item).h;
    init_head(g, H, csr_offs + (size_t)h * (g.nb + 1), csr_list + (size_t)h * csr_cap, item);
  }
  // Same, given the item's head's CSR offsets [nb + 1] and lists.
  __host__ __device__ void init_head(const Geom& g, int H, const int* offs, const int* list,
                                     int item) {
    const ItemMeta m = item_meta(g, H, item);
    bh = m.bh;
    b = m.b;
    bs = g.bs;
    pend_tile = -1;
    pend_mask = 0;
    nl = 0;
    global = m.global;
    gi = m.gi;
    chunk = m.chunk;
    t[0] = m.t[0];
    t[1] = m.t[1];
    gvalid = m.gvalid;
    if (global) {
      gmask = expand_groups(gvalid, 3);
      cur = chunk * g.chunk;
      end = g.nt < cur + g.chunk ? g.nt : cur + g.chunk;
      return;
    }
    for (int gr = 0; gr < 4; ++gr) {
      if (!(gvalid & (1 << gr))) continue;
      const int j = block_of(g, t[gr >> 1] * kTile + 32 * (gr & 1));
      int x = 0;
      while (x < nl && lp[x] != list + offs[j]) ++x;
      if (x == nl) {
        lp[nl] = list + offs[j];
        ln[nl] = offs[j + 1] - offs[j];
        li[nl] = 0;
        lg[nl] = 0;
        ++nl;
      }
      lg[x] |= 1 << gr;
    }
  }

  // Smallest unconsumed query block over the lists (INT_MAX when done) and
  // the groups whose lists hold it.
  __host__ __device__ __forceinline__ int peek(int& groups) const {
    int qb = 0x7FFFFFFF;
    groups = 0;
    for (int x = 0; x < nl; ++x)
      if (li[x] < ln[x]) {
        const int v = lp[x][li[x]];
        if (v < qb) {
          qb = v;
          groups = lg[x];
        } else if (v == qb) {
          groups |= lg[x];
        }
      }
    return qb;
  }
  __host__ __device__ __forceinline__ void consume(int qb) {
    for (int x = 0; x < nl; ++x)
      if (li[x] < ln[x] && lp[x][li[x]] == qb) ++li[x];
  }

  // Next query tile and its mask; false at the end.
  __host__ __device__ bool next(int& tile, int& mask) {
    if (global) {
      if (cur >= end) return false;
      tile = cur++;
      mask = gmask;
      return true;
    }
    if (pend_tile >= 0) {
      tile = pend_tile;
      mask = pend_mask;
      pend_tile = -1;
      return true;
    }
    int groups;
    const int qb = peek(groups);
    if (qb == 0x7FFFFFFF) return false;
    consume(qb);
    if (bs == 32) {
      tile = qb >> 1;
      mask = expand_groups(groups, 1 << (qb & 1));
      // the other block of the same query tile, if attended too
      int g2;
      const int qb2 = peek(g2);
      if (qb2 != 0x7FFFFFFF && (qb2 >> 1) == tile) {
        consume(qb2);
        mask |= expand_groups(g2, 1 << (qb2 & 1));
      }
    } else if (bs == 64) {
      tile = qb;
      mask = expand_groups(groups, 3);
    } else {
      tile = 2 * qb;
      mask = expand_groups(groups, 3);
      pend_tile = 2 * qb + 1;
      pend_mask = mask;
    }
    return true;
  }
};

// Validity bitmap of the 64 keys of key tile j (bit k set = attend): one
// mask byte per lane and half, gathered by two ballots.  All 32 lanes of the
// warp must call it.
__device__ __forceinline__ uint64_t key_bits(const Problem& p, int b, int j) {
  const uint8_t* m = p.key_mask + (size_t)b * p.L + (size_t)j * kTile;
  const int lane = threadIdx.x & 31;
  const uint32_t lo = __ballot_sync(0xffffffffu, __ldg(m + lane) != 0);
  const uint32_t hi = __ballot_sync(0xffffffffu, __ldg(m + 32 + lane) != 0);
  return ((uint64_t)hi << 32) | lo;
}

// Column-validity bitmap of a tile from its two mask bits for one group
// (bit k set = column k belongs to an attended block).
__device__ __forceinline__ uint64_t half_bits(int m2) {
  return ((m2 & 1) ? 0x00000000FFFFFFFFull : 0ull) |
         ((m2 & 2) ? 0xFFFFFFFF00000000ull : 0ull);
}

// Tensor-core path conditions shared by forward and backward.
inline bool tc_shape_ok(const Problem& p) {
  if (p.dtype != BB_BF16 || p.d != kHeadDim) return false;
  if (p.bs != 32 && p.bs != 64 && p.bs != 128) return false;
  if (p.L % kTile != 0) return false;
  if ((size_t)p.B * p.H * p.L >= (1ull << 31)) return false;
  // Planner bounds: a middle item's (group, block, tile) candidates fit the
  // 128-entry sort (4 groups x (5 + r) blocks x tiles per block) and its
  // distinct tiles fit kMaxT.
  const int per = p.bs == 64 ? 2 * (5 + p.r) : 4 * (5 + p.r);
  return per <= kMaxT;
}

}  // namespace bb
