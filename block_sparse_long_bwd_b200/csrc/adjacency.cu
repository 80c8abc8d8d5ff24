// Planning and preprocessing: the tensor-core kernels' tile plans (query
// side: each item's merged, ordered key tiles with group masks; key side:
// each item's walk of attending query tiles), the transposed block
// adjacency (for each key block j, the sorted query blocks i with j in A(i);
// built per head in shared memory by the backward's planning launch, or in
// global memory), and D = rowsum(dO * O) for the CUDA-core backward.
#include "tc_common.cuh"

namespace bb {
namespace {

__device__ __forceinline__ float2 load2(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

// One warp per token row; each lane reads two of the 64 elements.
template <typename T>
__global__ void __launch_bounds__(256) bwd_pre_kernel(Problem p) {
  const size_t rows = (size_t)p.B * p.H * p.L;
  const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T* O = static_cast<const T*>(p.o) + row * kHeadDim + lane * 2;
  const T* G = static_cast<const T*>(p.dout) + row * kHeadDim + lane * 2;
  const float2 o = load2(O), g = load2(G);
  float acc = o.x * g.x + o.y * g.y;
#pragma unroll
  for (int w = 16; w > 0; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
  if (lane == 0) p.D[row] = acc;
}

// Random entry a of middle row i counts toward key block j iff it is in
// range, outside {0, nb-1, i-1, i, i+1} and not a repeat of an earlier entry
// of the row (the attended set is a set).  Out-of-range entries are flagged.
__device__ __forceinline__ int random_target(const int32_t* row, int a, int i,
                                             int nb, int* status) {
  const int j = row[a];
  if (j == -1) return -1;
  if (j < 0 || j >= nb) {
    set_status(status, BB_ERR_BAD_TABLE);
    return -1;
  }
  if (j == 0 || j == nb - 1 || (j >= i - 1 && j <= i + 1)) return -1;
  for (int c = 0; c < a; ++c)
    if (row[c] == j) return -1;
  return j;
}

constexpr int kCsrThreads = 1024;

// Total list length: the inclusive scan's last element.
__device__ __forceinline__ int total_sh(const int* tsum) { return tsum[kCsrThreads - 1]; }

// One CTA per head.  Shared memory: count[nb], cursor[nb], tsum[1024] and,
// when it fits (in_smem), the head's whole list, built there and copied out
// once; otherwise the list is built in place in global memory.
__global__ void __launch_bounds__(kCsrThreads) csr_build_kernel(Problem p, int in_smem) {
  extern __shared__ int smi[];
  const int nb = p.nb, r = p.r, h = blockIdx.x, tid = threadIdx.x;
  int* cnt = smi;
  int* cur = cnt + nb;
  int* tsum = cur + nb;
  const int32_t* table = p.rand_idx + (size_t)h * nb * r;
  int* offs = p.csr_offs + (size_t)h * (nb + 1);
  int* glist = p.csr_list + (size_t)h * p.csr_cap;
  int* list = in_smem ? tsum + kCsrThreads : glist;

  for (int j = tid; j < nb; j += kCsrThreads) {
    int c;
    if (j == 0 || j == nb - 1) {
      c = nb;
    } else {
      c = 2;  // global query rows 0 and nb-1
      for (int i = j - 1; i <= j + 1; ++i) c += (i >= 1 && i <= nb - 2);
    }
    cnt[j] = c;
  }
  __syncthreads();
  for (int x = tid; x < nb * r; x += kCsrThreads) {
    const int i = x / r, a = x % r;
    if (i == 0 || i == nb - 1) continue;
    const int j = random_target(table + (size_t)i * r, a, i, nb, p.status);
    if (j >= 0) atomicAdd(&cnt[j], 1);
  }
  __syncthreads();
  // Exclusive scan: contiguous chunks per thread, then a scan of chunk sums.
  const int chunk = (nb + kCsrThreads - 1) / kCsrThreads;
  const int c0 = tid * chunk, c1 = min(nb, c0 + chunk);
  int local = 0;
  for (int j = c0; j < c1; ++j) local += cnt[j];
  tsum[tid] = local;
  __syncthreads();
  for (int step = 1; step < kCsrThreads; step <<= 1) {
    int add = tid >= step ? tsum[tid - step] : 0;
    __syncthreads();
    tsum[tid] += add;
    __syncthreads();
  }
  int run = tsum[tid] - local;  // exclusive prefix of this chunk
  for (int j = c0; j < c1; ++j) {
    const int c = cnt[j];
    cur[j] = run;
    offs[j] = run;
    cnt[j] = run;  // from here on: start offset of list j
    run += c;
  }
  if (tid == kCsrThreads - 1) offs[nb] = tsum[kCsrThreads - 1];
  __syncthreads();
  // Fill.  Global key blocks: every query block, in order.
  for (int x = tid; x < 2 * nb; x += kCsrThreads) {
    const int j = x < nb ? 0 : nb - 1;
    const int i = x % nb;
    if (x >= nb && nb == 1) continue;  // single block: j=0 already filled
    list[cur[j] + i] = i;
  }
  for (int j = tid; j < nb; j += kCsrThreads) {
    if (j == 0 || j == nb - 1) continue;
    // Structural entries (global rows, window rows) reserve their slots
    // with the same cursor the random entries below append through.
    int pos = atomicAdd(&cur[j], 2 + (j - 1 >= 1) + 1 + (j + 1 <= nb - 2));
    list[pos++] = 0;
    list[pos++] = nb - 1;
    for (int i = j - 1; i <= j + 1; ++i)
      if (i >= 1 && i <= nb - 2) list[pos++] = i;
  }
  for (int x = tid; x < nb * r; x += kCsrThreads) {
    const int i = x / r, a = x % r;
    if (i == 0 || i == nb - 1) continue;
    const int j = random_target(table + (size_t)i * r, a, i, nb, p.status);
    if (j >= 0) list[atomicAdd(&cur[j], 1)] = i;
  }
  __syncthreads();
  // Sort each non-global list (short: 2 + 3 + random in-degree).
  for (int j = tid; j < nb; j += kCsrThreads) {
    if (j == 0 || j == nb - 1) continue;
    const int o0 = in_smem ? cnt[j] : offs[j];
    int* L = list + o0;
    const int n = (in_smem ? (j + 1 < nb ? cnt[j + 1] : total_sh(tsum)) : offs[j + 1]) - o0;
    for (int a = 1; a < n; ++a) {
      int x = L[a], c = a - 1;
      while (c >= 0 && L[c] > x) {
        L[c + 1] = L[c];
        --c;
      }
      L[c + 1] = x;
    }
  }
  if (in_smem) {
    __syncthreads();
    const int total = total_sh(tsum);
    for (int x = tid; x < total; x += kCsrThreads) glist[x] = list[x];
  }
}

constexpr int kPlanWarps = 4;
constexpr int kStageCap = 512;  // CSR entries staged per warp (key side)

// Bitonic sort of 128 ints in shared memory by one warp.
__device__ __forceinline__ void warp_sort128(int* v, int lane) {
  for (int k = 2; k <= 128; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = lane + 32 * r;
        const int x = i ^ j;
        if (x > i) {
          const int a = v[i], b = v[x];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            v[i] = b;
            v[x] = a;
          }
        }
      }
      __syncwarp();
    }
  }
}

// Bitonic sort of 64 ints held two per lane (element lane in a, lane + 32
// in b), by shuffles: no shared memory and no barriers.
__device__ __forceinline__ void warp_sort64(int& a, int& b, int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 32) {  // partners in the same lane (only for k = 64: ascending)
        const int lo = min(a, b), hi = max(a, b);
        a = lo;
        b = hi;
      } else {
        const int oa = __shfl_xor_sync(0xFFFFFFFFu, a, j);
        const int ob = __shfl_xor_sync(0xFFFFFFFFu, b, j);
        const bool lower = (lane & j) == 0;
        const bool upa = (lane & k) == 0, upb = ((lane + 32) & k) == 0;
        a = (lower == upa) ? min(a, oa) : max(a, oa);
        b = (lower == upb) ? min(b, ob) : max(b, ob);
      }
    }
  }
}

// Sorts cand[0..128); when every real entry sits in cand[0..64) (the rest
// being the 0x7FFFFFFF filler), in registers.
__device__ __forceinline__ void warp_sort_cand(int* cand, int used, int lane) {
  if (used <= 64) {
    int a = cand[lane], b = cand[lane + 32];
    __syncwarp();
    warp_sort64(a, b, lane);
    cand[lane] = a;
    cand[lane + 32] = b;
    __syncwarp();
  } else {
    warp_sort128(cand, lane);
  }
}

// Query-side plan of item (h, loc), one warp: every (group, attended block,
// tile) candidate as (tile << 8 | mask bits), sorted, equal tiles merged.
__device__ void plan_q_item(const Problem& p, const Geom& g, int h, int loc,
                            int* cand, int* merged, int lane) {
  const ItemMeta m = item_meta(g, p.H, h * g.per_bh + loc);
  TileList& L = static_cast<TileList*>(p.qplan)[(size_t)h * g.per_bh + loc];
  if (m.global) {
    const int bits = expand_groups(m.gvalid, 3);
    const int j0 = m.chunk * g.chunk, j1 = min(g.nt, j0 + g.chunk);
    for (int x = lane; x < j1 - j0; x += 32) {
      L.tile[x] = (int16_t)(j0 + x);
      L.mask[x] = (uint8_t)bits;
    }
    if (lane == 0) L.n = j1 - j0;
    return;
  }
  const int S = 5 + p.r, T = g.bs == 128 ? 2 : 1;
  bool bad = false;
  for (int idx = lane; idx < 128; idx += 32) {
    int v = 0x7FFFFFFF;
    const int gr = idx / (S * T), s = (idx / T) % S, tt = idx % T;
    if (gr < 4 && (m.gvalid >> gr) & 1) {
      const int i = block_of(g, m.t[gr >> 1] * kTile + 32 * (gr & 1));
      int j;
      if (s < 5) {
        const int base[5] = {0, i - 1, i, i + 1, g.nb - 1};
        j = base[s];
      } else {
        j = p.rand_idx[((size_t)h * g.nb + i) * p.r + (s - 5)];
        if (j != -1 && (j < 0 || j >= g.nb)) bad = true;
        if (j < 0 || j >= g.nb) j = -1;
      }
      if (j >= 0) {
        int tile, halves;
        if (g.bs == 32) {
          tile = j >> 1;
          halves = 1 << (j & 1);
        } else if (g.bs == 64) {
          tile = j;
          halves = 3;
        } else {
          tile = 2 * j + tt;
          halves = 3;
        }
        v = (tile << 8) | (halves << (2 * gr));
      }
    }
    cand[idx] = v;
  }
  if (bad) set_status(p.status, BB_ERR_BAD_TABLE);
  __syncwarp();
  warp_sort_cand(cand, 4 * S * T, lane);
  // Merge equal tiles into the sorted list (mt, mm) in shared memory.
  int* mt = merged;
  int* mm = merged + kMaxT;
  int base_pos = 0;
  for (int r = 0; r < 4; ++r) {
    const int e = lane + 32 * r;
    const int v = cand[e];
    const bool head = v != 0x7FFFFFFF && (e == 0 || (cand[e - 1] >> 8) != (v >> 8));
    int bits = 0;
    if (head) {
      for (int x = e; x < 128 && (cand[x] >> 8) == (v >> 8) && cand[x] != 0x7FFFFFFF; ++x)
        bits |= cand[x] & 0xFF;
    }
    const unsigned hb = __ballot_sync(0xFFFFFFFFu, head);
    if (head) {
      const int pos = base_pos + __popc(hb & ((1u << lane) - 1));
      if (pos < kMaxT) {
        mt[pos] = v >> 8;
        mm[pos] = bits;
      }
    }
    base_pos += __popc(hb);
  }
  const int n = min(base_pos, kMaxT);
  __syncwarp();
  // Visiting order: tiles both 64-row halves of the item attend first, then
  // tiles of the upper half (groups 0, 1) and of the lower half (groups 2,
  // 3) alternately, so the half with nothing to do on a tile starts on the
  // next one (its own) while the other works; results do not depend on the
  // order.  Each class keeps ascending tile order.
  int cls[2], rk[2];
  unsigned cnt_b = 0, cnt_u = 0, cnt_l = 0;
  for (int r = 0; r < 2; ++r) {
    const int e = lane + 32 * r;
    int c = -1;
    if (e < n) {
      const bool up = (mm[e] & 0x0F) != 0, lo = (mm[e] & 0xF0) != 0;
      c = (up && lo) ? 0 : up ? 1 : 2;
    }
    const unsigned bb = __ballot_sync(0xFFFFFFFFu, c == 0);
    const unsigned bu = __ballot_sync(0xFFFFFFFFu, c == 1);
    const unsigned bl = __ballot_sync(0xFFFFFFFFu, c == 2);
    const unsigned below = (1u << lane) - 1;
    cls[r] = c;
    rk[r] = c == 0 ? cnt_b + __popc(bb & below)
          : c == 1 ? cnt_u + __popc(bu & below)
                   : cnt_l + __popc(bl & below);
    cnt_b += __popc(bb);
    cnt_u += __popc(bu);
    cnt_l += __popc(bl);
  }
  const int nbo = (int)cnt_b, nu = (int)cnt_u, nl = (int)cnt_l;
  const int np = min(nu, nl);  // alternating pairs
  for (int r = 0; r < 2; ++r) {
    const int e = lane + 32 * r;
    if (e >= n) continue;
    int pos;
    if (cls[r] == 0) {
      pos = rk[r];
    } else if (cls[r] == 1) {
      pos = rk[r] < np ? nbo + 2 * rk[r] : nbo + 2 * np + (rk[r] - np);
    } else {
      pos = rk[r] < np ? nbo + 2 * rk[r] + 1 : nbo + 2 * np + (nu - np) + (rk[r] - np);
    }
    L.tile[pos] = (int16_t)mt[e];
    L.mask[pos] = (uint8_t)mm[e];
  }
  if (lane == 0) L.n = n;
}

// Key-side walk of item (h, loc), one warp: the attending query tiles of
// its key rows, ascending.  Each item owns a fixed region of the head's walk
// area, so no allocator is needed: a middle window's walk has at most T x
// (the CSR list lengths of its key blocks) entries (T = 2 query tiles per
// query block at block size 128, else 1), so its region starts at T times
// the CSR offset of its first key block; global chunks (g.chunk query tiles
// each) follow T x (all CSR entries).
// offs / list: the head's CSR (global memory, or shared memory when
// stage is null: the lists are then read in place).
__device__ void plan_k_item(const Problem& p, const Geom& g, int h, int loc,
                            const int* offs, const int* list, int* stage, int* cand,
                            int lane) {
  const int item = h * g.per_bh + loc;
  KeyWalk w;
  w.init_head(g, p.H, offs, list, item);
  uint32_t* walk = p.kplan + (size_t)h * p.kcap;
  int* kofs = p.kof + 2 * (size_t)item;
  const int T = g.bs == 128 ? 2 : 1;
  int base, cap;
  if (w.global) {
    base = T * offs[g.nb] + (w.gi * g.nchunks + w.chunk) * g.chunk;
    cap = g.chunk;
  } else {
    const int row0 = w.t[0] * kTile;  // window rows [row0, row0 + 128)
    const int jf = block_of(g, row0);
    const int jl = min(g.nb - 1, block_of(g, min(row0 + 127, g.nb * g.bs - 1)));
    base = T * offs[jf];
    cap = T * (offs[jl + 1] - offs[jf]);
  }
  if (base < 0 || base + cap > p.kcap) {  // cannot happen within the bound
    if (lane == 0) {
      set_status(p.status, BB_ERR_BAD_TABLE);
      kofs[0] = 0;
      kofs[1] = 0;
    }
    return;
  }
  int total = 0;
  for (int x = 0; x < w.nl; ++x) total += w.ln[x];
  if (!w.global && total * T <= 128) {
    // Warp-parallel: every (list entry, tile of its query block) as
    // (tile << 8 | group-half bits), sorted, equal tiles merged.
    int cum[5];
    cum[0] = 0;
    for (int x = 0; x < 4; ++x) cum[x + 1] = cum[x] + (x < w.nl ? w.ln[x] * T : 0);
    for (int e = lane; e < 128; e += 32) {
      int v = 0x7FFFFFFF;
      if (e < cum[w.nl]) {
        int x = 0;
        while (e >= cum[x + 1]) ++x;
        const int k = e - cum[x];
        const int i = w.lp[x][k / T];  // attending query block
        int tile, halves;
        if (g.bs == 32) {
          tile = i >> 1;
          halves = 1 << (i & 1);
        } else if (g.bs == 64) {
          tile = i;
          halves = 3;
        } else {
          tile = 2 * i + (k % T);
          halves = 3;
        }
        v = (tile << 8) | expand_groups(w.lg[x], halves);
      }
      cand[e] = v;
    }
    __syncwarp();
    warp_sort_cand(cand, cum[w.nl], lane);
    int pos0 = 0;
    for (int r = 0; r < 4; ++r) {
      const int e = lane + 32 * r;
      const int v = cand[e];
      const bool head = v != 0x7FFFFFFF && (e == 0 || (cand[e - 1] >> 8) != (v >> 8));
      int bits = 0;
      if (head)
        for (int x = e; x < 128 && cand[x] != 0x7FFFFFFF && (cand[x] >> 8) == (v >> 8); ++x)
          bits |= cand[x] & 0xFF;
      const unsigned hb = __ballot_sync(0xFFFFFFFFu, head);
      if (head) {
        const int pos = pos0 + __popc(hb & ((1u << lane) - 1));
        if (pos < cap) walk[base + pos] = kentry(v >> 8, bits);
      }
      pos0 += __popc(hb);
    }
    if (lane == 0) {
      kofs[0] = base;
      kofs[1] = min(pos0, cap);
    }
    return;
  }
  // Otherwise one lane merges the lists (staged in shared memory when they
  // fit).
  if (stage && !w.global && total <= kStageCap) {
    int off = 0;
    for (int x = 0; x < w.nl; ++x) {
      for (int e = lane; e < w.ln[x]; e += 32) stage[off + e] = w.lp[x][e];
      w.lp[x] = stage + off;
      off += w.ln[x];
    }
  }
  __syncwarp();
  if (lane == 0) {
    int n = 0, tile, mask;
    while (n < cap && w.next(tile, mask)) walk[base + n++] = kentry(tile, mask);
    kofs[0] = base;
    kofs[1] = n;
  }
}

// One word of the masked-tile bitmap (see Problem::tdead): warp w
// of batch b writes word w (w = 0: the flag word, from the first 32 keys;
// w >= 1: tiles 32 (w - 1) .. 32 (w - 1) + 31, lane i testing the 64 keys of
// one tile).
__device__ void dead_tile_word(const Problem& p, int nt, int b, int w, int lane) {
  const uint8_t* km = p.key_mask + (size_t)b * p.L;
  bool bit;
  if (w == 0) {
    bit = km[lane] != 0;  // keys 0..31 lie in block 0 for every block size
  } else {
    const int j = 32 * (w - 1) + lane;
    bit = false;
    if (j < nt) {
      const uint4* m4 = reinterpret_cast<const uint4*>(km + (size_t)j * kTile);
      uint32_t any = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 x = __ldg(m4 + c);
        any |= x.x | x.y | x.z | x.w;
      }
      bit = any == 0;
    }
  }
  const uint32_t word = __ballot_sync(0xffffffffu, bit);
  if (lane == 0) p.tdead[(size_t)b * p.tdead_words + w] = w == 0 ? (word != 0 ? 1u : 0u) : word;
}

// Plans, one warp per item: query-side lists (do_q) and key-side walks
// (do_k, after the CSR exists); with do_dead, then one warp per word of the
// masked-tile bitmap.
__global__ void __launch_bounds__(32 * kPlanWarps) plan_kernel(Problem p, int do_q,
                                                               int do_k, int do_dead) {
  __shared__ int cand[kPlanWarps][128];
  __shared__ int stage[kPlanWarps][kStageCap];
  const Geom g = make_geom(p);    // query side
  const Geom kg = make_kgeom(p);  // key side
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The work counters of the tensor-core launches that follow.
  if (blockIdx.x == 0 && threadIdx.x < 4) p.sched[threadIdx.x] = 0;
  const int id = blockIdx.x * kPlanWarps + warp;
  const int nq = do_q ? p.H * g.per_bh : 0;
  const int nk = do_k ? p.H * kg.per_bh : 0;
  if (do_dead && id >= nq + nk) {
    const int x = id - nq - nk;
    if (x < p.B * p.tdead_words) dead_tile_word(p, g.nt, x / p.tdead_words, x % p.tdead_words, lane);
    return;
  }
  if (id < nq) {
    plan_q_item(p, g, id / g.per_bh, id % g.per_bh, cand[warp], stage[warp], lane);
  } else if (id - nq < nk) {
    const int k = id - nq;
    const int h = k / kg.per_bh;
    plan_k_item(p, kg, h, k % kg.per_bh, p.csr_offs + (size_t)h * (kg.nb + 1),
                p.csr_list + (size_t)h * p.csr_cap, stage[warp], cand[warp], lane);
  }
}

// Transposed adjacency of head h built in shared memory by the whole CTA
// (the same construction as csr_build_kernel): offs[nb + 1], then the lists.
// Returns the lists' base; sm holds 2 nb + blockDim.x + (nb + 1) + csr_cap
// ints.
__device__ int* build_head_csr(const Problem& p, int h, int* sm, int*& offs) {
  const int nb = p.nb, r = p.r, tid = threadIdx.x, nth = blockDim.x;
  int* cnt = sm;
  int* cur = cnt + nb;
  int* tsum = cur + nb;
  offs = tsum + nth;
  int* list = offs + nb + 1;
  const int32_t* table = p.rand_idx + (size_t)h * nb * r;
  for (int j = tid; j < nb; j += nth) {
    int c;
    if (j == 0 || j == nb - 1) {
      c = nb;
    } else {
      c = 2;  // global query rows 0 and nb-1
      for (int i = j - 1; i <= j + 1; ++i) c += (i >= 1 && i <= nb - 2);
    }
    cnt[j] = c;
  }
  __syncthreads();
  for (int x = tid; x < nb * r; x += nth) {
    const int i = x / r, a = x % r;
    if (i == 0 || i == nb - 1) continue;
    const int j = random_target(table + (size_t)i * r, a, i, nb, p.status);
    if (j >= 0) atomicAdd(&cnt[j], 1);
  }
  __syncthreads();
  const int chunk = (nb + nth - 1) / nth;
  const int c0 = tid * chunk, c1 = min(nb, c0 + chunk);
  int local = 0;
  for (int j = c0; j < c1; ++j) local += cnt[j];
  tsum[tid] = local;
  __syncthreads();
  for (int step = 1; step < nth; step <<= 1) {
    int add = tid >= step ? tsum[tid - step] : 0;
    __syncthreads();
    tsum[tid] += add;
    __syncthreads();
  }
  int run = tsum[tid] - local;
  for (int j = c0; j < c1; ++j) {
    cur[j] = run;
    offs[j] = run;
    run += cnt[j];
  }
  if (tid == nth - 1) offs[nb] = tsum[nth - 1];
  __syncthreads();
  for (int x = tid; x < 2 * nb; x += nth) {
    const int j = x < nb ? 0 : nb - 1;
    const int i = x % nb;
    if (x >= nb && nb == 1) continue;
    list[cur[j] + i] = i;
  }
  for (int j = tid; j < nb; j += nth) {
    if (j == 0 || j == nb - 1) continue;
    int pos = atomicAdd(&cur[j], 2 + (j - 1 >= 1) + 1 + (j + 1 <= nb - 2));
    list[pos++] = 0;
    list[pos++] = nb - 1;
    for (int i = j - 1; i <= j + 1; ++i)
      if (i >= 1 && i <= nb - 2) list[pos++] = i;
  }
  for (int x = tid; x < nb * r; x += nth) {
    const int i = x / r, a = x % r;
    if (i == 0 || i == nb - 1) continue;
    const int j = random_target(table + (size_t)i * r, a, i, nb, p.status);
    if (j >= 0) list[atomicAdd(&cur[j], 1)] = i;
  }
  __syncthreads();
  for (int j = tid; j < nb; j += nth) {
    if (j == 0 || j == nb - 1) continue;
    int* L = list + offs[j];
    const int n = offs[j + 1] - offs[j];
    for (int a = 1; a < n; ++a) {
      int x = L[a], c = a - 1;
      while (c >= 0 && L[c] > x) {
        L[c + 1] = L[c];
        --c;
      }
      L[c + 1] = x;
    }
  }
  __syncthreads();
  return list;
}

constexpr int kFusedWarps = 8;

// Backward plans in one launch: the first qctas CTAs plan query-side items
// (one warp each); the next dctas CTAs write the masked-tile bitmap (one
// warp per word); the others each build one head's transposed adjacency in
// shared memory and plan a slice of that head's key-side items from it
// (kslices CTAs per head, so no CTA waits for another).
__global__ void __launch_bounds__(32 * kFusedWarps) plan_bwd_kernel(Problem p, int qctas,
                                                                    int dctas, int kslices) {
  extern __shared__ int csr_sm[];
  __shared__ int cand[kFusedWarps][128];
  __shared__ int merged[kFusedWarps][128];
  const Geom g = make_geom(p);    // query side
  const Geom kg = make_kgeom(p);  // key side
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0 && threadIdx.x < 4) p.sched[threadIdx.x] = 0;
  if ((int)blockIdx.x < qctas) {
    const int id = blockIdx.x * kFusedWarps + warp;
    if (id < p.H * g.per_bh)
      plan_q_item(p, g, id / g.per_bh, id % g.per_bh, cand[warp], merged[warp], lane);
    return;
  }
  if ((int)blockIdx.x < qctas + dctas) {
    const int x = ((int)blockIdx.x - qctas) * kFusedWarps + warp;
    if (x < p.B * p.tdead_words)
      dead_tile_word(p, g.nt, x / p.tdead_words, x % p.tdead_words, lane);
    return;
  }
  const int kb = blockIdx.x - qctas - dctas;
  const int h = kb / kslices, slice = kb % kslices;
  int* offs;
  const int* list = build_head_csr(p, h, csr_sm, offs);
  for (int loc = slice * kFusedWarps + warp; loc < kg.per_bh; loc += kslices * kFusedWarps)
    plan_k_item(p, kg, h, loc, offs, list, nullptr, cand[warp], lane);
}

size_t fused_plan_smem(const Problem& p) {
  return (size_t)(2 * p.nb + 32 * kFusedWarps + p.nb + 1 + pair_cap(p.nb, p.r)) * sizeof(int);
}

}  // namespace

bool tc_bwd_plan_fused(const Problem& p) { return fused_plan_smem(p) <= 160u * 1024u; }

cudaError_t launch_plan_bwd(const Problem& p, cudaStream_t s) {
  const Geom g = make_geom(p);
  const int nitems = p.H * g.per_bh;
  const int qctas = (nitems + kFusedWarps - 1) / kFusedWarps;
  // One key-side item per warp (each CTA rebuilds its head's small
  // adjacency, so more CTAs per head cost only parallel work).
  const int kslices = max(1, (make_kgeom(p).per_bh + kFusedWarps - 1) / kFusedWarps);
  // With a key mask, the masked-tile bitmap.
  const int dctas = (p.key_mask && p.tdead)
                        ? (p.B * p.tdead_words + kFusedWarps - 1) / kFusedWarps
                        : 0;
  const size_t smem = fused_plan_smem(p);
  cudaError_t e = cudaFuncSetAttribute(
      plan_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  plan_bwd_kernel<<<qctas + dctas + p.H * kslices, 32 * kFusedWarps, smem, s>>>(p, qctas, dctas,
                                                                                kslices);
  return cudaGetLastError();
}

cudaError_t launch_bwd_pre(const Problem& p, cudaStream_t s) {
  const size_t rows = (size_t)p.B * p.H * p.L;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (p.dtype == BB_F32)
    bwd_pre_kernel<float><<<grid, 256, 0, s>>>(p);
  else
    bwd_pre_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

size_t tc_items_per_bh(const Problem& p) { return make_geom(p).per_bh; }

size_t tc_key_items_per_bh(const Problem& p) { return make_kgeom(p).per_bh; }

size_t tc_qplan_bytes(const Problem& p) {
  return (size_t)p.H * tc_items_per_bh(p) * sizeof(TileList);
}

// Upper bound of key-side walk entries per head: every entry of a middle
// window stands for at least one attended (query block, key block) pair
// (two tiles per block at block size 128); global items visit all tiles.
int tc_kplan_cap(const Problem& p) {
  const Geom g = make_geom(p);
  return 2 * pair_cap(p.nb, p.r) + g.n_git * g.nt + 64;
}

int tc_tdead_words(const Problem& p) { return 1 + (make_geom(p).nt + 31) / 32; }

cudaError_t launch_plan(const Problem& p, bool key_side, cudaStream_t s) {
  const int items = p.H * (int)tc_items_per_bh(p);
  const int kitems = key_side ? p.H * (int)tc_key_items_per_bh(p) : 0;
  // With a key mask the plans also write the masked-tile bitmap.
  const int dead = (p.key_mask && p.tdead) ? 1 : 0;
  const int n = items + kitems + (dead ? p.B * p.tdead_words : 0);
  plan_kernel<<<(n + kPlanWarps - 1) / kPlanWarps, 32 * kPlanWarps, 0, s>>>(
      p, 1, key_side ? 1 : 0, dead);
  return cudaGetLastError();
}

cudaError_t launch_csr_build(const Problem& p, cudaStream_t s) {
  const size_t base = (size_t)(2 * p.nb + kCsrThreads) * sizeof(int);
  const size_t with_list = base + (size_t)p.csr_cap * sizeof(int);
  const int in_smem = with_list <= 200u * 1024u ? 1 : 0;
  const size_t smem = in_smem ? with_list : base;
  cudaError_t e = cudaFuncSetAttribute(
      csr_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  csr_build_kernel<<<p.H, kCsrThreads, smem, s>>>(p, in_smem);
  return cudaGetLastError();
}

}  // namespace bb
