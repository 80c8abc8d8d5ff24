// Tensor-core backward of the block-sparse attention (bf16 I/O, blocks of
// 32, 64 or 128 tokens, d 64) for sm_100a.  Probabilities are recomputed
// from the forward's lse (P = exp(S - lse)), so nothing of size pairs x bs^2
// is stored.  Items (see tc_common.cuh) are taken from a per-launch counter.
//
// tc_dq_kernel: query-side items (as in the forward).  Per key tile of the
//   item: S = Q K^T and dP = dO V^T into TMEM; one thread per row forms
//   dS = P (dP - D) (D = <dO, O> of the row, computed at the start of the
//   item and also written to the workspace with -lse*log2(e) for the next
//   kernel) into dS columns of its own, so the next tile's S and dP are
//   computed as soon as this tile's have been read; dQ += dS K accumulates
//   in TMEM across the item.  Global rows write fp32 partials per chunk.
// tc_dkdv_kernel: key-side items take 128 key rows (a middle window of two
//   key tiles) and walk the planned query tiles that attend them (from the
//   transposed adjacency), each with a group/half mask; the global key
//   blocks, attended by every query block, are split into chunks of query
//   tiles.  Per query tile: S^T = K_pair Q^T and dP^T = V_pair dO^T (issued
//   by a warp of their own into double-buffered TMEM, so a tile's scores
//   are computed while the softmax works on the one before); P^T and dS^T
//   (bf16) into TMEM buffers of their own, formed by eight softmax warps,
//   two per TMEM lane quarter on the two 32-column halves of the tile;
//   dV += P^T dO and dK += dS^T Q (issued by the MMA warp) accumulate in
//   TMEM.  One CTA per SM holds all 512 TMEM columns.  From kSplitMinL
//   the global key blocks run in a launch of their own with a bf16 low part
//   of P^T and dS^T.  The loader hands each visited query tile's walk entry
//   to the other warps through shared memory with the tile's stage, so it
//   can leave tiles out per (b, h): with the query-side mask, query tiles
//   whose tokens are all padding (P = 0).  Each key row is owned by exactly
//   one item (or one chunk partial), so there are no atomics on data.
// bwd_finish_kernel: sums the chunk partials of the global query rows (dQ)
//   and of the global key blocks (dK, dV) in a fixed order.
#include "dropout.cuh"
#include "tc_common.cuh"

namespace bb {
namespace {

using namespace sm100;

// 1-CTA-per-SM kernels: warp 0 loads, warp 1 issues the gradient MMAs,
// warp 2 issues S / dP (S^T / dP^T), warps 3-10 run the softmax, two per
// SM sub-partition on the two column halves of each tile.  A tcgen05.mma
// costs its issuing thread ~50 cycles, so the score MMAs get a thread of
// their own and follow the loads as soon as data and TMEM buffer are ready.
constexpr int kThreads1 = 352;
// Per-tile information the loader passes to the score-MMA warp through the
// stage barriers (written before the stage's expect_tx arrive).
constexpr int kTinfo = 16;          // ring entries (> stages in flight)
constexpr uint8_t kTinfoEnd = 0x80; // no more tiles
// dQ kernel: two CTAs per SM, 192 threads (TMA warp, MMA warp, four
// softmax warps), 256 TMEM columns each, three K / V stages.
constexpr int kThreads2 = 192;
constexpr uint32_t kTmemCols = 256;
constexpr int kKvStages = 3;
constexpr uint32_t kQStageBytes = 2 * kTileBytes + 1024;  // dK/dV: Q, dO, NL, D

struct BwdArgs {
  PairArgs qa;       // query side (dq): problem, geometry, items
  // Key side (dkdv): its geometry (the query side's items, with its own
  // chunking of the global key blocks) and the items this launch takes:
  // per (b, h) the locs [kloc0, kloc0 + knloc).
  Geom kgeo;
  int kitems, kloc0, knloc;
  int* kctr;  // this launch's work counter
  float* D;          // [B*H*L]
  float* NL;         // [B*H*L]: -lse * log2(e)
  float* dqpart;     // [B*H][n_git][nchunks][128][64]
  float* kvpart;     // [B*H][n_git][nchunks][128][128] (dK | dV)
};

__device__ __forceinline__ void ld_bf16x8_as_f(const __nv_bfloat16* p,
                                               float (&f)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(ws[e] << 16);
    f[2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
  }
}

// One 64-element gradient row (fp32 bit patterns, columns 0-31 in lo and
// 32-63 in hi) times mul, stored as bf16 (rounded to nearest even) or, when
// the call asked for fp32 gradients, as fp32.
__device__ __forceinline__ void store_grad_row(const Problem& p, void* base, size_t row,
                                               const uint32_t (&lo)[32],
                                               const uint32_t (&hi)[32], float mul) {
  if (p.grad_f32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(base) + row * kHeadDim);
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      const uint32_t* src = v < 8 ? lo + 4 * v : hi + 4 * (v - 8);
      dst[v] = make_float4(__uint_as_float(src[0]) * mul, __uint_as_float(src[1]) * mul,
                           __uint_as_float(src[2]) * mul, __uint_as_float(src[3]) * mul);
    }
    return;
  }
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + row * kHeadDim);
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const uint32_t* src = v < 4 ? lo + 8 * v : hi + 8 * (v - 4);
    uint4 w;
    w.x = pack_bf16(__uint_as_float(src[0]) * mul, __uint_as_float(src[1]) * mul);
    w.y = pack_bf16(__uint_as_float(src[2]) * mul, __uint_as_float(src[3]) * mul);
    w.z = pack_bf16(__uint_as_float(src[4]) * mul, __uint_as_float(src[5]) * mul);
    w.w = pack_bf16(__uint_as_float(src[6]) * mul, __uint_as_float(src[7]) * mul);
    dst[v] = w;
  }
}

// Half a gradient row: 32 fp32 bit patterns (columns col0 .. col0 + 31)
// times mul, stored as bf16 (rounded to nearest even) or fp32 as the call
// asked.
__device__ __forceinline__ void store_grad_half(const Problem& p, void* base, size_t row,
                                                int col0, const uint32_t (&v)[32],
                                                float mul) {
  if (p.grad_f32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(base) + row * kHeadDim + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(__uint_as_float(v[4 * i]) * mul, __uint_as_float(v[4 * i + 1]) * mul,
                           __uint_as_float(v[4 * i + 2]) * mul,
                           __uint_as_float(v[4 * i + 3]) * mul);
    return;
  }
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + row * kHeadDim + col0);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t* x = v + 8 * i;
    dst[i] = make_uint4(pack_bf16(__uint_as_float(x[0]) * mul, __uint_as_float(x[1]) * mul),
                        pack_bf16(__uint_as_float(x[2]) * mul, __uint_as_float(x[3]) * mul),
                        pack_bf16(__uint_as_float(x[4]) * mul, __uint_as_float(x[5]) * mul),
                        pack_bf16(__uint_as_float(x[6]) * mul, __uint_as_float(x[7]) * mul));
  }
}

// 32 fp32 values (bit patterns) to consecutive floats of a partial row.
__device__ __forceinline__ void store_part32(float* dst, const uint32_t (&v)[32]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    d4[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                        __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
}

// ======================= dQ =======================

// P = 2^(S c + NL) of 32 key columns (col0: 0 or 32 within the tile) of
// one row, in place over S; masked keys are offset by mvl.
__device__ __forceinline__ void dq_p_half(uint32_t (&s)[32], uint64_t kb, int col0, float c,
                                          float nl2, float mvl) {
  if (((kb >> col0) & 0xFFFFFFFFull) == 0xFFFFFFFFull) {
    // No masked key in these columns: paired (f32x2) arithmetic.
    const float2 c2 = make_float2(c, c), nl22 = make_float2(nl2, nl2);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float2 a =
          fma2(make_float2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2, nl22);
      s[e] = __float_as_uint(ex2(a.x));
      s[e + 1] = __float_as_uint(ex2(a.y));
    }
    return;
  }
  // Some keys masked: their offset added, paired (each element rounded as
  // in the form fmaf(s, c, nl2 + offset)).
  const float2 c2 = make_float2(c, c);
  const float nlm = nl2 + mvl;
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float2 b2 = make_float2(((kb >> (col0 + e)) & 1ull) ? nl2 : nlm,
                                  ((kb >> (col0 + e + 1)) & 1ull) ? nl2 : nlm);
    const float2 a =
        fma2(make_float2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2, b2);
    s[e] = __float_as_uint(ex2(a.x));
    s[e + 1] = __float_as_uint(ex2(a.y));
  }
}

// dS = P (dP - D) of 32 key columns of one row, as 16 bf16 pairs.
__device__ __forceinline__ void dq_ds_half(const uint32_t (&pv)[32], const uint32_t (&dp)[32],
                                           float Dr, uint32_t* out) {
  const float2 D2 = make_float2(Dr, Dr);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float2 d = mul2(make_float2(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1])),
                          sub2(make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])), D2));
    out[e >> 1] = pack_bf16(d.x, d.y);
  }
}

// Dropout form of dq_ds_half: dS = P (m dP - D), m = 1 / keep probability
// where kept (bit e of keep), 0 where dropped.
__device__ __forceinline__ void dq_ds_half_drop(const uint32_t (&pv)[32],
                                                const uint32_t (&dp)[32], float Dr, float sc,
                                                uint32_t keep, uint32_t* out) {
  const float2 nD2 = make_float2(-Dr, -Dr);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    // Paired (f32x2): m dP - D, then times P, each element rounded once.
    const float2 m = make_float2(keep_factor(keep, e, sc), keep_factor(keep, e + 1, sc));
    const float2 t =
        fma2(m, make_float2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])), nD2);
    const float2 d = mul2(make_float2(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1])), t);
    out[e >> 1] = pack_bf16(d.x, d.y);
  }
}

struct DqBars {
  // list_full: the slot's tile list landed (the producer's bulk copy);
  // list_ready: the list, compacted, and the item are published.
  uint64_t list_full[2], list_ready[2], list_empty[2];
  uint64_t q_full, q_empty;
  uint64_t kv_full[kKvStages], kv_empty[kKvStages];
  uint64_t s_full, s_free, dp_free, p_full, dq_done, dq_full, dq_empty;
};

// kMask: a key mask is given (else every key is attended).
// kWhole: global rows run whole (every item's rows are final here).
template <bool kDrop, bool kMask, bool kWhole>
__global__ void __launch_bounds__(kThreads2, 2)
    tc_dq_kernel(const __grid_constant__ BwdArgs ba,
                 const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmG) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ DqBars bars;
  __shared__ TileList lists[2];  // bulk-copy destinations (16-byte aligned)
  __shared__ int4 item_sh[2];    // (b, h, loc, 1) of the slot's item; w = 0: no more items
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const PairArgs& a = ba.qa;
  const Problem& p = a.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* Qs = base;                          // [128][64] Q pair
  uint8_t* Gs = base + 2 * kTileBytes;         // [128][64] dO pair
  uint8_t* KVs = base + 4 * kTileBytes;        // [stage][K, V]

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.list_full[s], 1);
      mbar_init(&bars.list_ready[s], 1);
      mbar_init(&bars.list_empty[s], 5);
    }
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(&bars.kv_full[s], 1);
      mbar_init(&bars.kv_empty[s], 1);
    }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.s_free, 4);
    mbar_init(&bars.dp_free, 4);
    mbar_init(&bars.p_full, 4);
    mbar_init(&bars.dq_done, 1);
    mbar_init(&bars.dq_full, 1);
    mbar_init(&bars.dq_empty, 4);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmG);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // dQ | S | dP | dS (bf16 pairs): dS has its own columns, so S and dP of
  // the next tile can be computed while this tile's dS is still formed.
  const uint32_t tDQ = tmem, tS = tmem + 64, tDP = tmem + 128, tDS = tmem + 192;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t g = 0;
      int q_issued = 0;
      uint32_t q_par = 0;
      for (int k = 0;; ++k) {
        const int slot = k & 1;
        if (!mbar_wait(&bars.list_empty[slot], ((k >> 1) & 1) ^ 1, &abort_flag,
                       p.status))
          break;
        // Planned key-tile list: one bulk copy into the slot.
        // Items are taken from the launch's counter (longest first); the
        // slot's (b, h, loc) is published by the list_ready arrive.
        int ib, ih, iloc;
        if (!next_work(a.geo, p.B, p.H, 0, a.geo.per_bh, p.sched, ib, ih, iloc)) {
          item_sh[slot] = make_int4(0, 0, 0, 0);
          mbar_arrive_release(&bars.list_ready[slot]);
          break;
        }
        item_sh[slot] = make_int4(ib, ih, iloc, 1);
        const ItemMeta m = item_meta_at(a.geo, ib, ih, p.H, iloc);
        const TileList& L = lists[slot];
        mbar_expect_tx(&bars.list_full[slot], sizeof(TileList));
        bulk_load(&lists[slot],
                  static_cast<const TileList*>(p.qplan) + (size_t)m.h * a.geo.per_bh + m.loc,
                  sizeof(TileList), &bars.list_full[slot]);
        if (!mbar_wait(&bars.list_full[slot], (k >> 1) & 1, &abort_flag, p.status)) break;
        if (p.key_mask && p.tdead) {
          const uint32_t* dw = p.tdead + (size_t)m.b * p.tdead_words;
          auto dead = [&](int j) { return (__ldg(dw + 1 + (j >> 5)) >> (j & 31)) & 1u; };
          TileList& Lw = lists[slot];
          if (p.mask_q && dead(m.t[0]) && (m.t[1] < 0 || dead(m.t[1]))) {
            // Every row is a padding token (query-side mask): P is 0 on
            // them, so their dq is 0 and no key tile is needed.
            Lw.n = 0;
          } else if (__ldg(dw) & 1u) {
            // Drop key tiles whose 64 keys are all masked: exact when every
            // row has a valid attended key (the flag word), as in the
            // forward.
            int n2 = 0;
            for (int t = 0; t < Lw.n; ++t) {
              if (dead(Lw.tile[t])) continue;
              Lw.tile[n2] = Lw.tile[t];
              Lw.mask[n2] = Lw.mask[t];
              ++n2;
            }
            Lw.n = n2;
          }
          fence_proxy_async_smem();  // before the slot's next bulk copy
        }
        mbar_arrive_release(&bars.list_ready[slot]);
        if (!mbar_wait(&bars.q_empty, (k & 1) ^ 1, &abort_flag, p.status)) break;
        const int row0 = m.bh * p.L;
        const int nh = m.t[1] >= 0 ? 2 : 1;
        mbar_expect_tx(&bars.q_full, 2u * nh * kTileBytes);
        for (int hh = 0; hh < nh; ++hh) {
          const int y = row0 + m.t[hh] * kTile;
          tma_load_2d(Qs + hh * kTileBytes, &tmQ, &bars.q_full, 0, y);
          tma_load_2d(Gs + hh * kTileBytes, &tmG, &bars.q_full, 0, y);
        }
        q_issued = 1;
        q_par = k & 1;
        bool ok = true;
        for (int t = 0; t < L.n; ++t) {
          const int st = g % kKvStages;
          if (!mbar_wait(&bars.kv_empty[st], ((g / kKvStages) & 1) ^ 1,
                         &abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&bars.kv_full[st], 2 * kTileBytes);
          uint8_t* kv = KVs + st * 2 * kTileBytes;
          const int y = row0 + L.tile[t] * kTile;
          tma_load_2d(kv, &tmK, &bars.kv_full[st], 0, y);
          tma_load_2d(kv + kTileBytes, &tmV, &bars.kv_full[st], 0, y);
          ++g;
        }
        if (!ok) break;
      }
      if (abort_flag) {
        for (uint32_t s = 0; s < (uint32_t)kKvStages; ++s) {
          if (g < s + 1) continue;
          const uint32_t last = g - 1 - ((g - 1 - s) % kKvStages);
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&bars.kv_full[s], (last / kKvStages) & 1) &&
                 globaltimer() - t0 < 100000000ull) {
          }
        }
        if (q_issued) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&bars.q_full, q_par) &&
                 globaltimer() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    const uint32_t idS = idesc_bf16(128, 64, 0, 0);
    const uint32_t idDQ = idesc_bf16(128, 64, 0, 1);
    const uint32_t qaddr = smem_u32(Qs), gaddr = smem_u32(Gs);
    uint32_t g = 0, u = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k & 1;
      if (!mbar_wait(&bars.list_ready[slot], (k >> 1) & 1, &abort_flag, p.status))
        break;
      if (!item_sh[slot].w) break;
      const int n = lists[slot].n;
      if (!mbar_wait(&bars.q_full, k & 1, &abort_flag, p.status)) break;
      tc_fence_after();
      // dQ += dS K of item tile t (global tile uu, K/V stage st).
      auto issue_dq = [&](int t, uint32_t uu, int st) -> bool {
        if (!mbar_wait(&bars.p_full, uu & 1, &abort_flag, p.status) ||
            (t == 0 && !mbar_wait(&bars.dq_empty, (k & 1) ^ 1, &abort_flag, p.status)))
          return false;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kaddr = smem_u32(KVs + st * 2 * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tDQ, tDS + kk * 8, sdesc_sw128(kaddr + kk * 2048, 8192), idDQ,
                   (t > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars.dq_done);
          mma_commit(&bars.kv_empty[st]);
          if (t == n - 1) mma_commit(&bars.dq_full);
        }
        __syncwarp();
        return true;
      };
      for (int t = 0; t < n; ++t) {
        const uint32_t uu = u + t;
        const int st = (g + t) % kKvStages;
        // S and dP of this tile overwrite the previous tile's once the
        // softmax has read them (s_free, dp_free); dS has its own columns.
        if (!mbar_wait(&bars.kv_full[st], ((g + t) / kKvStages) & 1, &abort_flag,
                       p.status) ||
            (uu > 0 && !mbar_wait(&bars.s_free, (uu - 1) & 1, &abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kaddr = smem_u32(KVs + st * 2 * kTileBytes);
        const uint32_t vaddr = kaddr + kTileBytes;
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tS, sdesc_sw128(qaddr + kk * 32, 16),
                   sdesc_sw128(kaddr + kk * 32, 16), idS, kk > 0);
        }
        __syncwarp();
        if (uu > 0 && !mbar_wait(&bars.dp_free, (uu - 1) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tDP, sdesc_sw128(gaddr + kk * 32, 16),
                   sdesc_sw128(vaddr + kk * 32, 16), idS, kk > 0);
          mma_commit(&bars.s_full);
          if (t == n - 1) mma_commit(&bars.q_empty);  // Q, dO read only here
        }
        __syncwarp();
        // The previous tile's dQ goes to the tensor pipe after this tile's
        // S and dP, while the softmax works on the previous tile's dS.
        if (t > 0 && !issue_dq(t - 1, uu - 1, (g + t - 1) % kKvStages)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      if (n > 0) {
        if (!issue_dq(n - 1, u + n - 1, (g + n - 1) % kKvStages)) break;
      } else {
        if (!mbar_wait(&bars.dq_empty, (k & 1) ^ 1, &abort_flag, p.status)) break;
        if (lane == 0) {
          mma_commit(&bars.dq_full);
          mma_commit(&bars.q_empty);
        }
        __syncwarp();
      }
      g += n;
      u += n;
      if (lane == 0) mbar_arrive(&bars.list_empty[slot]);
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int half = row >> 6, r64 = row & 63;
    const int gshift = 2 * quarter;  // this warp's row group = its quarter
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float c = p.scale * kLog2e;
    const float mvl = p.mask_value * kLog2e;
    uint32_t u = 0;
    for (int k = 0;; ++k) {
      const int slot = k & 1;
      if (!mbar_wait(&bars.list_ready[slot], (k >> 1) & 1, &abort_flag, p.status))
        break;
      const int4 wi = item_sh[slot];
      if (!wi.w) break;
      const TileList& L = lists[slot];
      const ItemMeta im = item_meta_at(a.geo, wi.x, wi.y, p.H, wi.z);
      const int n = L.n;
      const bool rvalid = (im.gvalid >> quarter) & 1;
      const int tq = (rvalid ? im.t[half] : 0) * kTile + r64;  // query token
      const size_t grow = (size_t)im.bh * p.L + tq;
      float nl2 = 0.f, Dr = 0.f;
      if (rvalid) {
        nl2 = -p.lse[grow] * kLog2e;
        // Query-side mask: a padding token's P is 0 (NL = -inf), so its dS
        // is 0 here and in the dK/dV pass, which reads NL.
        if (p.mask_q && !p.key_mask[(size_t)im.b * p.L + tq]) nl2 = -INFINITY;
        const __nv_bfloat16* Or = static_cast<const __nv_bfloat16*>(p.o) + grow * kHeadDim;
        const __nv_bfloat16* Gr = static_cast<const __nv_bfloat16*>(p.dout) + grow * kHeadDim;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          float fo[8], fg[8];
          ld_bf16x8_as_f(Or + 8 * v, fo);
          ld_bf16x8_as_f(Gr + 8 * v, fg);
#pragma unroll
          for (int e = 0; e < 8; ++e) Dr = fmaf(fo[e], fg[e], Dr);
        }
        if (!im.global || im.chunk == 0) {
          ba.D[grow] = Dr;
          ba.NL[grow] = nl2;
        }
      }
      bool ok = true;
      // Stored dropout decisions: this row's table row, and the words of
      // each tile loaded one tile ahead.
      KeepRow kr;
      if (kDrop && p.keep_bits) kr = keep_row(p, im.h, tq);
      auto keep_words = [&](int tt) -> uint64_t {
        const int mm = (L.mask[tt] >> gshift) & 3;
        return mm ? keep_load64(p, im.bh, im.h, kr, tq, L.tile[tt], mm) : 0ull;
      };
      uint64_t dbn = (kDrop && p.keep_bits && n > 0) ? keep_words(0) : 0ull;
      for (int t = 0; t < n; ++t, ++u) {
        const int m2 = (L.mask[t] >> gshift) & 3;  // attended column halves
        const uint64_t dbs = dbn;
        if (kDrop && p.keep_bits && t + 1 < n) dbn = keep_words(t + 1);
        // Valid keys of the tile (loaded while the scores are computed).
        const uint64_t kb = (kMask && m2) ? key_bits(p, im.b, L.tile[t]) : ~0ull;
        if (!mbar_wait(&bars.s_full, u & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // S of the attended halves into registers: once every warp has it
        // (s_free) the MMA warp computes the next tile's S; P is formed in
        // place.  dP follows half by half; after the second half (dp_free)
        // the next tile's dP may be computed.
        uint32_t s0[32], s1[32], dp[32];
        if (m2 & 1) tmem_ld32(tS + lane_off, s0);
        if (m2 & 2) tmem_ld32(tS + 32 + lane_off, s1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_free);
        const uint64_t db = (kDrop && m2)
                                ? (p.keep_bits ? dbs : keep_row64(p, im.b, im.h, tq, L.tile[t]))
                                : 0ull;
        if (m2 & 1) dq_p_half(s0, kb, 0, c, nl2, mvl);
        if (m2 & 2) dq_p_half(s1, kb, 32, c, nl2, mvl);
        uint32_t dS[32];
        if (m2 & 1) {
          tmem_ld32(tDP + lane_off, dp);
          tmem_ld_wait();
          if (kDrop)
            dq_ds_half_drop(s0, dp, Dr, p.drop_scale, (uint32_t)db, dS);
          else
            dq_ds_half(s0, dp, Dr, dS);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) dS[e] = 0u;
        }
        if (m2 & 2) {
          tmem_ld32(tDP + 32 + lane_off, dp);
          tmem_ld_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.dp_free);
        if (m2 & 2) {
          if (kDrop)
            dq_ds_half_drop(s1, dp, Dr, p.drop_scale, (uint32_t)(db >> 32), dS + 16);
          else
            dq_ds_half(s1, dp, Dr, dS + 16);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) dS[16 + e] = 0u;
        }
        // The dS columns are free once the previous tile's dQ MMA completed.
        if (u > 0 && !mbar_wait(&bars.dq_done, (u - 1) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t d0[16], d1[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          d0[e] = dS[e];
          d1[e] = dS[16 + e];
        }
        tmem_st16(tDS + lane_off, d0);
        tmem_st16(tDS + 16 + lane_off, d1);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full);
      }
      if (!ok) break;
      if (!mbar_wait(&bars.dq_full, k & 1, &abort_flag, p.status)) break;
      tc_fence_after();
      uint32_t q0[32], q1[32];
      tmem_ld32(tDQ + lane_off, q0);
      tmem_ld32(tDQ + 32 + lane_off, q1);
      tmem_ld_wait();
      if (n == 0) {  // no tile accumulated: the rows' dq is 0
#pragma unroll
        for (int e = 0; e < 32; ++e) q0[e] = q1[e] = 0u;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.dq_empty);
      if (rvalid) {
        if (kWhole || !im.global) {  // final rows (no chunk partials)
          store_grad_row(p, p.dq, grow, q0, q1, p.scale);
        } else {
          float4* dst = reinterpret_cast<float4*>(
              ba.dqpart + ((((size_t)im.bh * a.geo.n_git + im.gi) * a.geo.nchunks + im.chunk) *
                               128 + row) * 64);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(q0[4 * v]), __uint_as_float(q0[4 * v + 1]),
                                 __uint_as_float(q0[4 * v + 2]), __uint_as_float(q0[4 * v + 3]));
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[8 + v] = make_float4(__uint_as_float(q1[4 * v]), __uint_as_float(q1[4 * v + 1]),
                                     __uint_as_float(q1[4 * v + 2]), __uint_as_float(q1[4 * v + 3]));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.list_empty[slot]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ======================= dK / dV =======================

// Entries [e0, e1) of this head's walk area that hold the item's query
// tiles.  Walks are planned per (head, item) - they do not depend on the
// batch index - so they are looked up by (h, loc), and the range is clamped
// to the area the plan allocated.
__device__ __forceinline__ void walk_range(const Problem& p, const Geom& g,
                                           const ItemMeta& it, int& e0, int& e1) {
  const size_t k = (size_t)it.h * g.per_bh + it.loc;
  e0 = max(0, min(p.kof[2 * k], p.kcap));
  e1 = max(e0, min(e0 + p.kof[2 * k + 1], p.kcap));
}

// The dK/dV kernel runs one CTA per SM with all 512 TMEM columns:
//   acc (dK 0-63, dV 64-127), S^T[2] (128-255), dP^T[2] (256-383),
//   P^T[2] (bf16 pairs, 384-447), dS^T[2] (bf16 pairs, 448-511).
// Query tile g uses buffers g & 1.  P^T and dS^T have columns of their own,
// so S^T / dP^T of tile g + 2 are computed as soon as the softmax has read
// tile g's (and while it still works on it); the dV / dK MMAs of tile g
// read P^T / dS^T, which the softmax of tile g + 2 overwrites only after
// those MMAs completed.  The launch of the global key blocks at long
// lengths (hi/lo split) keeps one S^T / dP^T buffer (128-191, 256-319) and
// puts the double-buffered low parts of P^T / dS^T in the other halves
// (192-255, 320-383): there S^T / dP^T of tile g + 1 are computed as soon
// as the softmax has read tile g's.
constexpr int kKvQStages = 8;  // query-tile stages (Q, dO, NL, D)
constexpr uint32_t kKvTmemCols = 512;
constexpr uint32_t kKvDK = 0, kKvDV = 64, kKvS = 128, kKvDP = 256, kKvP = 384, kKvDS = 448;
// hi/lo split launch: low parts of P^T / dS^T, buffer b at + 32 b
constexpr uint32_t kKvPL = kKvS + 64, kKvDSL = kKvDP + 64;

struct KvBars {
  // K / V pair of item k in slot k & 1: kp_full = landed (and kitem[] of the
  // slot published); kp_empty = its last S^T / dP^T MMAs completed and the
  // MMA warp and the eight softmax warps have read kitem[].
  uint64_t kp_full[2], kp_empty[2];
  uint64_t qt_full[kKvQStages], qt_empty[kKvQStages];
  // per tile buffer b: S^T / dP^T computed; read by the softmax; P^T / dS^T
  // written; the dV / dK MMAs that read them completed
  uint64_t s_full[2], s_free[2], p_full[2], g_done[2];
  uint64_t acc_full, acc_empty;
};

// kSplit: bf16 hi/lo split of the global key blocks' P^T and dS^T, where
// their gradients can grow large enough for bf16 products to cost accuracy:
// lengths >= 16K (they sum over every query row), and calls with a key mask
// (masked keys can concentrate many rows' probability on them).  A
// template flag keeps the low parts out of the other calls' register
// budget.
// kDrop: seeded attention dropout (P^T kept times 1 / keep probability for
// dV; dS^T = P^T (m dP^T - D)).
// kWhole: the global key blocks run whole (every item's rows are final here).
template <bool kSplit, bool kDrop, bool kWhole>
__global__ void __launch_bounds__(kThreads1, 1)
    tc_dkdv_kernel(const __grid_constant__ BwdArgs ba,
                   const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmG) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ KvBars bars;
  __shared__ int4 kitem[2];  // (b, h, loc, 1) of the item in pair slot s; w = 0: no more items
  // Item in pair slot s visits at least one query tile (published with it).
  __shared__ int kwalk[2];
  // flat tile g at g % kTinfo: pair slot | kp_full parity << 1 | last tile
  // of its item << 2, or kTinfoEnd; its walk entry (query tile | group
  // mask << 16) and the entry of the item's next visited tile.  Written by
  // the loader before the tile's qt_full arrive.
  __shared__ uint8_t tinfo[kTinfo];
  __shared__ uint32_t went[kTinfo], wnext[kTinfo];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const Problem& p = ba.qa.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  // [2 slots][K pair (2 tiles) | V pair (2 tiles)], then the query stages
  // [Q | dO | NL[64] | D[64]].
  uint8_t* KV = base;
  uint8_t* QT = base + 2 * 4 * kTileBytes;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.kp_full[s], 1);
      mbar_init(&bars.kp_empty[s], 10);  // last S^T commit + MMA warp + 8 softmax warps
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.s_free[s], 8);
      mbar_init(&bars.p_full[s], 8);
      mbar_init(&bars.g_done[s], 1);
    }
    for (int s = 0; s < kKvQStages; ++s) {
      mbar_init(&bars.qt_full[s], 1);
      mbar_init(&bars.qt_empty[s], 1);
    }
    mbar_init(&bars.acc_full, 1);
    mbar_init(&bars.acc_empty, 8);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kKvTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmG);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ---------------- loads (one thread) ----------------
    if (lane == 0) {
      uint32_t gq = 0;  // query stages loaded (flat tiles)
      int kp_issued[2] = {0, 0};
      uint32_t kp_par[2] = {0, 0};
      bool ok = true;
      for (int k = 0;; ++k) {
        const int ps = k & 1;
        // Pair slot ps held item k - 2: released once its last S^T / dP^T
        // completed and every role has read kitem[].
        if (!mbar_wait(&bars.kp_empty[ps], ((k >> 1) & 1) ^ 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        // Items are taken from the launch's counter (middle windows first);
        // the slot's (b, h, loc) is published by the kp_full arrive.
        int ib, ih, iloc;
        if (!next_work(ba.kgeo, p.B, p.H, ba.kloc0, ba.knloc, ba.kctr, ib, ih, iloc)) {
          kitem[ps] = make_int4(0, 0, 0, 0);
          mbar_arrive_release(&bars.kp_full[ps]);
          break;
        }
        kitem[ps] = make_int4(ib, ih, iloc, 1);
        const ItemMeta it = item_meta_at(ba.kgeo, ib, ih, p.H, iloc);
        const uint32_t* walk = p.kplan + (size_t)it.h * p.kcap;
        int e0, e1;
        walk_range(p, ba.kgeo, it, e0, e1);
        const bool tdead = p.key_mask && p.tdead;
        const uint32_t* dw = tdead ? p.tdead + (size_t)it.b * p.tdead_words : nullptr;
        auto dead = [&](int j) { return (__ldg(dw + 1 + (j >> 5)) >> (j & 31)) & 1u; };
        // Key rows whose keys are all masked get probability 0 from every
        // row when every row has a valid attended key (the flag word): their
        // dK and dV are 0, so the item visits no query tile.
        if (tdead && (__ldg(dw) & 1u) && dead(it.t[0]) && (it.t[1] < 0 || dead(it.t[1])))
          e1 = e0;
        // With the query-side mask, padding rows pass no gradient (P = 0):
        // query tiles whose tokens are all padding are left out of the walk.
        const bool qskip = tdead && p.mask_q;
        int e = e0;  // next walk entry to read
        auto next_live = [&](uint32_t& ent) -> bool {
          for (; e < e1; ++e) {
            ent = __ldg(walk + e);
            if (!qskip || !dead((int)(ent & 0xFFFFu))) {
              ++e;
              return true;
            }
          }
          return false;
        };
        uint32_t ent = 0u;
        bool have = next_live(ent);
        kwalk[ps] = have ? 1 : 0;
        const int row0 = it.bh * p.L;
        const int nh = it.t[1] >= 0 ? 2 : 1;
        uint8_t* kv = KV + ps * 4 * kTileBytes;
        mbar_expect_tx(&bars.kp_full[ps], 2u * nh * kTileBytes);
        for (int hh = 0; hh < nh; ++hh) {
          const int y = row0 + it.t[hh] * kTile;
          tma_load_2d(kv + hh * kTileBytes, &tmK, &bars.kp_full[ps], 0, y);
          tma_load_2d(kv + (2 + hh) * kTileBytes, &tmV, &bars.kp_full[ps], 0, y);
        }
        kp_issued[ps] = 1;
        kp_par[ps] = (k >> 1) & 1;
        if (!have) mma_commit(&bars.kp_empty[ps]);  // no MMA reads this pair
        while (have) {
          const int i = (int)(ent & 0xFFFFu);  // query tile
          // The next visited entry (read while the stage is awaited): this
          // tile is the item's last when there is none.
          uint32_t nent = 0u;
          const bool nhave = next_live(nent);
          const uint32_t g = gq;
          const uint32_t st = g % kKvQStages;
          if (!mbar_wait(&bars.qt_empty[st], ((g / kKvQStages) & 1) ^ 1, &abort_flag,
                         p.status)) {
            ok = false;
            break;
          }
          tinfo[g % kTinfo] = (uint8_t)(ps | (((k >> 1) & 1) << 1) | (nhave ? 0 : 4));
          went[g % kTinfo] = ent;
          wnext[g % kTinfo] = nent;
          uint8_t* q = QT + st * kQStageBytes;
          mbar_expect_tx(&bars.qt_full[st], 2 * kTileBytes + 512);
          const int y = row0 + i * kTile;
          tma_load_2d(q, &tmQ, &bars.qt_full[st], 0, y);
          tma_load_2d(q + kTileBytes, &tmG, &bars.qt_full[st], 0, y);
          bulk_load(q + 2 * kTileBytes, ba.NL + y, 256, &bars.qt_full[st]);
          bulk_load(q + 2 * kTileBytes + 256, ba.D + y, 256, &bars.qt_full[st]);
          ++gq;
          ent = nent;
          have = nhave;
        }
        if (!ok) break;
      }
      // No more tiles: tell the score-MMA warp through the next stage.
      if (ok) {
        const uint32_t st = gq % kKvQStages;
        if (mbar_wait(&bars.qt_empty[st], ((gq / kKvQStages) & 1) ^ 1, &abort_flag, p.status)) {
          tinfo[gq % kTinfo] = kTinfoEnd;
          mbar_arrive_release(&bars.qt_full[st]);
        }
      }
      if (abort_flag) {
        for (uint32_t s = 0; s < (uint32_t)kKvQStages; ++s)
          if (gq >= s + 1) {
            const uint32_t last = gq - 1 - ((gq - 1 - s) % kKvQStages);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&bars.qt_full[s], (last / kKvQStages) & 1) &&
                   globaltimer() - t0 < 100000000ull) {
            }
          }
        for (int s = 0; s < 2; ++s)
          if (kp_issued[s]) {
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&bars.kp_full[s], kp_par[s]) &&
                   globaltimer() - t0 < 100000000ull) {
            }
          }
      }
    }
  } else if (warp == 2) {
    // -------- S^T = K Q^T, dP^T = V dO^T (one thread) --------
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 64, 0, 0);
      for (uint32_t g = 0;; ++g) {
        const int b = g & 1;
        const uint32_t st = g % kKvQStages;
        if (!mbar_wait(&bars.qt_full[st], (g / kKvQStages) & 1, &abort_flag, p.status)) break;
        const int ti = tinfo[g % kTinfo];
        if (ti & kTinfoEnd) break;
        const int ps = ti & 1;
        // S^T / dP^T buffer: g & 1, or the one buffer of the split launch
        // (then used by every tile).
        const int sb = kSplit ? 0 : b;
        const uint32_t spar = kSplit ? (g & 1) : ((g >> 1) & 1);
        if (!mbar_wait(&bars.kp_full[ps], (ti >> 1) & 1, &abort_flag, p.status) ||
            !mbar_wait(&bars.s_free[sb], spar ^ 1, &abort_flag, p.status))
          break;
        tc_fence_after();
        const uint32_t kaddr = smem_u32(KV + ps * 4 * kTileBytes);
        const uint32_t vaddr = kaddr + 2 * kTileBytes;
        const uint32_t qaddr = smem_u32(QT + st * kQStageBytes);
        const uint32_t gaddr = qaddr + kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + kKvS + sb * 64, sdesc_sw128(kaddr + kk * 32, 16),
                 sdesc_sw128(qaddr + kk * 32, 16), idS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + kKvDP + sb * 64, sdesc_sw128(vaddr + kk * 32, 16),
                 sdesc_sw128(gaddr + kk * 32, 16), idS, kk > 0);
        mma_commit(&bars.s_full[sb]);
        if (ti & 4) mma_commit(&bars.kp_empty[ps]);  // the pair's last reader
      }
    }
  } else if (warp == 1) {
    // ---------- dV += P^T dO, dK += dS^T Q (one thread) ----------
    const uint32_t idAcc = idesc_bf16(128, 64, 0, 1);
    uint32_t u = 0, ai = 0;  // flat tile counter, items with tiles
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int ps = k & 1;
      if (!mbar_wait(&bars.kp_full[ps], (k >> 1) & 1, &abort_flag, p.status)) break;
      const int4 wi = kitem[ps];
      if (!wi.w) break;
      const ItemMeta it = item_meta_at(ba.kgeo, wi.x, wi.y, p.H, wi.z);
      const bool has = kwalk[ps] != 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.kp_empty[ps]);  // kitem, kwalk read
      // The item's tiles, up to the one marked last (its P^T / dS^T arrive
      // after the softmax observed the loader's tile information).
      for (int t = 0; has; ++t) {
        const uint32_t g = u;
        const int b = g & 1;
        const uint32_t st = g % kKvQStages;
        if (!mbar_wait(&bars.p_full[b], (g >> 1) & 1, &abort_flag, p.status) ||
            (t == 0 && !mbar_wait(&bars.acc_empty, (ai & 1) ^ 1, &abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool last = (tinfo[g % kTinfo] & 4) != 0;
        if (lane == 0) {
          const uint32_t qaddr = smem_u32(QT + st * kQStageBytes);
          const uint32_t gaddr = qaddr + kTileBytes;
          // A operands: 16 query rows per K step = 8 TMEM columns of bf16
          // pairs (high and low parts alike).
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + kKvDV, tmem + kKvP + b * 32 + kk * 8,
                   sdesc_sw128(gaddr + kk * 2048, 8192), idAcc, (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + kKvDK, tmem + kKvDS + b * 32 + kk * 8,
                   sdesc_sw128(qaddr + kk * 2048, 8192), idAcc, (t > 0 || kk > 0) ? 1u : 0u);
          if (kSplit && it.global) {
            // Global key blocks sum over every query row: at long lengths
            // their P^T and dS^T also carry a bf16 low part, so the products
            // keep ~16 bits instead of 8.
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tmem + kKvDV, tmem + kKvPL + b * 32 + kk * 8,
                     sdesc_sw128(gaddr + kk * 2048, 8192), idAcc, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tmem + kKvDK, tmem + kKvDSL + b * 32 + kk * 8,
                     sdesc_sw128(qaddr + kk * 2048, 8192), idAcc, 1u);
          }
          mma_commit(&bars.g_done[b]);
          mma_commit(&bars.qt_empty[st]);
          if (last) mma_commit(&bars.acc_full);
        }
        __syncwarp();
        ++u;
        if (last) break;
      }
      if (has) ++ai;
    }
  } else {
    // Softmax warps 3-10: two per TMEM lane quarter (one per SM sub-
    // partition), each owning one 32-column half (query columns) of the
    // tile: P^T comes from the stored lse, so no reduction between them.
    const int quarter = warp & 3;
    const int hc = (warp - 3) >> 2;  // query-column half
    const int row = quarter * 32 + lane;
    const int half = row >> 6, r64 = row & 63;
    const int gshift = 2 * quarter;  // this warp's key-row group = its quarter
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float c = p.scale * kLog2e;
    const float mvl = p.mask_value * kLog2e;
    uint32_t u = 0, ai = 0;
    for (int k = 0;; ++k) {
      const int ps = k & 1;
      // This iteration's item: published with its K / V pair (kp_full).
      if (!mbar_wait(&bars.kp_full[ps], (k >> 1) & 1, &abort_flag, p.status)) break;
      const int4 wi = kitem[ps];
      if (!wi.w) break;
      const ItemMeta it = item_meta_at(ba.kgeo, wi.x, wi.y, p.H, wi.z);
      const bool has = kwalk[ps] != 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.kp_empty[ps]);  // kitem, kwalk read
      const bool rvalid = (it.gvalid >> quarter) & 1;
      const size_t ktok = (size_t)(rvalid ? it.t[half] : 0) * kTile + r64;
      const size_t krow = (size_t)it.bh * p.L + ktok;
      float off = 0.f;
      if (rvalid && p.key_mask)
        off = p.key_mask[(size_t)it.b * p.L + ktok] ? 0.f : mvl;
      const bool split = kSplit && it.global;  // bf16 low parts too
      bool ok = true;
      // With stored dropout decisions, lane l loads the word of query token
      // t0 + l against the warp's 32 keys (transposed below).
      auto keep_word = [&](uint32_t ent) -> uint32_t {
        if (!(((int)(ent >> 16) >> (gshift + hc)) & 1)) return 0u;
        return __ldg(keep_ptr(p, it.bh, it.h, (int)(ent & 0xFFFFu) * kTile + hc * 32 + lane,
                              (int)(ktok & ~(size_t)31)));
      };
      // The item's tiles as the loader published them, up to the one
      // marked last.  With stored dropout decisions, each tile's keep word
      // is loaded one tile ahead (from the next entry published with the
      // tile).
      const bool keep_ahead = kDrop && p.keep_bits;
      uint32_t kwn = 0u;
      if (keep_ahead && has) {
        if (!mbar_wait(&bars.qt_full[u % kKvQStages], (u / kKvQStages) & 1, &abort_flag,
                       p.status))
          break;
        kwn = keep_word(went[u % kTinfo]);
      }
      for (bool more = has; more;) {
        const uint32_t g = u;
        const int b = g & 1;
        const int sb = kSplit ? 0 : b;  // S^T / dP^T buffer (as the score warp)
        const uint32_t st = g % kKvQStages;
        // The tile's walk entry and last mark were written before its
        // stage's qt_full arrive (its NL / D arrive by bulk copy there too).
        if (!mbar_wait(&bars.qt_full[st], (g / kKvQStages) & 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        const uint32_t ent = went[g % kTinfo];
        more = (tinfo[g % kTinfo] & 4) == 0;
        const int mask = (int)(ent >> 16);
        const int qtile = (int)(ent & 0xFFFFu);
        const uint32_t kw = kwn;
        if (keep_ahead && more) kwn = keep_word(wnext[g % kTinfo]);
        // Do query rows of this warp's column half attend this key group?
        const bool att = (mask >> (gshift + hc)) & 1;
        if (!mbar_wait(&bars.s_full[sb], kSplit ? (g & 1) : ((g >> 1) & 1), &abort_flag,
                       p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* NLs =
            reinterpret_cast<const float*>(QT + st * kQStageBytes + 2 * kTileBytes);
        const float* Ds = NLs + 64;
        uint32_t sv[32], dp[32];
        if (att) {
          tmem_ld32(tmem + kKvS + sb * 64 + hc * 32 + lane_off, sv);
          tmem_ld32(tmem + kKvDP + sb * 64 + hc * 32 + lane_off, dp);
          tmem_ld_wait();
        }
        // S^T / dP^T of this buffer are in registers: the score MMAs may
        // refill it.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_free[sb]);
        // Dropout keep bits of this lane's key against the half's 32 query
        // tokens (att is uniform over the warp, as the shuffles need).
        const uint32_t keep =
            (kDrop && att)
                ? (p.keep_bits ? transpose32(kw, lane)
                               : keep_cols32(p, it.b, it.h, (int)(ktok & ~(size_t)31),
                                             qtile * kTile + hc * 32, lane))
                : 0u;
        // P^T and dS^T of the half (bf16 pairs, 16 columns each): high parts
        // to the P^T / dS^T buffers, low parts (split tiles) to theirs.
        uint32_t ph[16], dh[16], pl[16], dl[16];
        if (att) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const int col = hc * 32 + e;
            const float4 nl = *reinterpret_cast<const float4*>(NLs + col);
            const float4 dd = *reinterpret_cast<const float4*>(Ds + col);
            const float nls[4] = {nl.x, nl.y, nl.z, nl.w};
            const float dds[4] = {dd.x, dd.y, dd.z, dd.w};
            float pv[4], dv[4];
            const float2 c2 = make_float2(c, c), off2 = make_float2(off, off);
#pragma unroll
            for (int x = 0; x < 4; x += 2) {
              // Paired (f32x2) arithmetic, each element rounded as before.
              const float2 a = fma2(
                  make_float2(__uint_as_float(sv[e + x]), __uint_as_float(sv[e + x + 1])), c2,
                  add2(make_float2(nls[x], nls[x + 1]), off2));
              pv[x] = ex2(a.x);
              pv[x + 1] = ex2(a.y);
              if (kDrop) {
                // m = 1 / keep probability where kept, 0 where dropped:
                // dS = P (m dP - D), and m P enters dV (paired, each element
                // rounded once).
                const float2 m = make_float2(keep_factor(keep, e + x, p.drop_scale),
                                             keep_factor(keep, e + x + 1, p.drop_scale));
                const float2 pp = make_float2(pv[x], pv[x + 1]);
                const float2 t = fma2(
                    m, make_float2(__uint_as_float(dp[e + x]), __uint_as_float(dp[e + x + 1])),
                    make_float2(-dds[x], -dds[x + 1]));
                const float2 d = mul2(pp, t);
                const float2 pk = mul2(pp, m);
                dv[x] = d.x;
                dv[x + 1] = d.y;
                pv[x] = pk.x;
                pv[x + 1] = pk.y;
              } else {
                const float2 d = mul2(
                    make_float2(pv[x], pv[x + 1]),
                    sub2(make_float2(__uint_as_float(dp[e + x]), __uint_as_float(dp[e + x + 1])),
                         make_float2(dds[x], dds[x + 1])));
                dv[x] = d.x;
                dv[x + 1] = d.y;
              }
            }
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const int o = (e >> 1) + x;
              ph[o] = pack_bf16(pv[2 * x], pv[2 * x + 1]);
              dh[o] = pack_bf16(dv[2 * x], dv[2 * x + 1]);
              if (split) {
                pl[o] = pack_bf16(pv[2 * x] - __uint_as_float(ph[o] << 16),
                                  pv[2 * x + 1] - __uint_as_float(ph[o] & 0xFFFF0000u));
                dl[o] = pack_bf16(dv[2 * x] - __uint_as_float(dh[o] << 16),
                                  dv[2 * x + 1] - __uint_as_float(dh[o] & 0xFFFF0000u));
              }
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) ph[e] = dh[e] = pl[e] = dl[e] = 0u;
        }
        // P^T / dS^T buffer b is free once the dV / dK MMAs of tile g - 2
        // completed.
        if (!mbar_wait(&bars.g_done[b], ((g >> 1) & 1) ^ 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st16(tmem + kKvP + b * 32 + hc * 16 + lane_off, ph);
        tmem_st16(tmem + kKvDS + b * 32 + hc * 16 + lane_off, dh);
        if (split) {
          tmem_st16(tmem + kKvPL + b * 32 + hc * 16 + lane_off, pl);
          tmem_st16(tmem + kKvDSL + b * 32 + hc * 16 + lane_off, dl);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[b]);
        ++u;
      }
      if (!ok) break;
      uint32_t kx[32], vx[32];
      if (!has) {
        // No query tile visits these keys (none attends them, or all their
        // keys are masked): their dK and dV are 0.
#pragma unroll
        for (int e = 0; e < 32; ++e) kx[e] = vx[e] = 0u;
      } else {
        if (!mbar_wait(&bars.acc_full, ai & 1, &abort_flag, p.status)) break;
        ++ai;
        tc_fence_after();
        tmem_ld32(tmem + kKvDK + hc * 32 + lane_off, kx);
        tmem_ld32(tmem + kKvDV + hc * 32 + lane_off, vx);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.acc_empty);
      }
      if (rvalid) {
        if (kWhole || !it.global) {  // final rows (no chunk partials)
          store_grad_half(p, p.dk, krow, hc * 32, kx, p.scale);
          store_grad_half(p, p.dv, krow, hc * 32, vx, 1.0f);
        } else {
          float* dst = ba.kvpart + ((((size_t)it.bh * ba.kgeo.n_git + it.gi) *
                                     ba.kgeo.nchunks + it.chunk) * 128 + row) * 128;
          store_part32(dst + hc * 32, kx);
          store_part32(dst + 64 + hc * 32, vx);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kKvTmemCols);
  }
}

// Element pair 2 lane, 2 lane + 1 of gradient row `grow` (fp32 or the I/O
// type, rounded once).
__device__ __forceinline__ void store_grad_pair(const Problem& p, void* base, size_t grow,
                                                int lane, float x, float y) {
  if (p.grad_f32)
    reinterpret_cast<float2*>(static_cast<float*>(base) + grow * kHeadDim)[lane] =
        make_float2(x, y);
  else
    reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(base) + grow * kHeadDim)[lane] =
        pack_bf16(x, y);
}

// One warp per row of a global item (query rows for dQ, key rows for
// dK / dV: both sides use the same tiles); lanes over d.  Chunks are summed
// in a fixed order; rows outside the global blocks are skipped.  Each side
// is merged only when its global rows were split into chunks.
__global__ void __launch_bounds__(256) bwd_finish_kernel(const BwdArgs ba) {
  const Problem& p = ba.qa.p;
  const Geom& g = ba.qa.geo;  // query side
  const Geom& kg = ba.kgeo;   // key side (same rows, its own chunks)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t id = (size_t)blockIdx.x * 8 + warp;  // over bh x gi x 128
  const size_t total = (size_t)p.B * p.H * g.n_git * 128;
  if (id >= total) return;
  const int row = id % 128;
  const int gi = (id / 128) % g.n_git;
  const size_t bh = id / (128 * g.n_git);
  int t[2], gvalid;
  item_rows(g, true, gi, t, gvalid);
  if (!((gvalid >> (row >> 5)) & 1)) return;
  const size_t grow = bh * p.L + (size_t)t[row >> 6] * kTile + (row & 63);
  // Unrolled so that several chunks' loads are in flight at once (the sums
  // keep the chunk order).
  if (g.nchunks > 1) {
    const size_t ib = (bh * g.n_git + gi) * g.nchunks;
    float q0 = 0.f, q1 = 0.f;
#pragma unroll 8
    for (int c = 0; c < g.nchunks; ++c) {
      const float2 x = reinterpret_cast<const float2*>(
          ba.dqpart + ((ib + c) * 128 + row) * 64)[lane];
      q0 += x.x;
      q1 += x.y;
    }
    store_grad_pair(p, p.dq, grow, lane, q0 * p.scale, q1 * p.scale);
  }
  if (kg.nchunks > 1) {
    const size_t ib = (bh * kg.n_git + gi) * kg.nchunks;
    float k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
#pragma unroll 8
    for (int c = 0; c < kg.nchunks; ++c) {
      const float* src = ba.kvpart + ((ib + c) * 128 + row) * 128;
      const float2 xk = reinterpret_cast<const float2*>(src)[lane];
      const float2 xv = reinterpret_cast<const float2*>(src + 64)[lane];
      k0 += xk.x;
      k1 += xk.y;
      v0 += xv.x;
      v1 += xv.y;
    }
    store_grad_pair(p, p.dk, grow, lane, k0 * p.scale, k1 * p.scale);
    store_grad_pair(p, p.dv, grow, lane, v0, v1);
  }
}

BwdArgs make_bwd_args(const Problem& p) {
  BwdArgs ba;
  ba.qa = make_pair_args(p);
  ba.kgeo = make_kgeom(p);
  ba.kitems = p.B * p.H * ba.kgeo.per_bh;
  ba.kloc0 = 0;
  ba.knloc = ba.kgeo.per_bh;
  ba.kctr = p.sched + 1;
  return ba;
}

}  // namespace

bool tc_bwd_supported(const Problem& p) { return tc_shape_ok(p); }

// D, NL: rows floats each; dq partials; dK/dV partials.
int tc_dkdv_launches(const Problem& p) {
  return (p.L >= kSplitMinL && make_geom(p).n_mid > 0) ? 2 : 1;
}

bool tc_global_rows_chunked(const Problem& p, int pass) {
  return make_geom(p).nchunks > 1 || (pass == 1 && make_kgeom(p).nchunks > 1);
}

size_t tc_bwd_extra_bytes(const Problem& p) {
  const size_t rows = (size_t)p.B * p.H * p.L;
  const Geom g = make_geom(p), kg = make_kgeom(p);
  const size_t uq = (size_t)p.B * p.H * g.n_git * g.nchunks * 128;
  const size_t uk = (size_t)p.B * p.H * kg.n_git * kg.nchunks * 128;
  return rows * 4 /* NL */ + uq * 64 * 4 + uk * 128 * 4 + 3 * 256;
}

cudaError_t launch_tc_bwd(const Problem& p, const TensorMaps& tm,
                          cudaStream_t s, EventMarks* marks) {
  BwdArgs ba = make_bwd_args(p);
  const size_t rows = (size_t)p.B * p.H * p.L;
  const size_t uq = (size_t)p.B * p.H * ba.qa.geo.n_git * ba.qa.geo.nchunks * 128;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* x = reinterpret_cast<uint8_t*>(p.part);
  ba.D = p.D;
  ba.NL = reinterpret_cast<float*>(x);
  x += al(rows * 4);
  ba.dqpart = reinterpret_cast<float*>(x);
  x += al(uq * 64 * 4);
  ba.kvpart = reinterpret_cast<float*>(x);

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

  const size_t smem_dq = 1024 + (4 + 2 * kKvStages) * kTileBytes;
  const bool drop = p.drop_thr != 0;
  const bool masked = p.key_mask != nullptr;
  using DqKernel = void (*)(const BwdArgs, const CUtensorMap, const CUtensorMap,
                            const CUtensorMap, const CUtensorMap);
  // [dropout][mask][whole]
  static const DqKernel dq_kernels[2][2][2] = {
      {{tc_dq_kernel<false, false, false>, tc_dq_kernel<false, false, true>},
       {tc_dq_kernel<false, true, false>, tc_dq_kernel<false, true, true>}},
      {{tc_dq_kernel<true, false, false>, tc_dq_kernel<true, false, true>},
       {tc_dq_kernel<true, true, false>, tc_dq_kernel<true, true, true>}}};
  const DqKernel dq_kernel =
      dq_kernels[drop ? 1 : 0][masked ? 1 : 0][ba.qa.geo.nchunks == 1 ? 1 : 0];
  cudaError_t e = cudaFuncSetAttribute(
      dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dq);
  if (e != cudaSuccess) return e;
  dq_kernel<<<min(ba.qa.items, 2 * sms), kThreads2, smem_dq, s>>>(
      ba, tm.q, tm.k, tm.v, tm.dout);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = marks->mark(s);
  if (e != cudaSuccess) return e;

  const size_t smem_kv = 1024 + 2 * 4 * kTileBytes + kKvQStages * kQStageBytes;
  // From kSplitMinL the global key blocks' items (the only ones with the
  // hi/lo split) run in a launch of their own, the middle windows without.
  const Geom& g = ba.kgeo;
  const int nglob = g.n_git * g.nchunks;
  struct Part {
    bool split;
    int per_bh, loc0;
  };
  Part parts[2];
  int nparts = 0;
  if (p.L >= kSplitMinL) {
    parts[nparts++] = {true, nglob, 0};
    if (g.n_mid > 0) parts[nparts++] = {false, g.n_mid, nglob};
  } else {
    // One launch.  Masked keys can concentrate the probability of many rows
    // on the global blocks and raise their gradients as a long sequence
    // does: the largest grows like sqrt(L) / block size (7.4 at L = 4096,
    // block 32, with three quarters of the keys masked), and bf16 products
    // cost ~1.7e-3 of it.  So with a key mask, from L = 2048 (block / 32)^2
    // on, the launch is the split variant (the global key blocks' P^T and
    // dS^T carry the bf16 low part).
    const bool masked_split =
        p.key_mask != nullptr && (long long)p.L * 1024 >= 2048LL * p.bs * p.bs;
    parts[nparts++] = {masked_split, g.per_bh, 0};
  }
  for (int i = 0; i < nparts; ++i) {
    BwdArgs bk = ba;
    bk.kloc0 = parts[i].loc0;
    bk.knloc = parts[i].per_bh;
    bk.kitems = p.B * p.H * parts[i].per_bh;
    bk.kctr = p.sched + 1 + i;  // sched[0]: dQ
    const bool kwhole = g.nchunks == 1;
    using KvKernel = void (*)(const BwdArgs, const CUtensorMap, const CUtensorMap,
                              const CUtensorMap, const CUtensorMap);
    // [split][dropout][whole]
    static const KvKernel kv_kernels[2][2][2] = {
        {{tc_dkdv_kernel<false, false, false>, tc_dkdv_kernel<false, false, true>},
         {tc_dkdv_kernel<false, true, false>, tc_dkdv_kernel<false, true, true>}},
        {{tc_dkdv_kernel<true, false, false>, tc_dkdv_kernel<true, false, true>},
         {tc_dkdv_kernel<true, true, false>, tc_dkdv_kernel<true, true, true>}}};
    const KvKernel kv_kernel =
        kv_kernels[parts[i].split ? 1 : 0][drop ? 1 : 0][kwhole ? 1 : 0];
    e = cudaFuncSetAttribute(kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_kv);
    if (e != cudaSuccess) return e;
    if (i > 0) {
      e = marks->mark(s);
      if (e != cudaSuccess) return e;
    }
    kv_kernel<<<min(bk.kitems, sms), kThreads1, smem_kv, s>>>(
        bk, tm.q, tm.k, tm.v, tm.dout);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

  // Global rows written whole on both sides: no chunk partials to merge.
  if (ba.qa.geo.nchunks == 1 && g.nchunks == 1) return cudaSuccess;
  e = marks->mark(s);
  if (e != cudaSuccess) return e;
  const size_t frows = (size_t)p.B * p.H * ba.qa.geo.n_git * 128;
  bwd_finish_kernel<<<(unsigned)((frows + 7) / 8), 256, 0, s>>>(ba);
  return cudaGetLastError();
}

}  // namespace bb
