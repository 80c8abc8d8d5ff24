// Tensor-core forward of the block-sparse attention (bf16 I/O, blocks of
// 32, 64 or 128 tokens, d 64) for sm_100a: TMA tile loads, tcgen05 MMAs with
// TMEM accumulators and an online softmax, in a persistent warp-specialised
// kernel.
//
// Work item = 128 query rows of one (b, h) in one 128-row MMA tile (see
// tc_common.cuh): a middle window streams the union of its row groups'
// attended key tiles, each with a mask of which 32-row group attends which
// 32 columns; a global item streams a chunk of all key tiles for the rows of
// blocks 0 and nb-1 and writes partial (O, m, l) that fwd_combine_kernel
// merges.  Blocks of 32, 64 and 128 tokens all map onto 64-token tiles.
// Items are taken from a per-launch counter (middle windows first).
//
// Roles (192 threads): warp 0 lane 0 takes the next item, bulk-copies its
// planned tile list and issues the TMA loads (Q pair once per item, K and V
// per key tile through a kNST-stage ring); warp 1 lane 0 issues the MMAs
// (S = Q K^T into one of two TMEM S buffers, O += P V with P read from one
// of two TMEM P buffers); warps 2-5 run the softmax, one thread per tile
// row: load S, fold scale, masks and the lazy running max, write P (bf16
// pairs) and rescale O in TMEM when the max moves; at the end of an item
// they normalise O and store it through shared memory with a TMA store.
#include "dropout.cuh"
#include "tc_common.cuh"

namespace bb {
namespace {

using namespace sm100;

constexpr int kNST = 4;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
// Rescale threshold of the lazy running max (log2 units): the max used for
// the exponent only moves when a row's true max exceeds it by more than
// this, so probabilities stay below 2^8 and O is rarely rescaled.
constexpr float kRescaleThreshold = 8.0f;

// TMEM columns: S[2] (fp32, 64 each), P[2] (bf16 pairs, 32 each), O (fp32).
// S, P and O are separate so the next S can be computed as soon as the
// softmax has read the current one, and P V accumulates straight into O.
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192;

struct Bars {
  // list_full: the tile list's bulk copy landed (producer only);
  // list_ready: the producer has dropped the item's fully masked key tiles
  // and publishes the list to the other roles.
  uint64_t list_full[2], list_ready[2], list_empty[2], q_full[2], q_empty[2];
  uint64_t kv_full[kNST], kv_empty[kNST];
  uint64_t s_full[2], s_empty[2], p_full[2];
  // One P V completion barrier per P buffer (it also frees the buffer):
  // P V(u) commits to pv_done[u & 1], so a wait for P V(u) by parity is
  // never confused with
  // P V(u - 1), which may still be in flight.
  uint64_t pv_done[2], o_empty;
};

// Maximum of 64 values with three-input max: 32 instructions, depth 4.
__device__ __forceinline__ float max64(const float* z) {
  float m[22];
#pragma unroll
  for (int i = 0; i < 21; ++i) m[i] = fmax3(z[3 * i], z[3 * i + 1], z[3 * i + 2]);
  m[21] = z[63];
  float n[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) n[i] = fmax3(m[3 * i], m[3 * i + 1], m[3 * i + 2]);
  n[7] = m[21];
  const float a = fmax3(n[0], n[1], n[2]), b = fmax3(n[3], n[4], n[5]);
  return fmax3(a, b, fmaxf(n[6], n[7]));
}

// Maximum of 32 values with three-input max: 16 instructions, depth 4.
__device__ __forceinline__ float max32(const float* z) {
  float m[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) m[i] = fmax3(z[3 * i], z[3 * i + 1], z[3 * i + 2]);
  m[10] = fmaxf(z[30], z[31]);
  const float a = fmax3(m[0], m[1], m[2]), b = fmax3(m[3], m[4], m[5]),
              d = fmax3(m[6], m[7], m[8]);
  return fmax3(fmax3(a, b, d), m[9], m[10]);
}

// kDrop: seeded attention dropout on the probabilities that enter P V (the
// row sums, hence the lse, stay those of the undropped softmax).
// kWhole: global items run whole (one chunk), so every row of every item is
// final in this kernel; else global items leave chunk partials.
// kMask: a key mask is given (else every key is attended).
// kHalf: block size 32, where a row group often attends only one 32-column
// half of a key tile: then only that half's scores are loaded and
// exponentiated (the other half's P is 0).
template <bool kDrop, bool kWhole, bool kMask, bool kHalf>
__global__ void __launch_bounds__(kThreads, 2)
    tc_fwd_kernel(const __grid_constant__ PairArgs a,
                  const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmO) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Bars bars;
  __shared__ TileList lists[2];  // bulk-copy destinations (16-byte aligned)
  __shared__ int4 item_sh[2];    // (b, h, loc, 1) of the slot's item; w = 0: no more items
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const Problem& p = a.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* Qs = base;                        // [2][128][64] bf16
  uint8_t* KVs = base + 2 * 2 * kTileBytes;  // [kNST][K, V][64][64] bf16

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.list_full[s], 1);
      mbar_init(&bars.list_ready[s], 1);
      mbar_init(&bars.list_empty[s], 5);
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.q_empty[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.s_empty[s], 4);
      mbar_init(&bars.p_full[s], 4);
      mbar_init(&bars.pv_done[s], 1);
    }
    mbar_init(&bars.o_empty, 4);
    for (int s = 0; s < kNST; ++s) {
      mbar_init(&bars.kv_full[s], 1);
      mbar_init(&bars.kv_empty[s], 1);
    }
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
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t g = 0;
      int qissued[2] = {0, 0};
      uint32_t qpar[2] = {0, 0};
      for (int k = 0;; ++k) {
        const int slot = k & 1;
        const uint32_t ph = (k >> 1) & 1;
        if (!mbar_wait(&bars.list_empty[slot], ph ^ 1, &abort_flag, p.status))
          break;
        // The item's key-tile list was planned before this kernel: one bulk
        // copy into the slot (the producer waits for it like the others).
        // Items are taken from the launch's counter (middle windows first);
        // the slot's (b, h, loc) is published by the list_ready arrive.
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
        if (!mbar_wait(&bars.list_full[slot], ph, &abort_flag, p.status)) break;
        if (p.key_mask && p.tdead) {
          // Drop key tiles whose 64 keys are all masked.  Exact when every
          // row has a valid attended key (the flag word: a valid key among
          // the first 32, which lie in block 0, attended by every row): a
          // masked key's probability is then exp(-10000 + ...) = 0.
          const uint32_t* dw = p.tdead + (size_t)m.b * p.tdead_words;
          if (__ldg(dw) & 1u) {
            TileList& Lw = lists[slot];
            int n2 = 0;
            for (int t = 0; t < Lw.n; ++t) {
              const int j = Lw.tile[t];
              if ((__ldg(dw + 1 + (j >> 5)) >> (j & 31)) & 1u) continue;
              Lw.tile[n2] = Lw.tile[t];
              Lw.mask[n2] = Lw.mask[t];
              ++n2;
            }
            Lw.n = n2;
            fence_proxy_async_smem();  // before the slot's next bulk copy
          }
        }
        mbar_arrive_release(&bars.list_ready[slot]);
        if (!mbar_wait(&bars.q_empty[slot], ph ^ 1, &abort_flag, p.status)) break;
        const int row0 = m.bh * p.L;
        const uint32_t qbytes = (m.t[1] >= 0 ? 2u : 1u) * kTileBytes;
        mbar_expect_tx(&bars.q_full[slot], qbytes);
        uint8_t* q = Qs + slot * 2 * kTileBytes;
        tma_load_2d(q, &tmQ, &bars.q_full[slot], 0, row0 + m.t[0] * kTile);
        if (m.t[1] >= 0)
          tma_load_2d(q + kTileBytes, &tmQ, &bars.q_full[slot], 0,
                      row0 + m.t[1] * kTile);
        qissued[slot] = 1;
        qpar[slot] = ph;
        bool ok = true;
        for (int t = 0; t < L.n; ++t) {
          const int st = g % kNST;
          const uint32_t kph = (g / kNST) & 1;
          if (!mbar_wait(&bars.kv_empty[st], kph ^ 1, &abort_flag, p.status)) {
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
        // Let issued copies land before the CTA's shared memory goes away:
        // wait (bounded) for the phase of the last load into each buffer.
        for (uint32_t s = 0; s < (uint32_t)kNST; ++s) {
          if (g < s + 1) continue;
          const uint32_t last = g - 1 - ((g - 1 - s) % kNST);
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&bars.kv_full[s], (last / kNST) & 1) &&
                 globaltimer() - t0 < 100000000ull) {
          }
        }
        for (int s = 0; s < 2; ++s) {
          if (!qissued[s]) continue;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&bars.q_full[s], qpar[s]) &&
                 globaltimer() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    const uint32_t idS = idesc_bf16(128, 64, 0, 0);   // Q (K-major) x K^T (K-major)
    const uint32_t idPV = idesc_bf16(128, 64, 0, 1);  // P (TMEM) x V (MN-major)
    uint32_t g = 0, u = 0;  // K/V stage counter, tile counter
    uint32_t oi = 0;        // items with at least one tile (O handed over)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k & 1;
      const uint32_t ph = (k >> 1) & 1;
      if (!mbar_wait(&bars.list_ready[slot], ph, &abort_flag, p.status)) break;
      if (!item_sh[slot].w) break;
      const int n = lists[slot].n;
      if (!mbar_wait(&bars.q_full[slot], ph, &abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t qaddr = smem_u32(Qs + slot * 2 * kTileBytes);
      // P V of tile t into O.
      auto issue_pv = [&](int t) -> bool {
        const uint32_t uu = u + t;
        const int b2 = uu & 1;
        const int st = (g + t) % kNST;
        if (!mbar_wait(&bars.p_full[b2], (uu >> 1) & 1, &abort_flag, p.status))
          return false;
        if (t == 0 && !mbar_wait(&bars.o_empty, (oi & 1) ^ 1, &abort_flag, p.status))
          return false;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t vaddr = smem_u32(KVs + st * 2 * kTileBytes + kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + kColO, tmem + kColP + b2 * 32 + kk * 8,
                   sdesc_sw128(vaddr + kk * 2048, 8192), idPV,
                   (t > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars.pv_done[b2]);
          mma_commit(&bars.kv_empty[st]);
        }
        __syncwarp();
        return true;
      };
      for (int t = 0; t < n; ++t) {
        const uint32_t uu = u + t;
        const int b2 = uu & 1;
        const int st = (g + t) % kNST;
        if (!mbar_wait(&bars.kv_full[st], ((g + t) / kNST) & 1, &abort_flag,
                       p.status) ||
            !mbar_wait(&bars.s_empty[b2], ((uu >> 1) & 1) ^ 1, &abort_flag,
                       p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kaddr = smem_u32(KVs + st * 2 * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + kColS + b2 * 64, sdesc_sw128(qaddr + kk * 32, 16),
                   sdesc_sw128(kaddr + kk * 32, 16), idS, kk > 0);
          mma_commit(&bars.s_full[b2]);
          if (t == n - 1) mma_commit(&bars.q_empty[slot]);
        }
        __syncwarp();
        if (t > 0 && !issue_pv(t - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && n > 0 && !issue_pv(n - 1)) ok = false;
      if (n == 0 && lane == 0) mma_commit(&bars.q_empty[slot]);  // nothing read Q
      __syncwarp();
      if (n > 0) ++oi;
      g += n;
      u += n;
      if (lane == 0) mbar_arrive(&bars.list_empty[slot]);
    }
  } else {
    // ---------------- softmax / epilogue (warps 2-5) ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // TMEM lane = tile row
    const int half = row >> 6;
    const int gshift = 2 * quarter;  // this warp's row group = its quarter
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tO = tmem + kColO + lane_off;
    const float c = p.scale * kLog2e;
    const float mvl = p.mask_value * kLog2e;
    uint32_t u = 0;  // tile counter (same sequence as the MMA warp)
    // Slot whose output store is in flight (lane 0): the slot is released
    // (list_empty) once the store has read the staged rows, which is
    // checked one tile into the next item instead of waiting right away.
    int pend = -1;
    auto release_pending = [&]() {
      if (lane == 0 && pend >= 0) {
        bulk_wait_read_all();
        mbar_arrive(&bars.list_empty[pend]);
      }
      pend = -1;
    };
    for (int k = 0;; ++k) {
      const int slot = k & 1;
      const uint32_t ph = (k >> 1) & 1;
      if (!mbar_wait(&bars.list_ready[slot], ph, &abort_flag, p.status)) break;
      const int4 wi = item_sh[slot];
      if (!wi.w) break;
      const TileList& L = lists[slot];
      const ItemMeta im = item_meta_at(a.geo, wi.x, wi.y, p.H, wi.z);
      const int n = L.n;
      if (n == 0) {
        // Every key tile of this chunk was masked (only global items can
        // lose all their tiles: middle items keep tile 0): an empty partial.
        if (im.global && ((im.gvalid >> quarter) & 1)) {
          float* part = p.part + ((((size_t)im.bh * a.geo.n_git + im.gi) * a.geo.nchunks +
                                   im.chunk) * 128 + row) * kPartStride;
#pragma unroll
          for (int e = 0; e < 16; ++e)
            reinterpret_cast<float4*>(part)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
          part[64] = -INFINITY;
          part[65] = 0.f;
        }
        __syncwarp();
        release_pending();
        if (lane == 0) mbar_arrive(&bars.list_empty[slot]);
        continue;
      }
      float m = -INFINITY, l = 0.f;
      // Query token of this row (dropout counters; any row when invalid).
      const int tq = (((im.gvalid >> quarter) & 1) ? im.t[half] : 0) * kTile + (row & 63);
      // Stored dropout decisions: this row's query block and its table row.
      const bool keep_out = kDrop && p.keep_bits && ((im.gvalid >> quarter) & 1);
      KeepRow kr;
      if (keep_out) kr = keep_row(p, im.h, tq);
      bool ok = true;
      for (int t = 0; t < n; ++t) {
        const uint32_t uu = u + t;
        const int b2 = uu & 1;
        const uint32_t par = (uu >> 1) & 1;
        const int m2 = (L.mask[t] >> gshift) & 3;  // attended column halves
        const bool att = m2 != 0;
        // Where this row's dropout decisions go when the caller keeps them
        // (worked out while the scores are still being computed).
        int ks0 = -1, ks1 = -1;
        if (keep_out && att) keep_slots64(p, im.h, kr, L.tile[t], m2, ks0, ks1);
        // Valid keys of the tile (loaded while the scores are computed).
        const uint64_t kb = (kMask && att) ? key_bits(p, im.b, L.tile[t]) : ~0ull;
        if (!mbar_wait(&bars.s_full[b2], par, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // One attended half (block 32): its scores in z[0, 32), written to
        // P half h0.
        const bool one = kHalf && m2 != 3;
        const int h0 = one ? (m2 >> 1) : 0;
        float z[64];
        if (att && one) {
          uint32_t s0[32];
          tmem_ld32(tmem + kColS + b2 * 64 + h0 * 32 + lane_off, s0);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) z[e] = __uint_as_float(s0[e]);
        } else if (att) {
          uint32_t s0[32], s1[32];
          tmem_ld32(tmem + kColS + b2 * 64 + lane_off, s0);
          tmem_ld32(tmem + kColS + b2 * 64 + 32 + lane_off, s1);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            z[e] = __uint_as_float(s0[e]);
            z[32 + e] = __uint_as_float(s1[e]);
          }
        }
        // S is in registers: its buffer may take the next tile's scores.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_empty[b2]);
        // P buffer b2 is free once the P V two tiles back has completed.
        if (!mbar_wait(&bars.pv_done[b2], par ^ 1, &abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tP = tmem + kColP + b2 * 32 + lane_off;
        if (att) {
          float mx;
          bool scaled;
          if (one) {
            // One attended half: its keys' offsets (if any masked), paired.
            const uint32_t kbh = (uint32_t)(kb >> (32 * h0));
            scaled = !(kbh == ~0u && c > 0.f);
            if (!scaled) {
              mx = max32(z) * c;
            } else {
              const float2 c2 = make_float2(c, c);
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float2 o = make_float2(((kbh >> e) & 1u) ? 0.f : mvl,
                                             ((kbh >> (e + 1)) & 1u) ? 0.f : mvl);
                const float2 r = fma2(make_float2(z[e], z[e + 1]), c2, o);
                z[e] = r.x;
                z[e + 1] = r.y;
              }
              mx = max32(z);
            }
          } else {
            const uint64_t hb = half_bits(m2);
            if (kb == ~0ull && hb == ~0ull && c > 0.f) {
              mx = max64(z) * c;
            } else if (kMask && hb == ~0ull) {
              // Every column attended, some keys masked (the finite offset):
              // paired, each element rounded once as below.
              const float2 c2 = make_float2(c, c);
#pragma unroll
              for (int e = 0; e < 64; e += 2) {
                const float2 o = make_float2(((kb >> e) & 1ull) ? 0.f : mvl,
                                             ((kb >> (e + 1)) & 1ull) ? 0.f : mvl);
                const float2 r = fma2(make_float2(z[e], z[e + 1]), c2, o);
                z[e] = r.x;
                z[e + 1] = r.y;
              }
              mx = max64(z);
            } else {
              // Columns outside the attended blocks are absent (-inf, p = 0);
              // masked keys inside them get the finite offset.
#pragma unroll
              for (int e = 0; e < 64; ++e)
                z[e] = ((hb >> e) & 1ull)
                           ? fmaf(z[e], c, ((kb >> e) & 1ull) ? 0.f : mvl)
                           : -INFINITY;
              mx = max64(z);
            }
            scaled = !(kb == ~0ull && hb == ~0ull && c > 0.f);
          }
          // Lazy running max: move it only when the row max exceeds it by
          // more than the threshold (or on the row's first attended tile).
          const bool first = (m == -INFINITY);
          const bool need = !first && mx > m + kRescaleThreshold;
          if (__any_sync(0xffffffffu, need)) {
            // O holds earlier tiles: wait for the last P V, then scale O by
            // 2^(m_old - m_new) on the rows that move.
            if (!mbar_wait(&bars.pv_done[(uu - 1) & 1], ((uu - 1) >> 1) & 1,
                           &abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float al = need ? ex2(m - mx) : 1.f;
#pragma unroll
            for (int q16 = 0; q16 < 4; ++q16) {
              uint32_t o[16];
              tmem_ld16(tO + q16 * 16, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 16; ++e)
                o[e] = __float_as_uint(__uint_as_float(o[e]) * al);
              tmem_st16(tO + q16 * 16, o);
            }
            tmem_st_wait();
            if (need) {
              l *= al;
              m = mx;
            }
          }
          if (first) m = mx;
          // Paired (f32x2) arithmetic: exponent arguments and row sums.
          float2 sum2[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) sum2[e] = make_float2(0.f, 0.f);
          const float cc = scaled ? 1.f : c;
          const float2 cc2 = make_float2(cc, cc), nm2 = make_float2(-m, -m);
          const uint64_t db = kDrop ? keep_row64(p, im.b, im.h, tq, L.tile[t]) : 0ull;
          // Hand the decisions to the backward when the caller keeps them.
          if (kDrop && p.keep_bits && (ks0 >= 0 || ks1 >= 0))
            keep_store64(p, im.bh, tq, L.tile[t], ks0, ks1, db);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            // z half hh goes to P half h0 + hh (one attended half: hh = 0
            // only).
            if (one && hh == 1) break;
            uint32_t Ph[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 a = fma2(make_float2(z[32 * hh + e], z[32 * hh + e + 1]), cc2, nm2);
              const float2 pp = make_float2(ex2(a.x), ex2(a.y));
              sum2[(e >> 1) & 3] = add2(sum2[(e >> 1) & 3], pp);
              if (kDrop) {
                // Kept probabilities times 1 / keep probability, dropped 0.
                const uint32_t dw = (uint32_t)(db >> (32 * (h0 + hh)));
                const float2 mk = make_float2(keep_factor(dw, e, p.drop_scale),
                                              keep_factor(dw, e + 1, p.drop_scale));
                const float2 pk = mul2(pp, mk);
                Ph[e >> 1] = pack_bf16(pk.x, pk.y);
              } else {
                Ph[e >> 1] = pack_bf16(pp.x, pp.y);
              }
            }
            tmem_st16(tP + 16 * (h0 + hh), Ph);
          }
          if (one) {
            uint32_t Z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) Z[e] = 0u;
            tmem_st16(tP + 16 * (1 - h0), Z);
          }
          const float2 s01 = add2(sum2[0], sum2[1]), s23 = add2(sum2[2], sum2[3]);
          const float2 s4 = add2(s01, s23);
          l += s4.x + s4.y;
        } else {
          uint32_t Z[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) Z[e] = 0u;
          tmem_st16(tP, Z);
          tmem_st16(tP + 16, Z);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[b2]);
        if (t == 0) release_pending();
      }
      if (!ok) break;
      u += n;
      // Wait for the item's last P V, then normalise O and write it.
      if (!mbar_wait(&bars.pv_done[(u - 1) & 1], ((u - 1) >> 1) & 1, &abort_flag,
                     p.status))
        break;
      tc_fence_after();
      const int r64 = row & 63;
      const bool write = (im.gvalid >> quarter) & 1;
      // Rows of a middle window or of an unchunked global item are final
      // here; a global chunk leaves an unnormalised partial (m, l, O).
      const bool whole = kWhole || !im.global;
      float inv = whole ? 1.f / l : 1.f;
      // Query-side mask: the output row of a padding token is 0 (chunked
      // global rows are zeroed when their chunks are combined).
      if (p.mask_q && write && whole && !p.key_mask[(size_t)im.b * p.L + tq]) inv = 0.f;
      const size_t grow = (size_t)im.bh * p.L + (size_t)(write ? im.t[half] : 0) * kTile + r64;
      float* part = p.part +
                    ((((size_t)im.bh * a.geo.n_git + im.gi) * a.geo.nchunks + im.chunk) * 128 +
                     row) * kPartStride;
      // Middle rows leave through shared memory and one TMA store per warp
      // (a row per lane would make every store instruction touch 32 lines).
      // The staging area is this warp's quarter of the item's Q slot: every
      // S MMA that read it has completed (they precede the last P V), and the
      // producer refills the slot only after this item's list_empty.
      uint8_t* stage = Qs + slot * 2 * kTileBytes + quarter * 4096;
      const bool tma_out = write && whole;
      // Not unrolled: runs once per item, so a small loop body costs less
      // instruction fetch than four copies.
#pragma unroll 1
      for (int q16 = 0; q16 < 4; ++q16) {
        uint32_t o[16];
        tmem_ld16(tO + q16 * 16, o);
        tmem_ld_wait();
        if (write) {
          float v[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(o[e]) * inv;
          if (whole) {
            // 16-byte chunks 2 q16 and 2 q16 + 1 of this row, 128-byte swizzle
            // (chunk index XOR row mod 8), as the store's tensor map expects.
            uint8_t* rowp = stage + lane * 128;
            const int c0 = 2 * q16;
            *reinterpret_cast<uint4*>(rowp + ((c0 ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                           pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
            *reinterpret_cast<uint4*>(rowp + (((c0 + 1) ^ (lane & 7)) << 4)) =
                make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]),
                           pack_bf16(v[12], v[13]), pack_bf16(v[14], v[15]));
          } else {
            float4* dst = reinterpret_cast<float4*>(part + q16 * 16);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          }
        }
      }
      tc_fence_before();
      if (tma_out) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars.o_empty);
        if (tma_out) {
          tma_store_2d(&tmO, stage, 0,
                       (int)((size_t)im.bh * p.L + (size_t)im.t[half] * kTile +
                             (quarter & 1) * 32));
          bulk_commit_group();
        } else {
          mbar_arrive(&bars.list_empty[slot]);
        }
      }
      if (tma_out) pend = slot;  // released after the store has read the rows
      if (write) {
        if (whole) {
          p.lse_out[grow] = (m + __log2f(l)) * (1.0f / kLog2e);
        } else {
          part[64] = m;
          part[65] = l;
        }
      }
    }
  }

  if (warp >= 2 && lane == 0) bulk_wait_all();  // output stores complete
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the global rows' split partials: one warp per row of a global item,
// lanes over d; rows outside the global blocks are skipped.
__global__ void __launch_bounds__(256) fwd_combine_kernel(const PairArgs a) {
  const Problem& p = a.p;
  const Geom& g = a.geo;
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
  const float* base = p.part + ((bh * g.n_git + gi) * g.nchunks * 128 + row) * kPartStride;
  // Unrolled so that several chunks' loads are in flight at once.
  float M = -INFINITY;
#pragma unroll 8
  for (int c = 0; c < g.nchunks; ++c) M = fmaxf(M, base[(size_t)c * 128 * kPartStride + 64]);
  float Lsum = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll 8
  for (int c = 0; c < g.nchunks; ++c) {
    const float* src = base + (size_t)c * 128 * kPartStride;
    const float w = ex2(src[64] - M);
    Lsum = fmaf(w, src[65], Lsum);
    const float2 o = reinterpret_cast<const float2*>(src)[lane];
    o0 = fmaf(w, o.x, o0);
    o1 = fmaf(w, o.y, o1);
  }
  const size_t tok = (size_t)t[row >> 6] * kTile + (row & 63);
  const size_t grow = bh * p.L + tok;
  // Query-side mask: the output row of a padding token is 0.
  const float inv =
      (p.mask_q && !p.key_mask[(bh / p.H) * p.L + tok]) ? 0.f : 1.f / Lsum;
  reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(p.out) +
                              grow * kHeadDim)[lane] =
      pack_bf16(o0 * inv, o1 * inv);
  if (lane == 0) p.lse_out[grow] = (M + __log2f(Lsum)) * (1.0f / kLog2e);
}

}  // namespace

// ---- host side ----------------------------------------------------------

size_t tc_fwd_part_bytes(const Problem& p) {
  const Geom g = make_geom(p);
  return (size_t)p.B * p.H * g.n_git * g.nchunks * 128 * kPartStride * sizeof(float);
}

bool tc_fwd_supported(const Problem& p) { return tc_shape_ok(p); }

cudaError_t launch_tc_fwd(const Problem& p, const TensorMaps& tm,
                          cudaStream_t s, EventMarks* marks) {
  const PairArgs a = make_pair_args(p);
  const size_t smem = 1024 + (2 * 2 + 2 * kNST) * kTileBytes;
  const bool whole = a.geo.nchunks == 1;
  const bool masked = p.key_mask != nullptr;
  using Kernel = void (*)(const PairArgs, const CUtensorMap, const CUtensorMap,
                          const CUtensorMap, const CUtensorMap);
  // [dropout][whole][mask][block 32]
  static const Kernel kernels[2][2][2][2] = {
      {{{tc_fwd_kernel<false, false, false, false>, tc_fwd_kernel<false, false, false, true>},
        {tc_fwd_kernel<false, false, true, false>, tc_fwd_kernel<false, false, true, true>}},
       {{tc_fwd_kernel<false, true, false, false>, tc_fwd_kernel<false, true, false, true>},
        {tc_fwd_kernel<false, true, true, false>, tc_fwd_kernel<false, true, true, true>}}},
      {{{tc_fwd_kernel<true, false, false, false>, tc_fwd_kernel<true, false, false, true>},
        {tc_fwd_kernel<true, false, true, false>, tc_fwd_kernel<true, false, true, true>}},
       {{tc_fwd_kernel<true, true, false, false>, tc_fwd_kernel<true, true, false, true>},
        {tc_fwd_kernel<true, true, true, false>, tc_fwd_kernel<true, true, true, true>}}}};
  const Kernel kernel = kernels[p.drop_thr ? 1 : 0][whole ? 1 : 0][masked ? 1 : 0]
                               [p.bs == 32 ? 1 : 0];
  cudaError_t e = cudaFuncSetAttribute(
      kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = min(a.items, 2 * sms);
  kernel<<<grid, kThreads, smem, s>>>(a, tm.q, tm.k, tm.v, tm.out32);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.geo.nchunks == 1) return cudaSuccess;  // global rows written whole
  e = marks->mark(s);
  if (e != cudaSuccess) return e;
  const size_t rows = (size_t)p.B * p.H * a.geo.n_git * 128;
  fwd_combine_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace bb
