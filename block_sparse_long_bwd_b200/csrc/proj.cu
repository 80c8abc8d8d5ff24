// The projections on either side of the attention in the pages' encoder
// layer (key_dim = hidden / heads): the fused Q/K/V projection, whose
// epilogue writes Q, K and V straight into the [B][H][L][64] layout the
// attention kernels read, and the output projection, which reads the
// attention output O in that layout.  One tcgen05 GEMM kernel serves both:
//
//   out[m][n] = bias[n] + sum_k A[m][k] W[n][k]     (W: nn.Linear layout)
//
// QKV: A = x [B*L][hidden], W = w_qkv [3*H*64][hidden]; column n is feature
//      n % (H*64) of Q (n < H*64), K or V, i.e. head (n % (H*64)) / 64,
//      component n % 64; row m = b*L + l.
// OUT: A = O viewed as [B*L][H*64] with A[b*L + l][h*64 + j] = O[b][h][l][j]
//      (each 64-wide K step is one head: a 128-row block of O's row view),
//      W = w_o [hidden][H*64], out [B*L][hidden].
//
// Persistent kernel, one CTA per SM (192 threads): warp 0 lane 0 streams the
// 128 x 64 A tile and the 256 x 64 W tile of every K step through a 3-stage
// TMA ring; warp 1 lane 0 issues M128 x N256 x K16 tcgen05 MMAs (full tensor
// rate at N = 256) into one of two 256-column TMEM accumulators, so a tile's
// epilogue overlaps the next tile's MMAs; warps 2-5 (32 rows each) add the
// bias, round to bf16, stage 32 x 64 blocks in shared memory (128-byte
// swizzle) and write them with TMA stores.  Output tiles are ordered M-major
// (the 256-column tiles of one 128-row block run together), so an A block is
// read from HBM once and from L2 for the other column tiles.
#include "common.cuh"
#include "sm100.cuh"

namespace bb {
namespace {

using namespace sm100;

constexpr int kPBM = 128, kPBN = 256, kPBK = 64;
constexpr int kPStages = 3;
constexpr uint32_t kPATile = kPBM * kPBK * 2;            // 16 KB
constexpr uint32_t kPBTile = kPBN * kPBK * 2;            // 32 KB
constexpr uint32_t kPStageBytes = kPATile + kPBTile;     // 48 KB
constexpr uint32_t kPStageOut = 4 * 4 * 4096;            // 4 warps x 4 blocks x 32 x 128 B
constexpr int kPThreads = 192;
constexpr uint32_t kPTmemCols = 512;                     // two 128 x 256 fp32 accumulators

struct ProjArgs {
  int mode;           // 0: Q/K/V projection, 1: output projection
  int M, N, K;        // rows (B*L), columns, reduction
  int B, L, H;        // attention geometry (head dim 64)
  int n_tiles_n;      // 256-column tiles along N
  int tiles;          // output tiles
  const float* bias;  // [N] or null
  int* status;        // device status word (bounded waits)
};

struct PBars {
  uint64_t full[kPStages], empty[kPStages], acc_full[2], acc_empty[2];
};

__global__ void __launch_bounds__(kPThreads, 1)
    proj_kernel(const __grid_constant__ ProjArgs pa, const __grid_constant__ CUtensorMap tmA,
                const __grid_constant__ CUtensorMap tmW,
                const __grid_constant__ CUtensorMap tmO0,
                const __grid_constant__ CUtensorMap tmO1,
                const __grid_constant__ CUtensorMap tmO2) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ PBars bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stages = base;                             // [kPStages][A | W]
  uint8_t* stage_out = base + kPStages * kPStageBytes;  // [4 warps][4 blocks][32][128 B]
  const int ksteps = pa.K / kPBK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.acc_full[s], 1);
      mbar_init(&bars.acc_empty[s], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kPTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmO0);
    if (pa.mode == 0) {
      prefetch_tmap(&tmO1);
      prefetch_tmap(&tmO2);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ---------------- TMA loads (one thread) ----------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < pa.tiles && ok; tile += gridDim.x) {
        const int m0 = (tile / pa.n_tiles_n) * kPBM, n0 = (tile % pa.n_tiles_n) * kPBN;
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const uint32_t st = it % kPStages;
          if (!mbar_wait(&bars.empty[st], ((it / kPStages) & 1) ^ 1, &abort_flag, pa.status)) {
            ok = false;
            break;
          }
          uint8_t* a = stages + st * kPStageBytes;
          mbar_expect_tx(&bars.full[st], kPStageBytes);
          if (pa.mode == 0) {
            tma_load_2d(a, &tmA, &bars.full[st], ks * kPBK, m0);
          } else {
            // K step ks is head ks: rows (b*H + ks)*L + l0 .. + 127 of O.
            const int b = m0 / pa.L, l0 = m0 % pa.L;
            tma_load_2d(a, &tmA, &bars.full[st], 0, (b * pa.H + ks) * pa.L + l0);
          }
          tma_load_2d(a + kPATile, &tmW, &bars.full[st], ks * kPBK, n0);
        }
      }
      if (abort_flag) {
        // Let issued copies land before shared memory goes away.
        for (uint32_t s = 0; s < (uint32_t)kPStages; ++s)
          if (it >= s + 1) {
            const uint32_t last = it - 1 - ((it - 1 - s) % kPStages);
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&bars.full[s], (last / kPStages) & 1) &&
                   globaltimer() - t0 < 100000000ull) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue (one thread) ----------------
    const uint32_t idesc = idesc_bf16(kPBM, kPBN, 0, 0);  // A, W both K-major
    uint32_t it = 0, tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < pa.tiles && ok; tile += gridDim.x, ++tc) {
      const int acc = tc & 1;
      if (!mbar_wait(&bars.acc_empty[acc], ((tc >> 1) & 1) ^ 1, &abort_flag, pa.status)) break;
      tc_fence_after();
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const uint32_t st = it % kPStages;
        if (!mbar_wait(&bars.full[st], (it / kPStages) & 1, &abort_flag, pa.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t aaddr = smem_u32(stages + st * kPStageBytes);
          const uint32_t waddr = aaddr + kPATile;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + acc * kPBN, sdesc_sw128(aaddr + kk * 32, 16),
                   sdesc_sw128(waddr + kk * 32, 16), idesc, (ks > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars.empty[st]);
          if (ks == ksteps - 1) mma_commit(&bars.acc_full[acc]);
        }
        __syncwarp();
      }
    }
  } else {
    // ---------------- epilogue (warps 2-5, 32 rows each) ----------------
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint8_t* stage = stage_out + quarter * 4 * 4096;
    uint32_t tc = 0;
    for (int tile = blockIdx.x; tile < pa.tiles; tile += gridDim.x, ++tc) {
      const int acc = tc & 1;
      const int m0 = (tile / pa.n_tiles_n) * kPBM, n0 = (tile % pa.n_tiles_n) * kPBN;
      if (!mbar_wait(&bars.acc_full[acc], (tc >> 1) & 1, &abort_flag, pa.status)) break;
      tc_fence_after();
      // The previous tile's stores have read this warp's staging area.
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + acc * kPBN + cb * 64 + lane_off, v0);
        tmem_ld32(tmem + acc * kPBN + cb * 64 + 32 + lane_off, v1);
        tmem_ld_wait();
        const int c0 = n0 + cb * 64;
        uint8_t* rowp = stage + cb * 4096 + lane * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {  // 16-byte chunk = 8 columns
          const uint32_t* src = ch < 4 ? v0 + 8 * ch : v1 + 8 * (ch - 4);
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(src[e]);
          if (pa.bias) {
            const float4 b0 = __ldg(reinterpret_cast<const float4*>(pa.bias + c0 + 8 * ch));
            const float4 b1 = __ldg(reinterpret_cast<const float4*>(pa.bias + c0 + 8 * ch + 4));
            f[0] += b0.x; f[1] += b0.y; f[2] += b0.z; f[3] += b0.w;
            f[4] += b1.x; f[5] += b1.y; f[6] += b1.z; f[7] += b1.w;
          }
          // 128-byte swizzle: chunk index XOR row mod 8, as the map expects.
          *reinterpret_cast<uint4*>(rowp + ((ch ^ (lane & 7)) << 4)) =
              make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                         pack_bf16(f[6], f[7]));
        }
      }
      // The accumulator is in registers / shared memory: the MMAs of the
      // tile after next may overwrite it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.acc_empty[acc]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        for (int cb = 0; cb < 4; ++cb) {
          if (pa.mode == 0) {
            const int hd = pa.H * 64;
            const int which = (n0 + cb * 64) / hd;        // 0 Q, 1 K, 2 V
            const int h = ((n0 + cb * 64) % hd) / 64;
            const int b = m0 / pa.L, l0 = m0 % pa.L;
            const CUtensorMap* map = which == 0 ? &tmO0 : which == 1 ? &tmO1 : &tmO2;
            tma_store_2d(map, stage + cb * 4096, 0, (b * pa.H + h) * pa.L + l0 + quarter * 32);
          } else {
            tma_store_2d(&tmO0, stage + cb * 4096, n0 + cb * 64, m0 + quarter * 32);
          }
        }
        bulk_commit_group();
      }
    }
    if (lane == 0) bulk_wait_all();  // output stores complete
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kPTmemCols);
  }
}

bool aligned16p(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int launch_proj(ProjArgs pa, const void* a, uint64_t a_inner, uint64_t a_rows, const void* w,
                void* o0, void* o1, void* o2, void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || ws_bytes < 256) return BB_ERR_WORKSPACE;
  if (!aligned16p(workspace)) return BB_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  pa.status = static_cast<int*>(workspace);
  CUtensorMap tmA, tmW, tmO0, tmO1, tmO2;
  const uint64_t rows_bhl = (uint64_t)pa.B * pa.H * pa.L;
  bool ok = encode_bf16_2d(&tmA, a, a_inner, a_rows, a_inner, 64, kPBM) &&
            encode_bf16_2d(&tmW, w, pa.K, pa.N, pa.K, 64, kPBN);
  if (pa.mode == 0) {
    ok = ok && encode_bf16_2d(&tmO0, o0, 64, rows_bhl, 64, 64, 32) &&
         encode_bf16_2d(&tmO1, o1, 64, rows_bhl, 64, 64, 32) &&
         encode_bf16_2d(&tmO2, o2, 64, rows_bhl, 64, 64, 32);
  } else {
    ok = ok && encode_bf16_2d(&tmO0, o0, pa.N, pa.M, pa.N, 64, 32);
    tmO1 = tmO0;
    tmO2 = tmO0;
  }
  if (!ok) return BB_ERR_CUDA;
  if (cudaMemsetAsync(pa.status, 0, sizeof(int), s) != cudaSuccess) return BB_ERR_CUDA;
  const size_t smem = 1024 + kPStages * kPStageBytes + kPStageOut;
  if (cudaFuncSetAttribute(proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return BB_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  proj_kernel<<<min(pa.tiles, sms), kPThreads, smem, s>>>(pa, tmA, tmW, tmO0, tmO1, tmO2);
  return cudaGetLastError() == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}

}  // namespace
}  // namespace bb

using namespace bb;

extern "C" {

int bb_qkv_proj(int B, int L, int hidden, int H, const void* x, const void* w_qkv,
                const float* b_qkv, void* q, void* k, void* v, void* workspace,
                size_t workspace_bytes, void* stream) {
  if (B <= 0 || L <= 0 || hidden <= 0 || H <= 0) return BB_ERR_INVALID;
  if (!x || !w_qkv || !q || !k || !v) return BB_ERR_INVALID;
  const void* ptrs[] = {x, w_qkv, b_qkv, q, k, v};
  for (const void* p : ptrs)
    if (!aligned16p(p)) return BB_ERR_INVALID;
  // Tiles: 128 rows within one sequence, 256 columns within one of Q, K, V.
  if (L % kPBM != 0 || hidden % kPBK != 0 || (H * 64) % kPBN != 0) return BB_ERR_UNSUPPORTED;
  if ((uint64_t)B * H * L >= (1ull << 31) || (uint64_t)B * L * hidden >= (1ull << 31))
    return BB_ERR_UNSUPPORTED;
  ProjArgs pa{};
  pa.mode = 0;
  pa.M = B * L;
  pa.N = 3 * H * 64;
  pa.K = hidden;
  pa.B = B;
  pa.L = L;
  pa.H = H;
  pa.n_tiles_n = pa.N / kPBN;
  pa.tiles = (pa.M / kPBM) * pa.n_tiles_n;
  pa.bias = b_qkv;
  return launch_proj(pa, x, hidden, (uint64_t)B * L, w_qkv, q, k, v, workspace,
                     workspace_bytes, stream);
}

int bb_out_proj(int B, int L, int H, int hidden, const void* o, const void* w_o,
                const float* b_o, void* out, void* workspace, size_t workspace_bytes,
                void* stream) {
  if (B <= 0 || L <= 0 || hidden <= 0 || H <= 0) return BB_ERR_INVALID;
  if (!o || !w_o || !out) return BB_ERR_INVALID;
  const void* ptrs[] = {o, w_o, b_o, out};
  for (const void* p : ptrs)
    if (!aligned16p(p)) return BB_ERR_INVALID;
  if (L % kPBM != 0 || hidden % kPBN != 0) return BB_ERR_UNSUPPORTED;
  if ((uint64_t)B * H * L >= (1ull << 31) || (uint64_t)B * L * hidden >= (1ull << 31))
    return BB_ERR_UNSUPPORTED;
  ProjArgs pa{};
  pa.mode = 1;
  pa.M = B * L;
  pa.N = hidden;
  pa.K = H * 64;
  pa.B = B;
  pa.L = L;
  pa.H = H;
  pa.n_tiles_n = pa.N / kPBN;
  pa.tiles = (pa.M / kPBM) * pa.n_tiles_n;
  pa.bias = b_o;
  return launch_proj(pa, o, 64, (uint64_t)B * H * L, w_o, out, nullptr, nullptr, workspace,
                     workspace_bytes, stream);
}

}  // extern "C"
