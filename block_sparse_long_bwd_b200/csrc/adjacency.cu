// Backward preprocessing: D = rowsum(dO * O) and the transposed block
// adjacency (for each key block j, the sorted query blocks i with j in A(i)).
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

// One CTA per head.  Shared memory: count[nb], cursor[nb], tsum[1024].
__global__ void __launch_bounds__(kCsrThreads) csr_build_kernel(Problem p) {
  extern __shared__ int smi[];
  const int nb = p.nb, r = p.r, h = blockIdx.x, tid = threadIdx.x;
  int* cnt = smi;
  int* cur = cnt + nb;
  int* tsum = cur + nb;
  const int32_t* table = p.rand_idx + (size_t)h * nb * r;
  int* offs = p.csr_offs + (size_t)h * (nb + 1);
  int* list = p.csr_list + (size_t)h * p.csr_cap;

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
    cur[j] = run;
    offs[j] = run;
    run += cnt[j];
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
  if (!p.qplan) return;  // CUDA-core path: the CSR is all it needs

  // Tensor-core plans of this head.  Query side: the key tiles of every
  // item.  Key side: each item's walk over the query tiles that attend its
  // key rows (merging this head's CSR lists, complete after the barrier).
  __syncthreads();
  const Geom g = make_geom(p.L, p.bs);
  TileList* qplan = static_cast<TileList*>(p.qplan) + (size_t)h * g.per_bh;
  for (int loc = tid; loc < g.per_bh; loc += kCsrThreads)
    if (!build_tile_list(p, g, h, loc, qplan[loc])) set_status(p.status, BB_ERR_BAD_TABLE);
  int* kof = p.kof + (size_t)h * (g.per_bh + 1);
  uint32_t* kplan = p.kplan + (size_t)h * p.kcap;
  // pass 1: walk lengths, into tsum-chunked exclusive offsets
  const int kchunk = (g.per_bh + kCsrThreads - 1) / kCsrThreads;
  const int k0 = tid * kchunk, k1 = min(g.per_bh, k0 + kchunk);
  int klocal = 0;
  for (int loc = k0; loc < k1; ++loc) {
    KeyWalk w;
    w.init(g, p.H, p.csr_offs, p.csr_list, p.csr_cap, h * g.per_bh + loc);
    int tile, mask, n = 0;
    while (w.next(tile, mask)) ++n;
    kof[loc] = n;
    klocal += n;
  }
  __syncthreads();
  tsum[tid] = klocal;
  __syncthreads();
  for (int step = 1; step < kCsrThreads; step <<= 1) {
    int add = tid >= step ? tsum[tid - step] : 0;
    __syncthreads();
    tsum[tid] += add;
    __syncthreads();
  }
  int krun = tsum[tid] - klocal;
  for (int loc = k0; loc < k1; ++loc) {
    const int n = kof[loc];
    kof[loc] = krun;
    krun += n;
  }
  if (tid == kCsrThreads - 1) kof[g.per_bh] = tsum[kCsrThreads - 1];
  __syncthreads();
  // pass 2: fill (the planner sized kcap for the worst case of this table)
  for (int loc = k0; loc < k1; ++loc) {
    KeyWalk w;
    w.init(g, p.H, p.csr_offs, p.csr_list, p.csr_cap, h * g.per_bh + loc);
    int tile, mask, e = kof[loc];
    while (w.next(tile, mask)) {
      if (e < p.kcap) kplan[e] = kentry(tile, mask);
      ++e;
    }
  }
}

// Query-side plans for the forward: one thread per (head, item).
__global__ void __launch_bounds__(128) plan_q_kernel(Problem p) {
  const Geom g = make_geom(p.L, p.bs);
  const int id = blockIdx.x * 128 + threadIdx.x;
  if (id >= p.H * g.per_bh) return;
  const int h = id / g.per_bh, loc = id % g.per_bh;
  TileList* qplan = static_cast<TileList*>(p.qplan);
  if (!build_tile_list(p, g, h, loc, qplan[id])) set_status(p.status, BB_ERR_BAD_TABLE);
}

}  // namespace

cudaError_t launch_bwd_pre(const Problem& p, cudaStream_t s) {
  const size_t rows = (size_t)p.B * p.H * p.L;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (p.dtype == BB_F32)
    bwd_pre_kernel<float><<<grid, 256, 0, s>>>(p);
  else
    bwd_pre_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

size_t tc_items_per_bh(const Problem& p) { return make_geom(p.L, p.bs).per_bh; }

size_t tc_qplan_bytes(const Problem& p) {
  return (size_t)p.H * tc_items_per_bh(p) * sizeof(TileList);
}

// Upper bound of key-side walk entries per head: every entry of a middle
// window stands for at least one attended (query block, key block) pair
// (two tiles per block at block size 128); global items visit all tiles.
int tc_kplan_cap(const Problem& p) {
  const Geom g = make_geom(p.L, p.bs);
  return 2 * pair_cap(p.nb, p.r) + g.n_git * g.nt + 64;
}

cudaError_t launch_plan_q(const Problem& p, cudaStream_t s) {
  const int n = p.H * (int)tc_items_per_bh(p);
  plan_q_kernel<<<(n + 127) / 128, 128, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_csr_build(const Problem& p, cudaStream_t s) {
  const size_t smem = (size_t)(2 * p.nb + kCsrThreads) * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(
      csr_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  csr_build_kernel<<<p.H, kCsrThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace bb
