// CUDA-core (FFMA) kernels of the block-sparse attention, one thread per
// token row.  They serve fp32 I/O, where a single tensor-core pass cannot
// reach fp32 accuracy, and every shape the tensor-core kernels do not take.
//
// Forward: one CTA per (b, h, query block i) walks the sorted attended set
// A(i) (all nb blocks for the global rows 0 and nb-1), staging each key and
// value block in shared memory, with an online softmax in the log2 domain.
// Backward: dQ per query block as above; dK/dV per key block over the
// transposed block adjacency (CSR, built by csr_build_kernel), without
// atomics.  With dropout each element's keep decision is drawn on its own
// (one Philox call per element; these kernels are the fp32 correctness path).
#include "common.cuh"
#include "dropout.cuh"

namespace bb {
namespace {

constexpr int kChunk = 32;  // keys scored per online-softmax step

template <typename T>
__device__ __forceinline__ void load_tile(float* dst, const T* src, int n,
                                          int tid, int nthreads) {
  for (int e = tid; e < n; e += nthreads) dst[e] = to_f(src[e]);
}

__device__ __forceinline__ float dot64(const float* a, const float* row) {
  const float4* r4 = reinterpret_cast<const float4*>(row);
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    float4 x = r4[c];
    acc = fmaf(a[4 * c + 0], x.x, acc);
    acc = fmaf(a[4 * c + 1], x.y, acc);
    acc = fmaf(a[4 * c + 2], x.z, acc);
    acc = fmaf(a[4 * c + 3], x.w, acc);
  }
  return acc;
}

__device__ __forceinline__ float dot32(const float* a, const float* row) {
  const float4* r4 = reinterpret_cast<const float4*>(row);
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float4 x = r4[c];
    acc = fmaf(a[4 * c + 0], x.x, acc);
    acc = fmaf(a[4 * c + 1], x.y, acc);
    acc = fmaf(a[4 * c + 2], x.z, acc);
    acc = fmaf(a[4 * c + 3], x.w, acc);
  }
  return acc;
}

// Key offsets in the log2 domain: 0 for attended keys, mask_value*log2(e)
// for masked ones.
__device__ __forceinline__ float key_off(const Problem& p, int b, int u) {
  if (!p.key_mask) return 0.f;
  return p.key_mask[(size_t)b * p.L + u] ? 0.f : p.mask_value * kLog2e;
}

template <typename T, int BS>
__global__ void __launch_bounds__(BS) simt_fwd_kernel(Problem p) {
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Vs = Ks + BS * kHeadDim;
  float* koff = Vs + BS * kHeadDim;
  __shared__ int blist[5 + kMaxRand];
  __shared__ int nlist;

  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int nb = p.nb;
  const bool global_row = (i == 0 || i == nb - 1);
  if (tid == 0 && !global_row)
    nlist = middle_row_blocks(p.rand_idx + ((size_t)h * nb + i) * p.r, p.r,
                              i, nb, blist, p.status);
  const size_t bh = (size_t)b * p.H + h;
  const T* Qg = static_cast<const T*>(p.q) + (bh * p.L + (size_t)i * BS) * kHeadDim;
  const T* Kg = static_cast<const T*>(p.k) + bh * p.L * kHeadDim;
  const T* Vg = static_cast<const T*>(p.v) + bh * p.L * kHeadDim;

  const float sl2 = p.scale * kLog2e;
  float q[kHeadDim], o[kHeadDim];
#pragma unroll
  for (int c = 0; c < kHeadDim; ++c) {
    q[c] = to_f(Qg[(size_t)tid * kHeadDim + c]) * sl2;
    o[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  __syncthreads();
  const int n = global_row ? nb : nlist;
  for (int a = 0; a < n; ++a) {
    const int j = global_row ? a : blist[a];
    __syncthreads();
    load_tile(Ks, Kg + (size_t)j * BS * kHeadDim, BS * kHeadDim, tid, BS);
    load_tile(Vs, Vg + (size_t)j * BS * kHeadDim, BS * kHeadDim, tid, BS);
    koff[tid] = key_off(p, b, j * BS + tid);
    __syncthreads();
#pragma unroll 1
    for (int c0 = 0; c0 < BS; c0 += kChunk) {
      float s[kChunk];
      float cm = -INFINITY;
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        s[u] = dot64(q, Ks + (c0 + u) * kHeadDim) + koff[c0 + u];
        cm = fmaxf(cm, s[u]);
      }
      const float mn = fmaxf(m, cm);
      const float alpha = exp2f(m - mn);  // m = -inf -> 0
      l *= alpha;
#pragma unroll
      for (int c = 0; c < kHeadDim; ++c) o[c] *= alpha;
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        const float pu = exp2f(s[u] - mn);
        l += pu;  // the lse is that of the undropped softmax
        float pw = pu;
        if (p.drop_thr)
          pw = keep_one(p, b, h, i * BS + tid, j * BS + c0 + u) ? pu * p.drop_scale : 0.f;
        const float4* v4 = reinterpret_cast<const float4*>(Vs + (c0 + u) * kHeadDim);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float4 x = v4[c];
          o[4 * c + 0] = fmaf(pw, x.x, o[4 * c + 0]);
          o[4 * c + 1] = fmaf(pw, x.y, o[4 * c + 1]);
          o[4 * c + 2] = fmaf(pw, x.z, o[4 * c + 2]);
          o[4 * c + 3] = fmaf(pw, x.w, o[4 * c + 3]);
        }
      }
      m = mn;
    }
  }
  // Query-side mask: the output row of a padding token is 0.
  const bool qpad = p.mask_q && !p.key_mask[(size_t)b * p.L + (size_t)i * BS + tid];
  const float inv = qpad ? 0.f : 1.f / l;
  T* Og = static_cast<T*>(p.out) + (bh * p.L + (size_t)i * BS + tid) * kHeadDim;
#pragma unroll
  for (int c = 0; c < kHeadDim; ++c) Og[c] = from_f<T>(o[c] * inv);
  p.lse_out[bh * p.L + (size_t)i * BS + tid] = (m + log2f(l)) * (1.0f / kLog2e);
}

// dQ for query block i: recompute p from lse, dp = <dO, v>, ds = p (dp - D),
// dq = scale * sum ds k.
template <typename T, int BS>
__global__ void __launch_bounds__(BS) simt_dq_kernel(Problem p) {
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Vs = Ks + BS * kHeadDim;
  float* koff = Vs + BS * kHeadDim;
  __shared__ int blist[5 + kMaxRand];
  __shared__ int nlist;

  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int nb = p.nb;
  const bool global_row = (i == 0 || i == nb - 1);
  if (tid == 0 && !global_row)
    nlist = middle_row_blocks(p.rand_idx + ((size_t)h * nb + i) * p.r, p.r,
                              i, nb, blist, p.status);
  const size_t bh = (size_t)b * p.H + h;
  const size_t row = bh * p.L + (size_t)i * BS + tid;
  const T* Kg = static_cast<const T*>(p.k) + bh * p.L * kHeadDim;
  const T* Vg = static_cast<const T*>(p.v) + bh * p.L * kHeadDim;
  const float sl2 = p.scale * kLog2e;
  float q[kHeadDim], g[kHeadDim], dq[kHeadDim];
#pragma unroll
  for (int c = 0; c < kHeadDim; ++c) {
    q[c] = to_f(static_cast<const T*>(p.q)[row * kHeadDim + c]) * sl2;
    g[c] = to_f(static_cast<const T*>(p.dout)[row * kHeadDim + c]);
    dq[c] = 0.f;
  }
  // Query-side mask: a padding token's p is 0 (lse taken as +inf).
  const float lse2 = (p.mask_q && !p.key_mask[(size_t)b * p.L + (size_t)i * BS + tid])
                         ? INFINITY
                         : p.lse[row] * kLog2e;
  const float Dt = p.D[row];
  __syncthreads();
  const int n = global_row ? nb : nlist;
  for (int a = 0; a < n; ++a) {
    const int j = global_row ? a : blist[a];
    __syncthreads();
    load_tile(Ks, Kg + (size_t)j * BS * kHeadDim, BS * kHeadDim, tid, BS);
    load_tile(Vs, Vg + (size_t)j * BS * kHeadDim, BS * kHeadDim, tid, BS);
    koff[tid] = key_off(p, b, j * BS + tid);
    __syncthreads();
#pragma unroll 2
    for (int u = 0; u < BS; ++u) {
      const float* kr = Ks + u * kHeadDim;
      const float pu = exp2f(dot64(q, kr) + koff[u] - lse2);
      float dpv = dot64(g, Vs + u * kHeadDim);
      if (p.drop_thr)
        dpv = keep_one(p, b, h, i * BS + tid, j * BS + u) ? dpv * p.drop_scale : 0.f;
      const float ds = pu * (dpv - Dt);
      const float4* k4 = reinterpret_cast<const float4*>(kr);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float4 x = k4[c];
        dq[4 * c + 0] = fmaf(ds, x.x, dq[4 * c + 0]);
        dq[4 * c + 1] = fmaf(ds, x.y, dq[4 * c + 1]);
        dq[4 * c + 2] = fmaf(ds, x.z, dq[4 * c + 2]);
        dq[4 * c + 3] = fmaf(ds, x.w, dq[4 * c + 3]);
      }
    }
  }
  const size_t q0 = (size_t)row * kHeadDim;
#pragma unroll
  for (int c = 0; c < kHeadDim; ++c) store_grad<T>(p, p.dq, q0 + c, dq[c] * p.scale);
}

// dK/dV for key block j over the query blocks of its CSR list.  Two threads
// per key row, each holding half of d; partial dots meet by one shuffle.
template <typename T, int BS>
__global__ void __launch_bounds__(2 * BS) simt_dkdv_kernel(Problem p) {
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;                         // [BS][64], pre-scaled by scale*log2e
  float* Gs = Qs + BS * kHeadDim;         // dO [BS][64]
  float* lse2 = Gs + BS * kHeadDim;       // [BS]
  float* Ds = lse2 + BS;                  // [BS]

  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int u = tid >> 1, half = tid & 1;
  const size_t bh = (size_t)b * p.H + h;
  const size_t krow = bh * p.L + (size_t)j * BS + u;
  const T* Kg = static_cast<const T*>(p.k) + krow * kHeadDim + half * 32;
  const T* Vg = static_cast<const T*>(p.v) + krow * kHeadDim + half * 32;
  float kr[32], vr[32], dk[32], dv[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    kr[c] = to_f(Kg[c]);
    vr[c] = to_f(Vg[c]);
    dk[c] = 0.f;
    dv[c] = 0.f;
  }
  const float ko = key_off(p, b, j * BS + u);
  const float sl2 = p.scale * kLog2e;
  const int* offs = p.csr_offs + (size_t)h * (p.nb + 1);
  const int* list = p.csr_list + (size_t)h * p.csr_cap;
  const int beg = offs[j], end = offs[j + 1];
  const T* Qb = static_cast<const T*>(p.q) + bh * p.L * kHeadDim;
  const T* Gb = static_cast<const T*>(p.dout) + bh * p.L * kHeadDim;
  for (int e = beg; e < end; ++e) {
    const int i = list[e];
    __syncthreads();
    for (int x = tid; x < BS * kHeadDim; x += 2 * BS) {
      Qs[x] = to_f(Qb[(size_t)i * BS * kHeadDim + x]) * sl2;
      Gs[x] = to_f(Gb[(size_t)i * BS * kHeadDim + x]);
    }
    if (tid < BS) {
      // Query-side mask: a padding token's p is 0 (lse taken as +inf).
      lse2[tid] = (p.mask_q && !p.key_mask[(size_t)b * p.L + (size_t)i * BS + tid])
                      ? INFINITY
                      : p.lse[bh * p.L + (size_t)i * BS + tid] * kLog2e;
      Ds[tid] = p.D[bh * p.L + (size_t)i * BS + tid];
    }
    __syncthreads();
#pragma unroll 2
    for (int t = 0; t < BS; ++t) {
      const float* qt = Qs + t * kHeadDim + half * 32;
      const float* gt = Gs + t * kHeadDim + half * 32;
      float s = dot32(kr, qt);
      float dp = dot32(vr, gt);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      const float pu = exp2f(s + ko - lse2[t]);
      float pw = pu;
      if (p.drop_thr) {
        const float m = keep_one(p, b, h, i * BS + t, j * BS + u) ? p.drop_scale : 0.f;
        dp *= m;
        pw = pu * m;
      }
      const float ds = pu * (dp - Ds[t]);
      const float4* q4 = reinterpret_cast<const float4*>(qt);
      const float4* g4 = reinterpret_cast<const float4*>(gt);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float4 a = g4[c], qq = q4[c];
        dv[4 * c + 0] = fmaf(pw, a.x, dv[4 * c + 0]);
        dv[4 * c + 1] = fmaf(pw, a.y, dv[4 * c + 1]);
        dv[4 * c + 2] = fmaf(pw, a.z, dv[4 * c + 2]);
        dv[4 * c + 3] = fmaf(pw, a.w, dv[4 * c + 3]);
        dk[4 * c + 0] = fmaf(ds, qq.x, dk[4 * c + 0]);
        dk[4 * c + 1] = fmaf(ds, qq.y, dk[4 * c + 1]);
        dk[4 * c + 2] = fmaf(ds, qq.z, dk[4 * c + 2]);
        dk[4 * c + 3] = fmaf(ds, qq.w, dk[4 * c + 3]);
      }
    }
  }
  // Qs held q * scale * log2(e); dk = scale * sum ds q = sum ds (Qs / log2 e).
  const size_t k0 = (size_t)krow * kHeadDim + half * 32;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    store_grad<T>(p, p.dk, k0 + c, dk[c] * (1.0f / kLog2e));
    store_grad<T>(p, p.dv, k0 + c, dv[c]);
  }
}

template <typename T, int BS>
cudaError_t fwd_t(const Problem& p, cudaStream_t s) {
  const size_t smem = (size_t)(2 * BS * kHeadDim + BS) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(simt_fwd_kernel<T, BS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  simt_fwd_kernel<T, BS><<<dim3(p.nb, p.H, p.B), BS, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int BS>
cudaError_t bwd_t(const Problem& p, cudaStream_t s, EventMarks* marks) {
  const size_t smem = (size_t)(2 * BS * kHeadDim + 2 * BS) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(simt_dq_kernel<T, BS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(simt_dkdv_kernel<T, BS>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  simt_dq_kernel<T, BS><<<dim3(p.nb, p.H, p.B), BS, smem, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = marks->mark(s);
  if (e != cudaSuccess) return e;
  simt_dkdv_kernel<T, BS><<<dim3(p.nb, p.H, p.B), 2 * BS, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_fwd(const Problem& p, cudaStream_t s) {
  if (p.dtype == BB_F32) {
    if (p.bs == 32) return fwd_t<float, 32>(p, s);
    if (p.bs == 64) return fwd_t<float, 64>(p, s);
    return fwd_t<float, 128>(p, s);
  }
  if (p.bs == 32) return fwd_t<__nv_bfloat16, 32>(p, s);
  if (p.bs == 64) return fwd_t<__nv_bfloat16, 64>(p, s);
  return fwd_t<__nv_bfloat16, 128>(p, s);
}

cudaError_t launch_simt_bwd(const Problem& p, cudaStream_t s, EventMarks* marks) {
  if (p.dtype == BB_F32) {
    if (p.bs == 32) return bwd_t<float, 32>(p, s, marks);
    if (p.bs == 64) return bwd_t<float, 64>(p, s, marks);
    return bwd_t<float, 128>(p, s, marks);
  }
  if (p.bs == 32) return bwd_t<__nv_bfloat16, 32>(p, s, marks);
  if (p.bs == 64) return bwd_t<__nv_bfloat16, 64>(p, s, marks);
  return bwd_t<__nv_bfloat16, 128>(p, s, marks);
}

}  // namespace bb
