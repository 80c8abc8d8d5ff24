// Internal declarations shared by the host API and the kernels of
// libbbattn.so.  Not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/bb_attn.h"

namespace bb {

constexpr int kHeadDim = 64;       // d supported by this release
constexpr int kMaxBlocks = 8192;   // nb limit (CSR builder keeps counts in smem)
constexpr int kMaxRand = 32;       // r limit (attended list fits in smem)
constexpr float kLog2e = 1.4426950408889634f;

// Everything a kernel needs about one call, passed by value.
struct Problem {
  int B, H, L, d, bs, r, nb, dtype;
  float scale;       // resolved (never 0)
  float mask_value;  // resolved (never 0)
  // attention dropout: byte threshold (0: off), 1 / keep probability, seed
  uint32_t drop_thr;
  float drop_scale;
  uint64_t drop_seed;
  int mask_q;  // 1: key_mask also zeroes the output rows of padding tokens
  int grad_f32;  // 1: dq, dk, dv are written as fp32 (else in dtype)
  // inputs
  const void* q;
  const void* k;
  const void* v;
  const void* o;     // bwd
  const void* dout;  // bwd
  const float* lse;  // bwd
  const uint8_t* key_mask;
  const int32_t* rand_idx;
  // outputs
  void* out;
  float* lse_out;
  void* dq;
  void* dk;
  void* dv;
  // workspace pieces
  int* status;
  int* sched;        // [4] work counters of the tensor-core launches (zeroed by the plan kernel)
  float* D;          // [B*H*L] (bwd)
  int* csr_offs;     // [H][nb+1] (bwd)
  int* csr_list;     // [H][csr_cap] (bwd)
  int csr_cap;
  float* part;       // split partials (tensor-core path)
  size_t part_floats;
  // tensor-core plans (see tc_common.cuh)
  void* qplan;       // [H][items per (b, h)] tile lists, query side
  int* kof;          // [H * items][2] (start, length) of the key-side walks,
                     // then [H] allocation counters
  uint32_t* kplan;   // [H][kcap] key-side walk entries
  int kcap;
  // with a key mask: per batch b, word 0 = 1 when key tiles may be skipped
  // (a key among the first 32 is valid), then one bit per 64-token tile
  // whose keys are all masked; [B][tdead_words] (built by the plan launch of
  // either pass)
  uint32_t* tdead;
  int tdead_words;
  // dropout keep decisions carried from the forward to the backward
  // (caller buffer, tensor-core path only; nullptr: drawn in every pass):
  // keep_slots slots of bs x bs bits per (b, h), see keep_slot()
  uint32_t* keep_bits;
  int keep_slots;
};

// Slots of the stored keep bits per (b, h): one per attended (query block,
// key block) pair, with a fixed stride of 5 + r for the middle blocks.
inline int keep_slots_per_bh(int nb, int r) {
  return nb == 1 ? 1 : 2 * nb + (nb - 2) * (5 + r);
}

// Upper bound of attended (query block, key block) pairs per head.
inline int pair_cap(int nb, int r) { return nb * (7 + r) + 8; }

// Workspace layout, identical for sizing and for carving.
struct WsLayout {
  size_t status_off, D_off, offs_off, list_off, part_off;
  size_t qplan_off, kof_off, kplan_off;  // tensor-core plans (0: none)
  size_t tdead_off;                      // masked-tile bitmap (0: none)
  size_t total;
};
WsLayout ws_layout(const Problem& p, int pass);

// Records caller-provided timing events between internal launches.
struct EventMarks {
  void* const* ev = nullptr;
  int n = 0;
  int next = 0;
  cudaError_t mark(cudaStream_t s) {
    if (next < n && ev && ev[next]) {
      cudaError_t e = cudaEventRecord((cudaEvent_t)ev[next], s);
      ++next;
      return e;
    }
    ++next;
    return cudaSuccess;
  }
};

// TMA descriptors of the [B*H*L][64] bf16 row views of Q, K, V (and more
// for the backward), 64 x 64 boxes, 128-byte swizzle.
struct TensorMaps {
  CUtensorMap q, k, v, o, dout;
  CUtensorMap out32;  // forward output, 32-row boxes (one softmax warp's rows)
};
// Encodes the maps a pass needs; false if the driver entry point or the
// encode call fails.
bool encode_tensor_maps(const Problem& p, int pass, TensorMaps* tm);
// 2-D bf16 map over [rows][inner] (row stride in elements, a multiple of 8),
// box box_inner x box_rows, 128-byte swizzle (box_inner = 64).
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_stride, uint32_t box_inner, uint32_t box_rows);

// Tensor-core path (bf16, block 64, d 64).
bool tc_fwd_supported(const Problem& p);
size_t tc_fwd_part_bytes(const Problem& p);
cudaError_t launch_tc_fwd(const Problem& p, const TensorMaps& tm,
                          cudaStream_t s, EventMarks* marks);

bool tc_bwd_supported(const Problem& p);
size_t tc_qplan_bytes(const Problem& p);
// Words per batch of the forward's masked-tile bitmap (a flag word, then one
// bit per 64-key tile).
int tc_tdead_words(const Problem& p);
int tc_kplan_cap(const Problem& p);
size_t tc_items_per_bh(const Problem& p);      // query side
size_t tc_key_items_per_bh(const Problem& p);  // key side
cudaError_t launch_plan(const Problem& p, bool key_side, cudaStream_t s);
size_t tc_bwd_extra_bytes(const Problem& p);
// Number of dK/dV launches of the tensor-core backward (1, or 2 at lengths
// where the global key blocks run with the hi/lo split on their own).
int tc_dkdv_launches(const Problem& p);
// True when the forward's (pass 0) or the backward's (pass 1) global rows
// are split into chunks whose partials a merge launch (fwd_combine /
// bwd_finish) combines; false when they run whole.
bool tc_global_rows_chunked(const Problem& p, int pass);
cudaError_t launch_tc_bwd(const Problem& p, const TensorMaps& tm,
                          cudaStream_t s, EventMarks* marks);

// Launchers (return cudaError_t of the launch).
cudaError_t launch_simt_fwd(const Problem& p, cudaStream_t s);
cudaError_t launch_bwd_pre(const Problem& p, cudaStream_t s);
cudaError_t launch_csr_build(const Problem& p, cudaStream_t s);
// Backward plans (query and key side, with each head's transposed adjacency
// built in shared memory) in one launch; possible when a head's adjacency
// fits in shared memory (tc_bwd_plan_fused).
bool tc_bwd_plan_fused(const Problem& p);
cudaError_t launch_plan_bwd(const Problem& p, cudaStream_t s);
cudaError_t launch_simt_bwd(const Problem& p, cudaStream_t s, EventMarks* marks);

// ---- device helpers -----------------------------------------------------

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Element i of a gradient output: fp32 when the call asked for fp32
// gradients, else the I/O type T (rounded to nearest even from x).
template <typename T>
__device__ __forceinline__ void store_grad(const Problem& p, void* base, size_t i, float x) {
  if (p.grad_f32)
    static_cast<float*>(base)[i] = x;
  else
    static_cast<T*>(base)[i] = from_f<T>(x);
}

// Record the first non-OK status of a call (integer atomic, not a result).
__device__ __forceinline__ void set_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

// Sorted set A(i) of key blocks for a middle query block i (0 < i < nb-1):
// {0, i-1, i, i+1, nb-1} U rand row, each once.  Entries outside [-1, nb)
// are ignored and flagged.  Returns the count written to out (<= 5 + r).
__device__ __forceinline__ int middle_row_blocks(const int32_t* rand_row,
                                                 int r, int i, int nb,
                                                 int* out, int* status) {
  int n = 0;
  int base[5] = {0, i - 1, i, i + 1, nb - 1};
  for (int a = 0; a < 5; ++a) {
    int j = base[a];
    bool dup = false;
    for (int c = 0; c < n; ++c) dup |= (out[c] == j);
    if (!dup) out[n++] = j;
  }
  for (int a = 0; a < r; ++a) {
    int j = rand_row[a];
    if (j == -1) continue;
    if (j < 0 || j >= nb) {
      set_status(status, BB_ERR_BAD_TABLE);
      continue;
    }
    bool dup = false;
    for (int c = 0; c < n; ++c) dup |= (out[c] == j);
    if (!dup) out[n++] = j;
  }
  // insertion sort (n is small)
  for (int a = 1; a < n; ++a) {
    int x = out[a];
    int c = a - 1;
    while (c >= 0 && out[c] > x) {
      out[c + 1] = out[c];
      --c;
    }
    out[c + 1] = x;
  }
  return n;
}

}  // namespace bb
