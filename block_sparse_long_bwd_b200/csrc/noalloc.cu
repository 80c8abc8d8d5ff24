// Forward entry point for callers that cannot allocate device memory.
//
// Some hosts of this library own every byte of device memory up front: an
// engine that reserves its whole memory budget at start-up and forbids any
// later cudaMalloc, a plugin inside a framework whose caching allocator must
// not be bypassed, or a C caller with no allocator of its own and no spare
// buffer to hand over as a workspace.  For them, bb_attn_fwd_noalloc runs the
// same forward kernels as bb_attn_fwd, with the workspace replaced by a
// scratch array built into the library (below).  Nothing here allocates.
#include "common.cuh"

namespace {

// Built-in scratch: the forward's status word, its work counters, the split
// partials of the two global query rows and the planned tile lists.  Fixed at
// 32 MiB; zero-filled when the module is loaded on a device and kept by every
// device that loads the library until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch in the CUDA context current on the calling
// thread.  In host code the array's name is only a host-side stand-in, never
// a device address, so it is looked up on every call: the lookup allocates
// nothing and is cheap, and an address cached per device could belong to
// another context (a caller's own driver-API context on the same device, or
// the context before a cudaDeviceReset).
int scratch_address(void** ptr) {
  *ptr = nullptr;
  if (cudaGetSymbolAddress(ptr, g_noalloc_scratch) != cudaSuccess || !*ptr) {
    cudaGetLastError();  // leave no sticky error behind for the caller
    return BB_ERR_CUDA;
  }
  return BB_OK;
}

}  // namespace

extern "C" int bb_attn_fwd_noalloc(const bb_attn_desc* desc, const void* q,
                                   const void* k, const void* v,
                                   const uint8_t* key_mask,
                                   const int32_t* rand_idx, void* out,
                                   float* lse, void* stream) {
  size_t need = 0;
  const int st = bb_attn_workspace_size(desc, 0, &need);
  if (st != BB_OK) return st;
  if (need > kNoAllocScratchBytes) return BB_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int sa = scratch_address(&scratch);
  if (sa != BB_OK) return sa;
  // The forward clears the status word at the start of the scratch on
  // `stream` before its first kernel, the plan kernel zeroes the work
  // counters, and every partial and tile list is written before it is read:
  // nothing depends on what an earlier call left in the array.
  return bb_attn_fwd(desc, q, k, v, key_mask, rand_idx, out, lse, scratch,
                     kNoAllocScratchBytes, stream);
}

extern "C" int bb_attn_noalloc_status(void* stream) {
  void* scratch = nullptr;
  const int sa = scratch_address(&scratch);
  if (sa != BB_OK) return sa;
  return bb_attn_check_status(scratch, stream);
}
