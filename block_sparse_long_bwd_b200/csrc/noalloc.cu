// Forward entry point for callers that cannot allocate device memory.
//
// Some hosts of this library own every byte of device memory up front: an
// engine that reserves its whole memory budget at start-up and forbids any
// later cudaMalloc, a plugin inside a framework whose caching allocator must
// not be bypassed, or a C caller with no allocator of its own and no spare
// buffer to hand over as a workspace.  For them, bb_attn_fwd_noalloc runs the
// same forward kernels as bb_attn_fwd, with the workspace replaced by a
// scratch array built into the library (below).  Nothing here allocates.
#include <mutex>

#include "common.cuh"

namespace {

// Built-in scratch: the forward's status word and the split partials of the
// two global query rows.  Fixed at 32 MiB; zero-filled when the module is
// loaded on a device and kept by every device that loads the library until
// the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch, looked up once per device.  In host code
// the array's name is only a host-side stand-in, never a device address.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];

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
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return BB_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
        return BB_ERR_CUDA;
      g_scratch_ptr[dev] = ptr;
    }
    scratch = g_scratch_ptr[dev];
  }
  // The status word at the start of the scratch is cleared by the forward
  // itself; the partials are written before they are read.
  return bb_attn_fwd(desc, q, k, v, key_mask, rand_idx, out, lse, scratch,
                     kNoAllocScratchBytes, stream);
}
