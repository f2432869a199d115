// na2d_noalloc.cu -- na2d_forward_host_noalloc: the host-buffer forward for
// callers that cannot allocate device memory.  na2d_forward_host stages the
// host inputs and the output in a device workspace that its caller
// allocates; this entry point stages them in one fixed array that the
// library itself reserves on every device that loads it, so the caller
// allocates nothing.  It adds a path; the existing ones are unchanged.
#include <cuda_runtime.h>

#include "na2d.h"
#include "na2d_internal.h"

#define NA_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

// The staging area.  Every device that loads the library holds these
// NA2D_NOALLOC_SCRATCH_BYTES until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NA2D_NOALLOC_SCRATCH_BYTES];

// In host code g_noalloc_scratch names a host-side stand-in, not device
// memory.  Its device address is looked up with the device current on every
// call: the lookup is a host-side table access in the runtime, and an
// address cached across calls would go stale after a device reset or a new
// primary context in the same process.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace

NA_EXPORT na_status na2d_forward_host_noalloc(const void* q_host, const void* k_host, const void* v_host,
                                              const void* rpb_host, void* out_host, int B, int heads, int H,
                                              int W, int d, int ksize, na_dtype dt, void* stream) {
  // The arguments are checked exactly as na2d_forward_host checks them.  Its
  // workspace size for this shape (0 for rejected arguments) decides whether
  // the fixed array is large enough; everything the call reads from the
  // array it first writes itself, so nothing needs clearing between calls.
  // Rejected arguments and empty batches go straight to na2d_forward_host,
  // which answers them without touching a workspace or the GPU.
  const size_t need = na2d_forward_host_workspace_bytes(B, heads, H, W, d, ksize, dt);
  if (need == 0 || B == 0 || heads == 0)
    return na2d_forward_host(q_host, k_host, v_host, rpb_host, out_host, nullptr, 0, B, heads, H, W, d, ksize,
                             dt, stream);
  if (need > NA2D_NOALLOC_SCRATCH_BYTES) return NA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return NA_ERR_CUDA;
  return na2d::forward_host_serial(q_host, k_host, v_host, rpb_host, out_host, scratch, NA2D_NOALLOC_SCRATCH_BYTES,
                                   B, heads, H, W, d, ksize, dt, stream);
}
