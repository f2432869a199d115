// na2d_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) fused forward for
// fp16 / bf16.  Placeholder until the kernel lands: nothing is supported,
// so na2d_forward uses the SIMT kernel.
#include "na2d_common.cuh"
#include "na2d_internal.h"

namespace na2d {

bool forward_tc_supported(const Shape&, na_dtype) { return false; }

cudaError_t launch_forward_tc(const void*, const void*, const void*, const void*, void*,
                              const Shape&, na_dtype, unsigned*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace na2d
