// na2d_internal.h -- launchers shared between the C-ABI front end
// (na2d_api.cu) and the kernel translation units.  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>

#include "na2d.h"

namespace na2d {

struct Shape {
  int B, heads, H, W, d, ks;
  long long queries() const { return (long long)B * heads * H * W; }
};

// SIMT kernels (na2d_simt.cu): every dtype, every supported shape.
cudaError_t launch_forward_simt(const void* q, const void* k, const void* v, const void* rpb,
                                void* out, const Shape& s, na_dtype dt, cudaStream_t st);
cudaError_t launch_qk_rpb_simt(const void* q, const void* k, const void* rpb, float* attn,
                               const Shape& s, na_dtype dt, cudaStream_t st);
cudaError_t launch_softmax_simt(float* attn, long long rows, int ks, float scale, cudaStream_t st);
cudaError_t launch_av_simt(const float* attn, const void* v, void* out, const Shape& s,
                           na_dtype dt, cudaStream_t st);

// Tensor-core fused forward (na2d_tc.cu), fp16/bf16.
bool forward_tc_supported(const Shape& s, na_dtype dt);
cudaError_t launch_forward_tc(const void* q, const void* k, const void* v, const void* rpb,
                              void* out, const Shape& s, na_dtype dt, unsigned* status,
                              cudaStream_t st);

}  // namespace na2d
