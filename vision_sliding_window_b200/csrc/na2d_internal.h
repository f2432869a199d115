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

// Backward (na2d_bwd.cu): every dtype and head size; the workspace holds
// two float64 per query.
size_t backward_workspace_bytes(const Shape& s);
cudaError_t launch_backward_simt(const void* q, const void* k, const void* v, const void* rpb, const void* dout,
                                 void* dq, void* dk, void* dv, float* drpb, void* workspace, const Shape& s,
                                 na_dtype dt, cudaStream_t st);

// na2d_forward_host with every copy and the kernel in order on the
// caller's stream (na2d_api.cu); used by na2d_forward_host_noalloc.
na_status forward_host_serial(const void* q_host, const void* k_host, const void* v_host, const void* rpb_host,
                              void* out_host, void* workspace, size_t workspace_bytes, int B, int heads, int H,
                              int W, int d, int ksize, na_dtype dt, void* stream);

// SASA (na2d_sasa.cu): the zero-padded copies of q, k, v and the padded
// output live in the caller's workspace (four 256-byte aligned parts).
size_t sasa_workspace_bytes(const Shape& s, size_t es);
cudaError_t launch_sasa_pad(const void* q, const void* k, const void* v, void* workspace, const Shape& s, size_t es,
                            cudaStream_t st, void** qp, void** kp, void** vp, void** outp);
cudaError_t launch_sasa_crop(const void* outp, void* out, const Shape& s, size_t es, cudaStream_t st);

// NA block (na2d_block.cu): projections in cuBLAS around na2d_forward.
size_t block_workspace_bytes(int B, int H, int W, int heads, int dh, size_t es);
na_status run_block(const void* x, const void* wqkv, const void* bqkv, const void* wo, const void* bo, const void* rpb,
                    void* y, void* workspace, int B, int H, int W, int heads, int dh, int ks, na_dtype dt,
                    cudaStream_t st);

// NA over 1-3 axes with dilation (na2d_nd.cu).
cudaError_t launch_forward_nd(const void* q, const void* k, const void* v, const void* rpb, void* out, int B,
                              int heads, const int (&L)[3], int d, const int (&ks)[3], const int (&dil)[3],
                              na_dtype dt, cudaStream_t st);

// Tensor-core fused forward (na2d_tc.cu), fp16/bf16.
bool forward_tc_supported(const Shape& s, na_dtype dt);
cudaError_t launch_forward_tc(const void* q, const void* k, const void* v, const void* rpb,
                              void* out, const Shape& s, na_dtype dt, unsigned* status,
                              cudaStream_t st);

}  // namespace na2d
