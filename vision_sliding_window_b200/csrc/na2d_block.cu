// na2d_block.cu -- an NA block on the GPU: the query/key/value projection,
// neighborhood attention, and the output projection (NAT App. A.1: linear
// projections for queries, keys and values followed by a final linear
// projection; Qiita "計算量": 4hwd^2 + 2hwdk^2 for the whole block):
//
//   qkv = x Wqkv + bqkv          x [B][H][W][C], Wqkv [C][3C], C = heads * dh
//   q, k, v = the C-channel thirds of qkv, each as heads x dh
//   o = NA_ks(q, k, v, rpb)      per head (na2d_forward)
//   y = o Wo + bo                o as [B][H][W][heads * dh], Wo [C][C]
//
// The two projections are plain GEMMs and run in cuBLAS with float32
// accumulation and float32 output; the kernels here add the biases, round
// to the storage type and move between the pixel-major layout of the
// projections and the head-major layout of the attention.
#include <cublas_v2.h>

#include <mutex>
#include <type_traits>

#include "na2d_common.cuh"
#include "na2d_internal.h"

namespace na2d {
namespace {

constexpr int kThreads = 256;
constexpr size_t kCublasWorkspace = 8u << 20;

NA_DEVICE void store8(float* p, const float (&f)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}
NA_DEVICE void store8(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 w;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&w);
  for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(f[2 * t], f[2 * t + 1]);
  *reinterpret_cast<uint4*>(p) = w;
}
NA_DEVICE void store8(__half* p, const float (&f)[8]) {
  uint4 w;
  __half2* h = reinterpret_cast<__half2*>(&w);
  for (int t = 0; t < 4; ++t) h[t] = __floats2half2_rn(f[2 * t], f[2 * t + 1]);
  *reinterpret_cast<uint4*>(p) = w;
}
template <typename T>
NA_DEVICE void load8(const T* p, float (&f)[8]) {
  for (int t = 0; t < 8; ++t) f[t] = (float)p[t];
}

// qkv (float32, [M][3C]) + bqkv, rounded to T, into q, k, v [B][heads][H][W][dh];
// one thread per 8 channels.
template <typename T>
__global__ void __launch_bounds__(kThreads)
split_qkv_kernel(const float* __restrict__ qkv, const T* __restrict__ bqkv, T* __restrict__ q, T* __restrict__ k,
                 T* __restrict__ v, long long M, int HW, int heads, int dh) {
  const int C = heads * dh, per = 3 * C / 8;
  const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (e >= M * per) return;
  const long long m = e / per;
  const int c8 = (int)(e - m * per) * 8;  // channel in [0, 3C)
  const int s = c8 / C, h = (c8 - s * C) / dh, x = c8 - s * C - h * dh;
  float f[8];
  const float4 a = reinterpret_cast<const float4*>(qkv + m * 3 * C + c8)[0];
  const float4 b = reinterpret_cast<const float4*>(qkv + m * 3 * C + c8)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  if (bqkv) {
    float bb[8];
    load8(bqkv + c8, bb);
    for (int t = 0; t < 8; ++t) f[t] += bb[t];
  }
  const long long bimg = m / HW, pix = m - bimg * HW;
  T* dst = (s == 0 ? q : s == 1 ? k : v) + (((bimg * heads + h) * HW + pix) * dh + x);
  store8(dst, f);
}

// o [B][heads][H][W][dh] -> o2 [M][heads * dh]; one thread per 8 channels.
template <typename T>
__global__ void __launch_bounds__(kThreads)
merge_heads_kernel(const T* __restrict__ o, T* __restrict__ o2, long long M, int HW, int heads, int dh) {
  const int C = heads * dh, per = C / 8;
  const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (e >= M * per) return;
  const long long m = e / per;
  const int c8 = (int)(e - m * per) * 8, h = c8 / dh, x = c8 - h * dh;
  const long long bimg = m / HW, pix = m - bimg * HW;
  *reinterpret_cast<uint4*>(o2 + m * C + c8) =
      *reinterpret_cast<const uint4*>(o + ((bimg * heads + h) * HW + pix) * dh + x);
}
template <>
__global__ void __launch_bounds__(kThreads)
merge_heads_kernel<float>(const float* __restrict__ o, float* __restrict__ o2, long long M, int HW, int heads,
                          int dh) {
  const int C = heads * dh, per = C / 4;
  const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (e >= M * per) return;
  const long long m = e / per;
  const int c4 = (int)(e - m * per) * 4, h = c4 / dh, x = c4 - h * dh;
  const long long bimg = m / HW, pix = m - bimg * HW;
  *reinterpret_cast<float4*>(o2 + m * C + c4) =
      *reinterpret_cast<const float4*>(o + ((bimg * heads + h) * HW + pix) * dh + x);
}

// y = y32 + bo, rounded to T; one thread per 8 values.
template <typename T>
__global__ void __launch_bounds__(kThreads)
bias_round_kernel(const float* __restrict__ y32, const T* __restrict__ bo, T* __restrict__ y, long long n, int C) {
  const long long e = ((long long)blockIdx.x * kThreads + threadIdx.x) * 8;
  if (e >= n) return;
  float f[8];
  const float4 a = reinterpret_cast<const float4*>(y32 + e)[0];
  const float4 b = reinterpret_cast<const float4*>(y32 + e)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  if (bo) {
    float bb[8];
    load8(bo + (int)(e % C), bb);
    for (int t = 0; t < 8; ++t) f[t] += bb[t];
  }
  store8(y + e, f);
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

struct BlockLayout {
  size_t qkv32, q, k, v, o, o2, y32, cublas, total;
};
BlockLayout block_layout(long long M, int C, size_t es) {
  BlockLayout L{};
  size_t off = 0;
  L.qkv32 = off; off = up256(off + (size_t)M * 3 * C * 4);
  L.q = off; off = up256(off + (size_t)M * C * es);
  L.k = off; off = up256(off + (size_t)M * C * es);
  L.v = off; off = up256(off + (size_t)M * C * es);
  L.o = off; off = up256(off + (size_t)M * C * es);
  L.o2 = off; off = up256(off + (size_t)M * C * es);
  L.y32 = off; off = up256(off + (size_t)M * C * 4);
  L.cublas = off; off = up256(off + kCublasWorkspace);
  L.total = off;
  return L;
}

// One cuBLAS handle per device, created by the first block call on it and
// kept; calls are enqueued one at a time (a host mutex), as the handle's
// stream and workspace are set per call.
constexpr int kMaxDevices = 64;
std::mutex g_blas_mu;
cublasHandle_t g_blas[kMaxDevices] = {};

cudaDataType_t blas_type(na_dtype dt) {
  return dt == NA_F32 ? CUDA_R_32F : dt == NA_F16 ? CUDA_R_16F : CUDA_R_16BF;
}

template <typename T>
cudaError_t launch_block_kernels(int stage, const void* a, const void* bias, void* b, void* c, void* d,
                                 long long M, int HW, int heads, int dh, cudaStream_t st) {
  const int C = heads * dh;
  if (stage == 0) {
    const long long n = M * (3 * C / 8);
    split_qkv_kernel<T><<<(unsigned)((n + kThreads - 1) / kThreads), kThreads, 0, st>>>(
        (const float*)a, (const T*)bias, (T*)b, (T*)c, (T*)d, M, HW, heads, dh);
  } else if (stage == 1) {
    const long long n = M * (C / (std::is_same<T, float>::value ? 4 : 8));
    merge_heads_kernel<T><<<(unsigned)((n + kThreads - 1) / kThreads), kThreads, 0, st>>>(
        (const T*)a, (T*)b, M, HW, heads, dh);
  } else {
    const long long n = M * C;
    bias_round_kernel<T><<<(unsigned)((n / 8 + kThreads - 1) / kThreads), kThreads, 0, st>>>(
        (const float*)a, (const T*)bias, (T*)b, n, C);
  }
  return cudaGetLastError();
}

cudaError_t block_kernels(na_dtype dt, int stage, const void* a, const void* bias, void* b, void* c, void* d,
                          long long M, int HW, int heads, int dh, cudaStream_t st) {
  if (dt == NA_F32) return launch_block_kernels<float>(stage, a, bias, b, c, d, M, HW, heads, dh, st);
  if (dt == NA_F16) return launch_block_kernels<__half>(stage, a, bias, b, c, d, M, HW, heads, dh, st);
  return launch_block_kernels<__nv_bfloat16>(stage, a, bias, b, c, d, M, HW, heads, dh, st);
}

}  // namespace

size_t block_workspace_bytes(int B, int H, int W, int heads, int dh, size_t es) {
  return block_layout((long long)B * H * W, heads * dh, es).total;
}

na_status run_block(const void* x, const void* wqkv, const void* bqkv, const void* wo, const void* bo, const void* rpb,
                    void* y, void* workspace, int B, int H, int W, int heads, int dh, int ks, na_dtype dt,
                    cudaStream_t st) {
  const long long M = (long long)B * H * W;
  const int C = heads * dh;
  const size_t es = dt == NA_F32 ? 4 : 2;
  const BlockLayout L = block_layout(M, C, es);
  char* ws = static_cast<char*>(workspace);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_blas_mu);
  if (!g_blas[dev] && cublasCreate(&g_blas[dev]) != CUBLAS_STATUS_SUCCESS) return NA_ERR_CUDA;
  cublasHandle_t h = g_blas[dev];
  if (cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS ||
      cublasSetWorkspace(h, ws + L.cublas, kCublasWorkspace) != CUBLAS_STATUS_SUCCESS)
    return NA_ERR_CUDA;
  const float one = 1.f, zero = 0.f;
  const cudaDataType_t tt = blas_type(dt);
  // qkv32 [M][3C] = x [M][C] Wqkv [C][3C]  (column-major: qkv^T = Wqkv^T x^T)
  if (cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_N, 3 * C, (int)M, C, &one, wqkv, tt, 3 * C, x, tt, C, &zero,
                   ws + L.qkv32, CUDA_R_32F, 3 * C, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
    return NA_ERR_CUDA;
  if (block_kernels(dt, 0, ws + L.qkv32, bqkv, ws + L.q, ws + L.k, ws + L.v, M, H * W, heads, dh, st) !=
      cudaSuccess)
    return NA_ERR_CUDA;
  na_status s = na2d_forward(ws + L.q, ws + L.k, ws + L.v, rpb, ws + L.o, B, heads, H, W, dh, ks, dt, (void*)st);
  if (s != NA_OK) return s;
  if (block_kernels(dt, 1, ws + L.o, nullptr, ws + L.o2, nullptr, nullptr, M, H * W, heads, dh, st) != cudaSuccess)
    return NA_ERR_CUDA;
  // y32 [M][C] = o2 [M][C] Wo [C][C]
  if (cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_N, C, (int)M, C, &one, wo, tt, C, ws + L.o2, tt, C, &zero,
                   ws + L.y32, CUDA_R_32F, C, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
    return NA_ERR_CUDA;
  if (block_kernels(dt, 2, ws + L.y32, bo, y, nullptr, nullptr, M, H * W, heads, dh, st) != cudaSuccess)
    return NA_ERR_CUDA;
  return NA_OK;
}

}  // namespace na2d
