// na2d_unfused.cu -- bandwidth kernels for the unfused calls: "QK+B" and
// "AV" of NATTEN (Qiita write-up, section "NATTEN"; NAT Sec. 3.2) for 16-bit
// inputs, and the softmax between them.
//
// QK+B and AV work on a tile of 8 x 32 queries per CTA, one query per
// thread.  The tile's key (or value) halo -- the rows and columns every
// window of the tile covers -- is staged in shared memory by one TMA box,
// so each key is read from HBM/L2 once per tile instead of once per query
// that sees it (NAT Sec. 3.2 and App. A.4: the tiled NA kernel).  Logits
// accumulate in float32 with mixed-precision FMAs of the 16-bit operands;
// the weighted sum accumulates in float32.  Each thread reads its row's
// 16-byte key chunks in a staggered order, so the 32 lanes of a warp spread
// over the shared-memory banks.
//
// The softmax runs one warp per row of ks^2 weights, in float32 with the
// row maximum subtracted.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "na2d_common.cuh"
#include "na2d_internal.h"
#include "na2d_sm100.cuh"

namespace na2d {
namespace {

using namespace sm100;

constexpr int TR = 8, TCOL = 32, kTileThreads = TR * TCOL;

// dot += x . y over one 16-byte chunk (8 elements of T), float32 accumulation
template <typename T> NA_DEVICE void dot8(float& acc, const uint4& x, const uint4& y);
template <> NA_DEVICE void dot8<__nv_bfloat16>(float& acc, const uint4& x, const uint4& y) {
  const uint32_t a[4] = {x.x, x.y, x.z, x.w}, b[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int t = 0; t < 4; ++t)
    asm("{\n .reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %1;\n mov.b32 {bl, bh}, %2;\n"
        " fma.rn.f32.bf16 %0, al, bl, %0;\n fma.rn.f32.bf16 %0, ah, bh, %0;\n}"
        : "+f"(acc) : "r"(a[t]), "r"(b[t]));
}
template <> NA_DEVICE void dot8<__half>(float& acc, const uint4& x, const uint4& y) {
  const uint32_t a[4] = {x.x, x.y, x.z, x.w}, b[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int t = 0; t < 4; ++t)
    asm("{\n .reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %1;\n mov.b32 {bl, bh}, %2;\n"
        " fma.rn.f32.f16 %0, al, bl, %0;\n fma.rn.f32.f16 %0, ah, bh, %0;\n}"
        : "+f"(acc) : "r"(a[t]), "r"(b[t]));
}

// o[0..8) += w * x (8 elements of T)
template <typename T>
NA_DEVICE void axpy8(float* o, float w, const uint4& x) {
  const uint32_t a[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    float lo, hi;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[t]));
      lo = f.x;
      hi = f.y;
    } else {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&a[t]));
      lo = f.x;
      hi = f.y;
    }
    fma2(o[2 * t], o[2 * t + 1], w, w, lo, hi, o[2 * t], o[2 * t + 1]);
  }
}

// The tile of work unit `tile` (tile columns fastest, then tile rows, then
// maps) and its halo origin: the window start of its first row and column,
// so the halo box covers every window of the tile.
struct Tile {
  long long map;  // b * heads + h
  int h, i0, j0, R0, C0;
};
NA_DEVICE Tile tile_of(int tile, int heads, int H, int W, int ks, int n_tr, int n_tc) {
  Tile t;
  const int tc = tile % n_tc, rest = tile / n_tc, tr = rest % n_tr;
  t.map = rest / n_tr;
  t.h = (int)(t.map % heads);
  t.i0 = tr * TR;
  t.j0 = tc * TCOL;
  t.R0 = window_start(t.i0, H, ks);
  t.C0 = window_start(t.j0, W, ks);
  return t;
}

// Stages the halo box (d, TCOL + ks - 1, TR + ks - 1) at (C0, R0) of map
// (b, h) into shared memory; every thread returns once it has landed (or
// the bounded wait ran out, which the status word records).
NA_DEVICE bool stage_halo(const CUtensorMap* tm, uint8_t* halo, uint64_t* bar, const Tile& t, int heads,
                          uint32_t bytes, unsigned* status, volatile int* abort_flag) {
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(bar), 1);
    mbar_init_fence();
    *abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_expect_tx(smem_addr(bar), bytes);
    tma_load_5d(smem_addr(halo), tm, smem_addr(bar), 0, t.C0, t.R0, t.h, (int)(t.map / heads));
  }
  return mbar_wait(smem_addr(bar), 0, abort_flag, status);
}

template <typename T, int D>
__global__ void __launch_bounds__(kTileThreads)
qk_rpb_tile_kernel(const __grid_constant__ CUtensorMap tm_k, const T* __restrict__ q, const T* __restrict__ rpb,
                   float* __restrict__ attn, int heads, int H, int W, int ks, int n_tr, int n_tc, unsigned* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int VEC = D / 8;  // 16-byte chunks per row
  const int HC = TCOL + ks - 1, HR = TR + ks - 1, span = 2 * ks - 1;
  uint8_t* halo = smem;
  float* tab = reinterpret_cast<float*>(smem + (size_t)HR * HC * D * 2);
  uint64_t* bar = reinterpret_cast<uint64_t*>(tab + round_up_int(span * span, 4));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 1);
  const Tile t = tile_of(blockIdx.x, heads, H, W, ks, n_tr, n_tc);
  for (int e = threadIdx.x; e < span * span; e += kTileThreads)
    tab[e] = rpb ? (float)rpb[(size_t)t.h * span * span + e] : 0.f;
  if (!stage_halo(&tm_k, halo, bar, t, heads, (uint32_t)(HR * HC * D * 2), status, abort_flag)) return;
  const int i = t.i0 + threadIdx.x / TCOL, j = t.j0 + threadIdx.x % TCOL;
  if (i >= H || j >= W) return;
  const int si = window_start(i, H, ks), sj = window_start(j, W, ks);
  const long long qidx = (t.map * H + i) * (long long)W + j;
  uint4 qv[VEC];
#pragma unroll
  for (int x = 0; x < VEC; ++x) qv[x] = reinterpret_cast<const uint4*>(q + qidx * D)[x];
  float* row = attn + qidx * (long long)(ks * ks);
  const int lane = threadIdx.x & 31;
  for (int a = 0; a < ks; ++a) {
    const uint4* krow = reinterpret_cast<const uint4*>(halo) + (size_t)((si + a - t.R0) * HC + (sj - t.C0)) * VEC;
    const float* brow = tab + (si + a - i + ks - 1) * span + (sj - j + ks - 1);
#pragma unroll 1
    for (int c = 0; c < ks; ++c) {
      float acc = 0.f;
#pragma unroll
      for (int x0 = 0; x0 < VEC; ++x0) {
        const int x = (x0 + lane) % VEC;  // staggered chunk order across the warp
        dot8<T>(acc, qv[x], krow[c * VEC + x]);
      }
      row[a * ks + c] = acc + brow[c];
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kTileThreads)
av_tile_kernel(const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ attn, T* __restrict__ out,
               int heads, int H, int W, int ks, int n_tr, int n_tc, unsigned* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int VEC = D / 8;
  const int HC = TCOL + ks - 1, HR = TR + ks - 1;
  uint8_t* halo = smem;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (size_t)HR * HC * D * 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 1);
  const Tile t = tile_of(blockIdx.x, heads, H, W, ks, n_tr, n_tc);
  if (!stage_halo(&tm_v, halo, bar, t, heads, (uint32_t)(HR * HC * D * 2), status, abort_flag)) return;
  const int i = t.i0 + threadIdx.x / TCOL, j = t.j0 + threadIdx.x % TCOL;
  if (i >= H || j >= W) return;
  const int si = window_start(i, H, ks), sj = window_start(j, W, ks);
  const long long qidx = (t.map * H + i) * (long long)W + j;
  const float* row = attn + qidx * (long long)(ks * ks);
  float o[D];
#pragma unroll
  for (int x = 0; x < D; ++x) o[x] = 0.f;
  const int lane = threadIdx.x & 31;
  for (int a = 0; a < ks; ++a) {
    const uint4* vrow = reinterpret_cast<const uint4*>(halo) + (size_t)((si + a - t.R0) * HC + (sj - t.C0)) * VEC;
#pragma unroll 1
    for (int c = 0; c < ks; ++c) {
      const float w = __ldg(row + a * ks + c);
#pragma unroll
      for (int x0 = 0; x0 < VEC; ++x0) {
        const int x = (x0 + lane) % VEC;
        axpy8<T>(o + 8 * x, w, vrow[c * VEC + x]);
      }
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(out + qidx * D);
#pragma unroll
  for (int x = 0; x < VEC; ++x) {
    uint4 w;
    uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(o[8 * x + 2 * e], o[8 * x + 2 * e + 1]);
        u[e] = *reinterpret_cast<const uint32_t*>(&b);
      } else {
        const __half2 b = __floats2half2_rn(o[8 * x + 2 * e], o[8 * x + 2 * e + 1]);
        u[e] = *reinterpret_cast<const uint32_t*>(&b);
      }
    }
    dst[x] = w;
  }
}

// Softmax of Eq. (4) in place: one warp per row of kk weights, float32, the
// row maximum subtracted.
__global__ void __launch_bounds__(256)
softmax_warp_kernel(float* __restrict__ attn, long long rows, int kk, float scale) {
  const long long r = ((long long)blockIdx.x * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;  // whole warps leave together
  float* row = attn + r * kk;
  float v[6];  // kk <= 169 = 6 * 32 - 23 for ks <= 13; longer rows take the loop below
  float m = -INFINITY;
  if (kk <= 192) {
#pragma unroll
    for (int t = 0; t < 6; ++t) {
      const int n = lane + 32 * t;
      v[t] = n < kk ? row[n] * scale : -INFINITY;
      m = fmaxf(m, v[t]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
#pragma unroll
    for (int t = 0; t < 6; ++t) {
      v[t] = lane + 32 * t < kk ? expf(v[t] - m) : 0.f;
      l += v[t];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    const float inv = 1.f / l;
#pragma unroll
    for (int t = 0; t < 6; ++t)
      if (lane + 32 * t < kk) row[lane + 32 * t] = v[t] * inv;
    return;
  }
  for (int n = lane; n < kk; n += 32) m = fmaxf(m, row[n] * scale);
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float l = 0.f;
  for (int n = lane; n < kk; n += 32) l += expf(row[n] * scale - m);
  for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  const float inv = 1.f / l;
  for (int n = lane; n < kk; n += 32) row[n] = expf(row[n] * scale - m) * inv;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult r;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// [B][heads][H][W][d] with a box of (d, TCOL + ks - 1, TR + ks - 1, 1, 1),
// no swizzle (rows of d elements, contiguous).
bool halo_map(CUtensorMap* m, const void* base, const Shape& s, bool bf16) {
  auto enc = encoder();
  if (!enc) return false;
  const cuuint64_t es = 2;
  cuuint64_t dims[5] = {(cuuint64_t)s.d, (cuuint64_t)s.W, (cuuint64_t)s.H, (cuuint64_t)s.heads, (cuuint64_t)s.B};
  cuuint64_t strides[4] = {s.d * es, (cuuint64_t)s.W * s.d * es, (cuuint64_t)s.H * s.W * s.d * es,
                           (cuuint64_t)s.heads * s.H * s.W * s.d * es};
  cuuint32_t box[5] = {(cuuint32_t)s.d, (cuuint32_t)(TCOL + s.ks - 1), (cuuint32_t)(TR + s.ks - 1), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, const_cast<void*>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Kern>
cudaError_t set_smem(Kern kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T, int D>
cudaError_t qk_tile(const void* q, const void* k, const void* rpb, float* attn, const Shape& s, unsigned* status,
                    cudaStream_t st) {
  CUtensorMap tm;
  if (!halo_map(&tm, k, s, std::is_same<T, __nv_bfloat16>::value)) return cudaErrorInvalidValue;
  const int n_tr = (s.H + TR - 1) / TR, n_tc = (s.W + TCOL - 1) / TCOL, span = 2 * s.ks - 1;
  const size_t smem = (size_t)(TR + s.ks - 1) * (TCOL + s.ks - 1) * D * 2 + round_up_int(span * span, 4) * 4 + 16;
  auto kern = qk_rpb_tile_kernel<T, D>;
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)s.B * s.heads * n_tr * n_tc;
  kern<<<(unsigned)tiles, kTileThreads, smem, st>>>(tm, (const T*)q, (const T*)rpb, attn, s.heads, s.H, s.W, s.ks,
                                                   n_tr, n_tc, status);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t av_tile(const float* attn, const void* v, void* out, const Shape& s, unsigned* status, cudaStream_t st) {
  CUtensorMap tm;
  if (!halo_map(&tm, v, s, std::is_same<T, __nv_bfloat16>::value)) return cudaErrorInvalidValue;
  const int n_tr = (s.H + TR - 1) / TR, n_tc = (s.W + TCOL - 1) / TCOL;
  const size_t smem = (size_t)(TR + s.ks - 1) * (TCOL + s.ks - 1) * D * 2 + 16;
  auto kern = av_tile_kernel<T, D>;
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)s.B * s.heads * n_tr * n_tc;
  kern<<<(unsigned)tiles, kTileThreads, smem, st>>>(tm, attn, (T*)out, s.heads, s.H, s.W, s.ks, n_tr, n_tc, status);
  return cudaGetLastError();
}

}  // namespace

bool unfused_tile_supported(const Shape& s, na_dtype dt) {
  if (dt != NA_F16 && dt != NA_BF16) return false;
  if (s.d != 16 && s.d != 32 && s.d != 64) return false;
  if (s.ks > 13) return false;
  const long long tiles = (long long)s.B * s.heads * ((s.H + TR - 1) / TR) * ((s.W + TCOL - 1) / TCOL);
  return tiles < (1ll << 31);
}

cudaError_t launch_qk_rpb_tile(const void* q, const void* k, const void* rpb, float* attn, const Shape& s,
                               na_dtype dt, unsigned* status, cudaStream_t st) {
  const bool bf = dt == NA_BF16;
  switch (s.d) {
    case 16: return bf ? qk_tile<__nv_bfloat16, 16>(q, k, rpb, attn, s, status, st) : qk_tile<__half, 16>(q, k, rpb, attn, s, status, st);
    case 32: return bf ? qk_tile<__nv_bfloat16, 32>(q, k, rpb, attn, s, status, st) : qk_tile<__half, 32>(q, k, rpb, attn, s, status, st);
    case 64: return bf ? qk_tile<__nv_bfloat16, 64>(q, k, rpb, attn, s, status, st) : qk_tile<__half, 64>(q, k, rpb, attn, s, status, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_av_tile(const float* attn, const void* v, void* out, const Shape& s, na_dtype dt, unsigned* status,
                           cudaStream_t st) {
  const bool bf = dt == NA_BF16;
  switch (s.d) {
    case 16: return bf ? av_tile<__nv_bfloat16, 16>(attn, v, out, s, status, st) : av_tile<__half, 16>(attn, v, out, s, status, st);
    case 32: return bf ? av_tile<__nv_bfloat16, 32>(attn, v, out, s, status, st) : av_tile<__half, 32>(attn, v, out, s, status, st);
    case 64: return bf ? av_tile<__nv_bfloat16, 64>(attn, v, out, s, status, st) : av_tile<__half, 64>(attn, v, out, s, status, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_softmax_warp(float* attn, long long rows, int ks, float scale, cudaStream_t st) {
  const long long blocks = (rows * 32 + 255) / 256;
  softmax_warp_kernel<<<(unsigned)blocks, 256, 0, st>>>(attn, rows, ks * ks, scale);
  return cudaGetLastError();
}

}  // namespace na2d
