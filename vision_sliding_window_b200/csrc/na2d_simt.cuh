// na2d_simt.cuh -- helpers of the CUDA-core kernels (na2d_simt.cu, na2d_bwd.cu):
// one group of G = d / (elements per 16-byte vector) lanes per query, each
// lane holding one 16-byte slice of the query row; group reductions by
// butterfly shuffles; the dtype / head-size dispatch of the launchers.
#pragma once

#include <cmath>
#include <limits>

#include "na2d_common.cuh"
#include "na2d_internal.h"

namespace na2d {
namespace simt {

constexpr int kThreads = 256;

template <int G, typename A>
NA_DEVICE A group_sum(A x) {
#pragma unroll
  for (int off = G >> 1; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

template <int G, typename A>
NA_DEVICE A group_max(A x) {
#pragma unroll
  for (int off = G >> 1; off > 0; off >>= 1) {
    A y = __shfl_xor_sync(0xffffffffu, x, off);
    x = y > x ? y : x;
  }
  return x;
}

struct QueryPos {
  long long bh;  // b * heads + h
  int h, i, j;
};

NA_DEVICE QueryPos decode(long long qidx, int heads, int H, int W) {
  QueryPos p;
  p.j = (int)(qidx % W);
  long long t = qidx / W;
  p.i = (int)(t % H);
  p.bh = t / H;
  p.h = (int)(p.bh % heads);
  return p;
}

// Logit of Eq. (2) for window entry (a, c) of the query held by this group.
template <typename T, int D>
NA_DEVICE typename Elem<T>::Acc group_logit(const typename Elem<T>::Acc (&qv)[Elem<T>::kVec],
                                            const T* kmap, const T* tab, int W, int ks, int span,
                                            int i, int j, int r, int t, int lane) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  constexpr int G = D / E::kVec;
  Acc kv[E::kVec];
  E::load(kmap + ((long long)r * W + t) * D + lane * E::kVec, kv);
  Acc part = 0;
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) part = fma(qv[x], kv[x], part);
  Acc s = group_sum<G>(part);
  if (tab) s += E::scalar(tab + (r - i + ks - 1) * span + (t - j + ks - 1));
  return s;
}

template <typename T, int D>
unsigned grid_for(long long nq) {
  constexpr int G = D / Elem<T>::kVec;
  return (unsigned)((nq * G + kThreads - 1) / kThreads);
}

// Calls f.template operator()<T, D>() for the runtime (dtype, d).
template <typename F>
cudaError_t dispatch(na_dtype dt, int d, F&& f) {
#define NA_D(T)                                  \
  switch (d) {                                   \
    case 16: return f.template operator()<T, 16>();  \
    case 32: return f.template operator()<T, 32>();  \
    case 64: return f.template operator()<T, 64>();  \
    case 128: return f.template operator()<T, 128>(); \
    default: return cudaErrorInvalidValue;       \
  }
  switch (dt) {
    case NA_F32: NA_D(float)
    case NA_F16: NA_D(__half)
    case NA_BF16: NA_D(__nv_bfloat16)
  }
#undef NA_D
  return cudaErrorInvalidValue;
}

}  // namespace simt
}  // namespace na2d
