// na2d_simt.cu -- CUDA-core kernels for 2D Neighborhood Attention.
//
// One group of G = d / (elements per 16-byte vector) lanes works on one
// query: each lane holds one 16-byte slice of the query / output row, so a
// group reads every key and value row with coalesced 16-byte loads, and the
// dot product is finished with a butterfly of G-lane shuffles.
//
// These kernels serve the float32 path (float64 accumulation, so the result
// is float32 rounding of the exact value) and every call of the unfused
// chain; for 16-bit inputs they accumulate in float32.
//
// Eq. numbers: Neighborhood Attention Transformer, Sec. 3.1.
#include <cmath>
#include <limits>

#include "na2d_simt.cuh"

namespace na2d {
namespace {

using namespace simt;

// Fused Eqs. (2)-(4): two passes over the window (maximum, then weights and
// weighted sum) so the softmax subtracts the exact maximum.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
forward_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                    const T* __restrict__ rpb, T* __restrict__ out,
                    long long nq, int heads, int H, int W, int ks) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  constexpr int G = D / E::kVec;
  long long g = ((long long)blockIdx.x * kThreads + threadIdx.x) / G;
  const int lane = threadIdx.x % G;
  const bool live = g < nq;
  const long long qidx = live ? g : nq - 1;  // dead groups shadow a live query, store nothing
  const QueryPos p = decode(qidx, heads, H, W);
  const int span = 2 * ks - 1;
  const long long map_off = p.bh * H * W * (long long)D;
  const T* kmap = k + map_off;
  const T* vmap = v + map_off;
  const T* tab = rpb ? rpb + (long long)p.h * span * span : nullptr;
  Acc qv[E::kVec];
  E::load(q + qidx * D + lane * E::kVec, qv);
  const int si = window_start(p.i, H, ks), sj = window_start(p.j, W, ks);

  Acc m = -std::numeric_limits<Acc>::infinity();
  for (int a = 0; a < ks; ++a)
    for (int c = 0; c < ks; ++c) {
      Acc s = group_logit<T, D>(qv, kmap, tab, W, ks, span, p.i, p.j, si + a, sj + c, lane);
      m = s > m ? s : m;
    }

  const Acc scale = (Acc)1 / sqrt((Acc)D);
  Acc l = 0, o[E::kVec];
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) o[x] = 0;
  for (int a = 0; a < ks; ++a)
    for (int c = 0; c < ks; ++c) {
      const int r = si + a, t = sj + c;
      Acc s = group_logit<T, D>(qv, kmap, tab, W, ks, span, p.i, p.j, r, t, lane);
      Acc w = acc_exp((s - m) * scale);
      l += w;
      Acc vv[E::kVec];
      E::load(vmap + ((long long)r * W + t) * D + lane * E::kVec, vv);
#pragma unroll
      for (int x = 0; x < E::kVec; ++x) o[x] = fma(w, vv[x], o[x]);
    }
  if (!live) return;
  const Acc inv = (Acc)1 / l;
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) o[x] *= inv;
  E::store(out + qidx * D + lane * E::kVec, o);
}

// Eq. (2) alone: unscaled logits, float32.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
qk_rpb_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ rpb,
                   float* __restrict__ attn, long long nq, int heads, int H, int W, int ks) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  constexpr int G = D / E::kVec;
  long long g = ((long long)blockIdx.x * kThreads + threadIdx.x) / G;
  const int lane = threadIdx.x % G;
  const bool live = g < nq;
  const long long qidx = live ? g : nq - 1;
  const QueryPos p = decode(qidx, heads, H, W);
  const int span = 2 * ks - 1;
  const T* kmap = k + p.bh * H * W * (long long)D;
  const T* tab = rpb ? rpb + (long long)p.h * span * span : nullptr;
  Acc qv[E::kVec];
  E::load(q + qidx * D + lane * E::kVec, qv);
  const int si = window_start(p.i, H, ks), sj = window_start(p.j, W, ks);
  float* row = attn + qidx * (long long)(ks * ks);
  for (int a = 0; a < ks; ++a)
    for (int c = 0; c < ks; ++c) {
      Acc s = group_logit<T, D>(qv, kmap, tab, W, ks, span, p.i, p.j, si + a, sj + c, lane);
      const int n = a * ks + c;
      if (live && (n % G) == lane) row[n] = (float)s;
    }
}

// Softmax of Eq. (4) in place on rows of ks*ks float32 entries, computed in
// float64; 8 lanes per row.
constexpr int kSoftmaxLanes = 8;
__global__ void __launch_bounds__(kThreads)
softmax_simt_kernel(float* __restrict__ attn, long long rows, int kk, float scale) {
  constexpr int G = kSoftmaxLanes;
  long long g = ((long long)blockIdx.x * kThreads + threadIdx.x) / G;
  const int lane = threadIdx.x % G;
  const bool live = g < rows;
  float* row = attn + (live ? g : rows - 1) * (long long)kk;
  const double sc = (double)scale;
  double m = -std::numeric_limits<double>::infinity();
  for (int n = lane; n < kk; n += G) {
    double x = sc * (double)row[n];
    m = x > m ? x : m;
  }
  m = group_max<G>(m);
  double l = 0;
  for (int n = lane; n < kk; n += G) l += exp(sc * (double)row[n] - m);
  l = group_sum<G>(l);
  const double inv = 1.0 / l;
  if (!live) return;
  for (int n = lane; n < kk; n += G) row[n] = (float)(exp(sc * (double)row[n] - m) * inv);
}

// Eqs. (3)-(4) with given weights.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
av_simt_kernel(const float* __restrict__ attn, const T* __restrict__ v, T* __restrict__ out,
               long long nq, int heads, int H, int W, int ks) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  constexpr int G = D / E::kVec;
  long long g = ((long long)blockIdx.x * kThreads + threadIdx.x) / G;
  const int lane = threadIdx.x % G;
  if (g >= nq) return;  // no shuffles below
  const QueryPos p = decode(g, heads, H, W);
  const T* vmap = v + p.bh * H * W * (long long)D;
  const float* row = attn + g * (long long)(ks * ks);
  const int si = window_start(p.i, H, ks), sj = window_start(p.j, W, ks);
  Acc o[E::kVec];
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) o[x] = 0;
  for (int a = 0; a < ks; ++a)
    for (int c = 0; c < ks; ++c) {
      const Acc w = (Acc)__ldg(row + a * ks + c);
      Acc vv[E::kVec];
      E::load(vmap + ((long long)(si + a) * W + (sj + c)) * D + lane * E::kVec, vv);
#pragma unroll
      for (int x = 0; x < E::kVec; ++x) o[x] = fma(w, vv[x], o[x]);
    }
  E::store(out + g * D + lane * E::kVec, o);
}

}  // namespace

cudaError_t launch_forward_simt(const void* q, const void* k, const void* v, const void* rpb,
                                void* out, const Shape& s, na_dtype dt, cudaStream_t st) {
  const long long nq = s.queries();
  return dispatch(dt, s.d, [&]<typename T, int D>() {
    forward_simt_kernel<T, D><<<grid_for<T, D>(nq), kThreads, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)v, (const T*)rpb, (T*)out, nq, s.heads, s.H, s.W, s.ks);
    return cudaGetLastError();
  });
}

cudaError_t launch_qk_rpb_simt(const void* q, const void* k, const void* rpb, float* attn,
                               const Shape& s, na_dtype dt, cudaStream_t st) {
  const long long nq = s.queries();
  return dispatch(dt, s.d, [&]<typename T, int D>() {
    qk_rpb_simt_kernel<T, D><<<grid_for<T, D>(nq), kThreads, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)rpb, attn, nq, s.heads, s.H, s.W, s.ks);
    return cudaGetLastError();
  });
}

cudaError_t launch_softmax_simt(float* attn, long long rows, int ks, float scale, cudaStream_t st) {
  const unsigned grid = (unsigned)((rows * kSoftmaxLanes + kThreads - 1) / kThreads);
  softmax_simt_kernel<<<grid, kThreads, 0, st>>>(attn, rows, ks * ks, scale);
  return cudaGetLastError();
}

cudaError_t launch_av_simt(const float* attn, const void* v, void* out, const Shape& s,
                           na_dtype dt, cudaStream_t st) {
  const long long nq = s.queries();
  return dispatch(dt, s.d, [&]<typename T, int D>() {
    av_simt_kernel<T, D><<<grid_for<T, D>(nq), kThreads, 0, st>>>(
        attn, (const T*)v, (T*)out, nq, s.heads, s.H, s.W, s.ks);
    return cudaGetLastError();
  });
}

}  // namespace na2d
