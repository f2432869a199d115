// na2d_nd.cu -- neighborhood attention over 1, 2 or 3 axes with dilation:
// NATTEN's NA "from 1D to 3D" (Qiita write-up, section "NATTEN"; NAT Sec. 3.2)
// and the dilated NA of DiNAT.  The pages give no formula for dilation; the
// reading is that a dilation dl splits an axis into dl interleaved
// sub-grids (positions congruent mod dl) and a query attends within its own
// with NA's clamped window of k positions, the bias indexed by the
// displacement on the sub-grid.  1D and 2D are the cases with unit extents
// and kernel sizes on the leading axes.
//
// One group of lanes per query (each lane one 16-byte slice of the row),
// two passes over the window (maximum, then weights and weighted sum) so the
// softmax subtracts the exact maximum; float64 accumulation for float32
// inputs.
#include "na2d_simt.cuh"

namespace na2d {
namespace {

using namespace simt;

struct NdShape {
  int L[3], k[3], dl[3];
};

// Start of the window on an axis, in sub-grid units, and the query's
// residue and sub-grid index.
NA_DEVICE int nd_axis_start(int i, int L, int ka, int dl, int& r, int& ip) {
  r = i % dl;
  ip = i / dl;
  const int Lp = (L - r + dl - 1) / dl;
  int s = ip - ka / 2;
  s = s < 0 ? 0 : s;
  return s > Lp - ka ? Lp - ka : s;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
nd_forward_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ rpb,
                  T* __restrict__ out, long long nq, int heads, NdShape s) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  constexpr int G = D / E::kVec;
  const long long g = ((long long)blockIdx.x * kThreads + threadIdx.x) / G;
  const int lane = threadIdx.x % G;
  const bool live = g < nq;
  const long long qidx = live ? g : nq - 1;  // dead groups shadow a live query, store nothing
  const int i2 = (int)(qidx % s.L[2]);
  long long t = qidx / s.L[2];
  const int i1 = (int)(t % s.L[1]);
  t /= s.L[1];
  const int i0 = (int)(t % s.L[0]);
  const long long bh = t / s.L[0];
  const int h = (int)(bh % heads);
  const long long map = bh * s.L[0] * s.L[1] * (long long)s.L[2];
  int r0, r1, r2, p0, p1, p2;
  const int st0 = nd_axis_start(i0, s.L[0], s.k[0], s.dl[0], r0, p0);
  const int st1 = nd_axis_start(i1, s.L[1], s.k[1], s.dl[1], r1, p1);
  const int st2 = nd_axis_start(i2, s.L[2], s.k[2], s.dl[2], r2, p2);
  const int b0 = 2 * s.k[0] - 1, b1 = 2 * s.k[1] - 1, b2 = 2 * s.k[2] - 1;
  const T* tab = rpb ? rpb + (long long)h * b0 * b1 * b2 : nullptr;
  Acc qv[E::kVec];
  E::load(q + qidx * D + lane * E::kVec, qv);
  auto key_of = [&](int a, int b, int c) {
    return map + ((long long)(r0 + (st0 + a) * s.dl[0]) * s.L[1] + (r1 + (st1 + b) * s.dl[1])) * s.L[2] +
           (r2 + (st2 + c) * s.dl[2]);
  };
  auto logit = [&](int a, int b, int c) {
    Acc kv[E::kVec];
    E::load(k + key_of(a, b, c) * D + lane * E::kVec, kv);
    Acc part = 0;
#pragma unroll
    for (int x = 0; x < E::kVec; ++x) part = fma(qv[x], kv[x], part);
    Acc sum = group_sum<G>(part);
    if (tab)
      sum += E::scalar(tab + ((st0 + a - p0 + s.k[0] - 1) * b1 + (st1 + b - p1 + s.k[1] - 1)) * b2 +
                       (st2 + c - p2 + s.k[2] - 1));
    return sum;
  };
  Acc m = -std::numeric_limits<Acc>::infinity();
  for (int a = 0; a < s.k[0]; ++a)
    for (int b = 0; b < s.k[1]; ++b)
      for (int c = 0; c < s.k[2]; ++c) {
        const Acc x = logit(a, b, c);
        m = x > m ? x : m;
      }
  const Acc scale = (Acc)1 / sqrt((Acc)D);
  Acc l = 0, o[E::kVec];
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) o[x] = 0;
  for (int a = 0; a < s.k[0]; ++a)
    for (int b = 0; b < s.k[1]; ++b)
      for (int c = 0; c < s.k[2]; ++c) {
        const Acc w = acc_exp((logit(a, b, c) - m) * scale);
        l += w;
        Acc vv[E::kVec];
        E::load(v + key_of(a, b, c) * D + lane * E::kVec, vv);
#pragma unroll
        for (int x = 0; x < E::kVec; ++x) o[x] = fma(w, vv[x], o[x]);
      }
  if (!live) return;
  const Acc inv = (Acc)1 / l;
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) o[x] *= inv;
  E::store(out + qidx * D + lane * E::kVec, o);
}

}  // namespace

cudaError_t launch_forward_nd(const void* q, const void* k, const void* v, const void* rpb, void* out, int B,
                              int heads, const int (&L)[3], int d, const int (&ks)[3], const int (&dil)[3],
                              na_dtype dt, cudaStream_t st) {
  NdShape s;
  for (int a = 0; a < 3; ++a) {
    s.L[a] = L[a];
    s.k[a] = ks[a];
    s.dl[a] = dil[a];
  }
  const long long nq = (long long)B * heads * L[0] * L[1] * (long long)L[2];
  return dispatch(dt, d, [&]<typename T, int D>() {
    nd_forward_kernel<T, D><<<grid_for<T, D>(nq), kThreads, 0, st>>>((const T*)q, (const T*)k, (const T*)v,
                                                                       (const T*)rpb, (T*)out, nq, heads, s);
    return cudaGetLastError();
  });
}

}  // namespace na2d
