// na2d_bwd.cu -- backward pass of 2D Neighborhood Attention: the gradients
// of a scalar loss L with respect to q, k, v and the bias table, given
// dout = dL/d(out).  NATTEN provides "QK+B" and "AV" together with the
// gradients of their backward passes (Qiita write-up, section "NATTEN"); the
// NAT paper, Sec. 3.2, makes the operator an autograd function.
//
// With A_n = q . k_n + B_n (Eq. 2), z = A / sqrt(d), P = softmax(z) and
// out = sum_n P_n v_n (Eqs. 3-4), the chain rule gives per query and window
// entry n:  dP_n = dout . v_n,  D = sum_n P_n dP_n = dout . out,
// dA_n = P_n (dP_n - D) / sqrt(d),  and
//   dq(query) = sum_n dA_n k_n,      dk(key) = sum_queries dA q,
//   dv(key)   = sum_queries P dout,  dB[h][disp] = sum over (query, n) with that displacement of dA_n.
//
// Three CUDA-core passes, each recomputing logits rather than storing the
// k^2 attention weights of every query:
//   1. per query (one group of lanes): the logits' maximum, the softmax sum
//      and D, then dq; the log-sum-exp and D go to the workspace;
//   2. per key: the queries whose window holds the key form a rectangle of
//      the map; dk and dv are summed over it with P = exp(z - lse);
//   3. per head and displacement (one CTA each): dB summed over every query
//      that has a key at that displacement, reduced in a fixed order.
// Accumulation is float64 for float32 inputs and float32 otherwise; every
// gradient is written exactly once, so no output needs clearing.
#include "na2d_simt.cuh"

namespace na2d {
namespace {

using namespace simt;

// Per-query values kept between the passes: the log-sum-exp of the scaled
// logits and D = sum_n P_n dP_n.
struct QueryStats {
  double lse, dsum;
};

// Dot product of two rows of d elements held as 16-byte slices by the G
// lanes of a group.
template <typename T, int D>
NA_DEVICE typename Elem<T>::Acc group_dot(const typename Elem<T>::Acc (&a)[Elem<T>::kVec], const T* row, int lane) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  Acc b[E::kVec];
  E::load(row + lane * E::kVec, b);
  Acc s = 0;
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) s = fma(a[x], b[x], s);
  return group_sum<D / E::kVec>(s);
}

// Pass 1, one group of lanes per query.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
bwd_query_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const T* __restrict__ rpb, const T* __restrict__ dout, T* __restrict__ dq,
                 QueryStats* __restrict__ stats, long long nq, int heads, int H, int W, int ks) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  constexpr int G = D / E::kVec;
  const long long g = ((long long)blockIdx.x * kThreads + threadIdx.x) / G;
  const int lane = threadIdx.x % G;
  const bool live = g < nq;
  const long long qidx = live ? g : nq - 1;  // dead groups shadow a live query, store nothing
  const QueryPos p = decode(qidx, heads, H, W);
  const int span = 2 * ks - 1;
  const long long map_off = p.bh * H * W * (long long)D;
  const T* kmap = k + map_off;
  const T* vmap = v + map_off;
  const T* tab = rpb ? rpb + (long long)p.h * span * span : nullptr;
  Acc qv[E::kVec], gv[E::kVec];
  E::load(q + qidx * D + lane * E::kVec, qv);
  E::load(dout + qidx * D + lane * E::kVec, gv);
  const int si = window_start(p.i, H, ks), sj = window_start(p.j, W, ks);
  const Acc scale = (Acc)1 / sqrt((Acc)D);

  Acc m = -std::numeric_limits<Acc>::infinity();
  for (int a = 0; a < ks; ++a)
    for (int c = 0; c < ks; ++c) {
      const Acc s = group_logit<T, D>(qv, kmap, tab, W, ks, span, p.i, p.j, si + a, sj + c, lane);
      m = s > m ? s : m;
    }
  Acc l = 0, pd = 0;  // sum of exp((s - m) scale) and of the same times dP
  for (int a = 0; a < ks; ++a)
    for (int c = 0; c < ks; ++c) {
      const int r = si + a, t = sj + c;
      const Acc s = group_logit<T, D>(qv, kmap, tab, W, ks, span, p.i, p.j, r, t, lane);
      const Acc w = acc_exp((s - m) * scale);
      l += w;
      pd = fma(w, group_dot<T, D>(gv, vmap + ((long long)r * W + t) * D, lane), pd);
    }
  const Acc inv = (Acc)1 / l, dsum = pd * inv;
  Acc dqv[E::kVec];
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) dqv[x] = 0;
  for (int a = 0; a < ks; ++a)
    for (int c = 0; c < ks; ++c) {
      const int r = si + a, t = sj + c;
      const Acc s = group_logit<T, D>(qv, kmap, tab, W, ks, span, p.i, p.j, r, t, lane);
      const Acc dp = group_dot<T, D>(gv, vmap + ((long long)r * W + t) * D, lane);
      const Acc dA = acc_exp((s - m) * scale) * inv * (dp - dsum) * scale;
      Acc kv[E::kVec];
      E::load(kmap + ((long long)r * W + t) * D + lane * E::kVec, kv);
#pragma unroll
      for (int x = 0; x < E::kVec; ++x) dqv[x] = fma(dA, kv[x], dqv[x]);
    }
  if (!live) return;
  E::store(dq + qidx * D + lane * E::kVec, dqv);
  if (lane == 0) stats[qidx] = QueryStats{(double)m * (double)scale + log((double)l), (double)dsum};
}

// The rows (or columns) of the queries whose window holds key row r on an
// axis of length L: with si = clamp(i - ks/2, 0, L - ks) non-decreasing in
// i, they form [lo, hi].
NA_DEVICE void inverse_range(int r, int L, int ks, int& lo, int& hi) {
  lo = r <= ks - 1 ? 0 : r - ks / 2;
  hi = r >= L - ks ? L - 1 : r + ks / 2;
}

// Pass 2, one group of lanes per key.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
bwd_key_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
               const T* __restrict__ rpb, const T* __restrict__ dout, const QueryStats* __restrict__ stats,
               T* __restrict__ dk, T* __restrict__ dv, long long nkeys, int heads, int H, int W, int ks) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  constexpr int G = D / E::kVec;
  const long long g = ((long long)blockIdx.x * kThreads + threadIdx.x) / G;
  const int lane = threadIdx.x % G;
  const bool live = g < nkeys;
  const long long kidx = live ? g : nkeys - 1;
  const QueryPos p = decode(kidx, heads, H, W);  // the key's (b, h, row, column)
  const int span = 2 * ks - 1;
  const long long map_q = p.bh * H * W;  // first query of the map
  const T* tab = rpb ? rpb + (long long)p.h * span * span : nullptr;
  Acc kv[E::kVec], vv[E::kVec];
  E::load(k + kidx * D + lane * E::kVec, kv);
  E::load(v + kidx * D + lane * E::kVec, vv);
  const Acc scale = (Acc)1 / sqrt((Acc)D);
  int i0, i1, j0, j1;
  inverse_range(p.i, H, ks, i0, i1);
  inverse_range(p.j, W, ks, j0, j1);
  Acc dkv[E::kVec], dvv[E::kVec];
#pragma unroll
  for (int x = 0; x < E::kVec; ++x) dkv[x] = dvv[x] = 0;
  for (int i = i0; i <= i1; ++i)
    for (int j = j0; j <= j1; ++j) {
      const long long qi = map_q + (long long)i * W + j;
      Acc qv[E::kVec], gv[E::kVec];
      E::load(q + qi * D + lane * E::kVec, qv);
      E::load(dout + qi * D + lane * E::kVec, gv);
      Acc s = 0, dp = 0;
#pragma unroll
      for (int x = 0; x < E::kVec; ++x) {
        s = fma(qv[x], kv[x], s);
        dp = fma(gv[x], vv[x], dp);
      }
      s = group_sum<G>(s);
      dp = group_sum<G>(dp);
      if (tab) s += E::scalar(tab + (p.i - i + ks - 1) * span + (p.j - j + ks - 1));
      const QueryStats st = stats[qi];
      const Acc P = (Acc)exp((double)s * (double)scale - st.lse);
      const Acc dA = P * (dp - (Acc)st.dsum) * scale;
#pragma unroll
      for (int x = 0; x < E::kVec; ++x) {
        dkv[x] = fma(dA, qv[x], dkv[x]);
        dvv[x] = fma(P, gv[x], dvv[x]);
      }
    }
  if (!live) return;
  E::store(dk + kidx * D + lane * E::kVec, dkv);
  E::store(dv + kidx * D + lane * E::kVec, dvv);
}

// Pass 3, one CTA per (head, displacement (dr, dc)): the sum over every
// query (b, i, j) of that head whose window holds key (i + dr, j + dc) of
// dA at that key.  Each thread takes queries kThreads apart; the partial
// sums are reduced in a fixed order.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
bwd_rpb_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
               const T* __restrict__ rpb, const T* __restrict__ dout, const QueryStats* __restrict__ stats,
               float* __restrict__ drpb, int B, int heads, int H, int W, int ks) {
  using E = Elem<T>;
  using Acc = typename E::Acc;
  const int span = 2 * ks - 1;
  const int h = blockIdx.x / (span * span), e = blockIdx.x % (span * span);
  const int dr = e / span - (ks - 1), dc = e % span - (ks - 1);
  const Acc scale = (Acc)1 / sqrt((Acc)D);
  const Acc bias = rpb ? E::scalar(rpb + (long long)h * span * span + e) : (Acc)0;
  const long long per_map = (long long)H * W, n = (long long)B * per_map;
  Acc acc = 0;
  for (long long t = threadIdx.x; t < n; t += kThreads) {
    const int b = (int)(t / per_map);
    const int rem = (int)(t - (long long)b * per_map), i = rem / W, j = rem - (rem / W) * W;
    const int r = i + dr, c = j + dc;
    const int si = window_start(i, H, ks), sj = window_start(j, W, ks);
    if (r < si || r >= si + ks || c < sj || c >= sj + ks) continue;
    const long long map = ((long long)b * heads + h) * per_map;
    const long long qi = map + (long long)i * W + j, ki = map + (long long)r * W + c;
    Acc s = 0, dp = 0;
    for (int x = 0; x < D; x += E::kVec) {
      Acc qv[E::kVec], kv[E::kVec], gv[E::kVec], vv[E::kVec];
      E::load(q + qi * D + x, qv);
      E::load(k + ki * D + x, kv);
      E::load(dout + qi * D + x, gv);
      E::load(v + ki * D + x, vv);
#pragma unroll
      for (int y = 0; y < E::kVec; ++y) {
        s = fma(qv[y], kv[y], s);
        dp = fma(gv[y], vv[y], dp);
      }
    }
    const QueryStats st = stats[qi];
    const Acc P = (Acc)exp((double)(s + bias) * (double)scale - st.lse);
    acc += P * (dp - (Acc)st.dsum) * scale;
  }
  __shared__ double red[kThreads];
  red[threadIdx.x] = (double)acc;
  __syncthreads();
  for (int off = kThreads / 2; off > 0; off >>= 1) {
    if (threadIdx.x < off) red[threadIdx.x] += red[threadIdx.x + off];
    __syncthreads();
  }
  if (threadIdx.x == 0) drpb[blockIdx.x] = (float)red[0];
}

}  // namespace

size_t backward_workspace_bytes(const Shape& s) { return (size_t)s.queries() * sizeof(QueryStats); }

cudaError_t launch_backward_simt(const void* q, const void* k, const void* v, const void* rpb, const void* dout,
                                 void* dq, void* dk, void* dv, float* drpb, void* workspace, const Shape& s,
                                 na_dtype dt, cudaStream_t st) {
  const long long nq = s.queries();
  QueryStats* stats = static_cast<QueryStats*>(workspace);
  return dispatch(dt, s.d, [&]<typename T, int D>() {
    bwd_query_kernel<T, D><<<grid_for<T, D>(nq), kThreads, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)v, (const T*)rpb, (const T*)dout, (T*)dq, stats, nq, s.heads, s.H,
        s.W, s.ks);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_key_kernel<T, D><<<grid_for<T, D>(nq), kThreads, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)v, (const T*)rpb, (const T*)dout, stats, (T*)dk, (T*)dv, nq, s.heads,
        s.H, s.W, s.ks);
    e = cudaGetLastError();
    if (e != cudaSuccess || !drpb) return e;
    const int span = 2 * s.ks - 1;
    bwd_rpb_kernel<T, D><<<(unsigned)(s.heads * span * span), kThreads, 0, st>>>(
        (const T*)q, (const T*)k, (const T*)v, (const T*)rpb, (const T*)dout, stats, drpb, s.B, s.heads, s.H, s.W,
        s.ks);
    return cudaGetLastError();
  });
}

}  // namespace na2d
