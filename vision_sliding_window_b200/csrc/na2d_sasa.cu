// na2d_sasa.cu -- SASA (stand-alone self-attention): the centred k x k window
// of every query with the positions outside the map taken as zero padding.
// The NAT paper, Sec. 3.2, calls SASA a special case of NA on a zero-padded
// input, and that is how it runs here: the map is padded by k/2 zero pixels
// on every side (q, k and v, into the caller's workspace), NA runs on the
// padded map -- there every original pixel's clamped window is its centred
// window -- and the original pixels' outputs are cropped out.
//
// The pad and crop kernels move 16-byte vectors, one per thread; d * element
// size is a multiple of 16 for every supported d.
#include "na2d_common.cuh"
#include "na2d_internal.h"

namespace na2d {
namespace {

constexpr int kThreads = 256;

// Writes the zero-padded copies of q, k and v: [B][heads][H+2p][W+2p][d],
// vec 16-byte vectors per pixel.
__global__ void __launch_bounds__(kThreads)
pad3_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
            uint4* __restrict__ qp, uint4* __restrict__ kp, uint4* __restrict__ vp, long long n_pad, int H, int W,
            int p, int vec) {
  const long long idx = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (idx >= 3 * n_pad) return;
  const int which = (int)(idx / n_pad);
  const long long e = idx - (long long)which * n_pad;
  const int Wp = W + 2 * p, Hp = H + 2 * p;
  const int x = (int)(e % vec);
  long long rest = e / vec;
  const int jp = (int)(rest % Wp);
  rest /= Wp;
  const int ip = (int)(rest % Hp);
  const long long map = rest / Hp;
  const int i = ip - p, j = jp - p;
  const uint4* src = which == 0 ? q : which == 1 ? k : v;
  uint4* dst = which == 0 ? qp : which == 1 ? kp : vp;
  uint4 val = make_uint4(0u, 0u, 0u, 0u);
  if (i >= 0 && i < H && j >= 0 && j < W) val = src[((map * H + i) * W + j) * vec + x];
  dst[e] = val;
}

// out[b][h][i][j] = outp[b][h][i+p][j+p].
__global__ void __launch_bounds__(kThreads)
crop_kernel(const uint4* __restrict__ outp, uint4* __restrict__ out, long long n, int H, int W, int p, int vec) {
  const long long e = (long long)blockIdx.x * kThreads + threadIdx.x;
  if (e >= n) return;
  const int x = (int)(e % vec);
  long long rest = e / vec;
  const int j = (int)(rest % W);
  rest /= W;
  const int i = (int)(rest % H);
  const long long map = rest / H;
  const int Wp = W + 2 * p, Hp = H + 2 * p;
  out[e] = outp[((map * Hp + i + p) * Wp + j + p) * vec + x];
}

size_t round_up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t sasa_workspace_bytes(const Shape& s, size_t es) {
  const int p = s.ks / 2;
  const size_t padded = (size_t)s.B * s.heads * (size_t)(s.H + 2 * p) * (size_t)(s.W + 2 * p) * s.d * es;
  return 4 * round_up256(padded);
}

cudaError_t launch_sasa_pad(const void* q, const void* k, const void* v, void* workspace, const Shape& s, size_t es,
                            cudaStream_t st, void** qp, void** kp, void** vp, void** outp) {
  const int p = s.ks / 2, vec = (int)(s.d * es / 16);
  const size_t one = sasa_workspace_bytes(s, es) / 4;
  char* ws = static_cast<char*>(workspace);
  *qp = ws;
  *kp = ws + one;
  *vp = ws + 2 * one;
  *outp = ws + 3 * one;
  const long long n_pad = (long long)s.B * s.heads * (s.H + 2 * p) * (long long)(s.W + 2 * p) * vec;
  const unsigned grid = (unsigned)((3 * n_pad + kThreads - 1) / kThreads);
  pad3_kernel<<<grid, kThreads, 0, st>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, (uint4*)*qp,
                                         (uint4*)*kp, (uint4*)*vp, n_pad, s.H, s.W, p, vec);
  return cudaGetLastError();
}

cudaError_t launch_sasa_crop(const void* outp, void* out, const Shape& s, size_t es, cudaStream_t st) {
  const int p = s.ks / 2, vec = (int)(s.d * es / 16);
  const long long n = s.queries() * vec;
  const unsigned grid = (unsigned)((n + kThreads - 1) / kThreads);
  crop_kernel<<<grid, kThreads, 0, st>>>((const uint4*)outp, (uint4*)out, n, s.H, s.W, p, vec);
  return cudaGetLastError();
}

}  // namespace na2d
