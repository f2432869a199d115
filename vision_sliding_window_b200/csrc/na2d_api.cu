// na2d_api.cu -- the extern "C" entry points of include/na2d.h: argument
// checks, kernel selection, the per-device status word, the host-buffer
// variant of the forward pass and the wait-timeout probe.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "na2d_common.cuh"
#include "na2d_internal.h"

#define NA_EXPORT extern "C" __attribute__((visibility("default")))

namespace na2d {
namespace {

// Status word of the device, written by kernels whose bounded waits ran
// out; read and cleared by na2d_device_status().
__device__ unsigned int g_status_word;

// Device address of the status word on the current device.  Looked up on
// every call (a host-side table lookup in the runtime): an address cached
// across calls would go stale if the process reset the device or created a
// new primary context, and the next kernel would write through it.
cudaError_t status_ptr(unsigned** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_status_word);
  if (e != cudaSuccess) return e;
  *out = static_cast<unsigned*>(p);
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

na_status check_shape(int B, int heads, int H, int W, int d, int ks, bool need_d, Shape* s) {
  if (B < 0 || heads < 0 || H < 1 || W < 1) return NA_ERR_INVALID_ARG;
  if (ks < 1 || (ks & 1) == 0 || ks > H || ks > W || ks > 63) return NA_ERR_INVALID_ARG;
  if (need_d && d != 16 && d != 32 && d != 64 && d != 128) return NA_ERR_INVALID_ARG;
  const long double n = (long double)B * heads * H * W;
  const long double per = (long double)(need_d ? (d > ks * ks ? d : ks * ks) : ks * ks);
  if (n * per >= (long double)(1ll << 62)) return NA_ERR_INVALID_ARG;
  *s = Shape{B, heads, H, W, need_d ? d : 0, ks};
  return NA_OK;
}

na_status check_dtype(na_dtype dt) {
  return (dt == NA_F32 || dt == NA_F16 || dt == NA_BF16) ? NA_OK : NA_ERR_INVALID_ARG;
}

size_t elem_size(na_dtype dt) { return dt == NA_F32 ? 4 : 2; }

na_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NA_OK : NA_ERR_CUDA; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Which forward kernel runs (shape already validated).
int forward_kernel_for(const Shape& s, na_dtype dt) {
  return forward_tc_supported(s, dt) ? 1 : 0;
}

__global__ void timeout_probe_kernel(unsigned* status, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  const unsigned addr = (unsigned)__cvta_generic_to_shared(&bar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(addr));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  // Nothing ever arrives on `bar`: this wait can only end by its limit.
  const unsigned long long t0 = globaltimer_ns();
  unsigned done = 0;
  while (!done) {
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr), "r"(0u)
        : "memory");
    if (!done && globaltimer_ns() - t0 > limit_ns) {
      atomicOr(status, kStatusTimeout);
      break;
    }
  }
}

}  // namespace
}  // namespace na2d

using namespace na2d;

NA_EXPORT const char* na_status_str(na_status s) {
  switch (s) {
    case NA_OK: return "NA_OK";
    case NA_ERR_INVALID_ARG: return "NA_ERR_INVALID_ARG";
    case NA_ERR_UNSUPPORTED: return "NA_ERR_UNSUPPORTED";
    case NA_ERR_CUDA: return "NA_ERR_CUDA";
    case NA_ERR_DEVICE_TIMEOUT: return "NA_ERR_DEVICE_TIMEOUT";
  }
  return "NA_ERR_UNKNOWN";
}

NA_EXPORT na_status na2d_qk_rpb(const void* q, const void* k, const void* rpb, float* attn,
                                int B, int heads, int H, int W, int d, int ksize, na_dtype dt,
                                void* stream) {
  Shape s;
  na_status st = check_dtype(dt);
  if (st == NA_OK) st = check_shape(B, heads, H, W, d, ksize, true, &s);
  if (st != NA_OK) return st;
  if (s.queries() == 0) return NA_OK;  // empty batch: nothing is read or written
  if (!q || !k || !attn || !aligned16(q) || !aligned16(k) || !aligned16(attn)) return NA_ERR_INVALID_ARG;
  if (rpb && !aligned16(rpb)) return NA_ERR_INVALID_ARG;
  return from_cuda(launch_qk_rpb_simt(q, k, rpb, attn, s, dt, (cudaStream_t)stream));
}

NA_EXPORT na_status na2d_softmax(float* attn, int B, int heads, int H, int W, int ksize,
                                 float scale, void* stream) {
  Shape s;
  na_status st = check_shape(B, heads, H, W, 0, ksize, false, &s);
  if (st != NA_OK) return st;
  if (!std::isfinite(scale)) return NA_ERR_INVALID_ARG;
  if (s.queries() == 0) return NA_OK;
  if (!attn || !aligned16(attn)) return NA_ERR_INVALID_ARG;
  return from_cuda(launch_softmax_simt(attn, s.queries(), ksize, scale, (cudaStream_t)stream));
}

NA_EXPORT na_status na2d_av(const float* attn, const void* v, void* out, int B, int heads, int H,
                            int W, int d, int ksize, na_dtype dt, void* stream) {
  Shape s;
  na_status st = check_dtype(dt);
  if (st == NA_OK) st = check_shape(B, heads, H, W, d, ksize, true, &s);
  if (st != NA_OK) return st;
  if (s.queries() == 0) return NA_OK;
  if (!attn || !v || !out || !aligned16(attn) || !aligned16(v) || !aligned16(out)) return NA_ERR_INVALID_ARG;
  return from_cuda(launch_av_simt(attn, v, out, s, dt, (cudaStream_t)stream));
}

NA_EXPORT int na2d_forward_kernel(int B, int heads, int H, int W, int d, int ksize, na_dtype dt) {
  Shape s;
  na_status st = check_dtype(dt);
  if (st == NA_OK) st = check_shape(B, heads, H, W, d, ksize, true, &s);
  if (st != NA_OK) return -(int)st;
  return forward_kernel_for(s, dt);
}

NA_EXPORT na_status na2d_forward(const void* q, const void* k, const void* v, const void* rpb,
                                 void* out, int B, int heads, int H, int W, int d, int ksize,
                                 na_dtype dt, void* stream) {
  Shape s;
  na_status st = check_dtype(dt);
  if (st == NA_OK) st = check_shape(B, heads, H, W, d, ksize, true, &s);
  if (st != NA_OK) return st;
  if (s.queries() == 0) return NA_OK;
  if (!q || !k || !v || !out) return NA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return NA_ERR_INVALID_ARG;
  if (rpb && !aligned16(rpb)) return NA_ERR_INVALID_ARG;
  cudaStream_t cs = (cudaStream_t)stream;
  if (forward_kernel_for(s, dt) == 1) {
    unsigned* status = nullptr;
    cudaError_t e = status_ptr(&status);
    if (e != cudaSuccess) return NA_ERR_CUDA;
    return from_cuda(launch_forward_tc(q, k, v, rpb, out, s, dt, status, cs));
  }
  return from_cuda(launch_forward_simt(q, k, v, rpb, out, s, dt, cs));
}

NA_EXPORT size_t na2d_backward_workspace_bytes(int B, int heads, int H, int W, int d, int ksize, na_dtype dt) {
  Shape s;
  if (check_dtype(dt) != NA_OK || check_shape(B, heads, H, W, d, ksize, true, &s) != NA_OK) return 0;
  return backward_workspace_bytes(s);
}

NA_EXPORT na_status na2d_backward(const void* q, const void* k, const void* v, const void* rpb, const void* dout,
                                  void* dq, void* dk, void* dv, float* drpb, void* workspace,
                                  size_t workspace_bytes, int B, int heads, int H, int W, int d, int ksize,
                                  na_dtype dt, void* stream) {
  Shape s;
  na_status st = check_dtype(dt);
  if (st == NA_OK) st = check_shape(B, heads, H, W, d, ksize, true, &s);
  if (st != NA_OK) return st;
  if (s.queries() == 0) return NA_OK;
  for (const void* ptr : {q, k, v, dout, (const void*)dq, (const void*)dk, (const void*)dv, (const void*)workspace})
    if (!ptr || !aligned16(ptr)) return NA_ERR_INVALID_ARG;
  if ((rpb && !aligned16(rpb)) || (drpb && !aligned16(drpb))) return NA_ERR_INVALID_ARG;
  if (workspace_bytes < backward_workspace_bytes(s)) return NA_ERR_INVALID_ARG;
  return from_cuda(launch_backward_simt(q, k, v, rpb, dout, dq, dk, dv, drpb, workspace, s, dt,
                                        (cudaStream_t)stream));
}

namespace {
// SASA takes any odd k: its padded map (H + k - 1 by W + k - 1) always holds
// a window.
na_status check_sasa_shape(int B, int heads, int H, int W, int d, int ks, Shape* s) {
  if (B < 0 || heads < 0 || H < 1 || W < 1) return NA_ERR_INVALID_ARG;
  if (ks < 1 || (ks & 1) == 0 || ks > 63) return NA_ERR_INVALID_ARG;
  if (d != 16 && d != 32 && d != 64 && d != 128) return NA_ERR_INVALID_ARG;
  const long double n = (long double)B * heads * (H + ks - 1) * (W + ks - 1);
  if (n * (long double)(d > ks * ks ? d : ks * ks) >= (long double)(1ll << 62)) return NA_ERR_INVALID_ARG;
  *s = Shape{B, heads, H, W, d, ks};
  return NA_OK;
}
}  // namespace

NA_EXPORT size_t na2d_sasa_workspace_bytes(int B, int heads, int H, int W, int d, int ksize, na_dtype dt) {
  Shape s;
  if (check_dtype(dt) != NA_OK || check_sasa_shape(B, heads, H, W, d, ksize, &s) != NA_OK) return 0;
  return sasa_workspace_bytes(s, elem_size(dt));
}

NA_EXPORT na_status na2d_sasa_forward(const void* q, const void* k, const void* v, const void* rpb, void* out,
                                      void* workspace, size_t workspace_bytes, int B, int heads, int H, int W,
                                      int d, int ksize, na_dtype dt, void* stream) {
  Shape s;
  na_status st = check_dtype(dt);
  if (st == NA_OK) st = check_sasa_shape(B, heads, H, W, d, ksize, &s);
  if (st != NA_OK) return st;
  if (s.queries() == 0) return NA_OK;
  for (const void* ptr : {q, k, v, (const void*)out})
    if (!ptr || !aligned16(ptr)) return NA_ERR_INVALID_ARG;
  if (rpb && !aligned16(rpb)) return NA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return NA_ERR_INVALID_ARG;
  const size_t es = elem_size(dt);
  if (workspace_bytes < sasa_workspace_bytes(s, es)) return NA_ERR_INVALID_ARG;
  cudaStream_t cs = (cudaStream_t)stream;
  void *qp, *kp, *vp, *outp;
  if (launch_sasa_pad(q, k, v, workspace, s, es, cs, &qp, &kp, &vp, &outp) != cudaSuccess) return NA_ERR_CUDA;
  const int pad = ksize / 2;
  st = na2d_forward(qp, kp, vp, rpb, outp, B, heads, H + 2 * pad, W + 2 * pad, d, ksize, dt, stream);
  if (st != NA_OK) return st;
  return from_cuda(launch_sasa_crop(outp, out, s, es, cs));
}

NA_EXPORT size_t na2d_block_workspace_bytes(int B, int H, int W, int heads, int dh, int ksize, na_dtype dt) {
  Shape s;
  if (check_dtype(dt) != NA_OK || check_shape(B, heads, H, W, dh, ksize, true, &s) != NA_OK) return 0;
  if ((long long)B * H * W >= (1ll << 31) || (long long)heads * dh * 3 >= (1ll << 31)) return 0;
  return block_workspace_bytes(B, H, W, heads, dh, elem_size(dt));
}

NA_EXPORT na_status na2d_block_forward(const void* x, const void* wqkv, const void* bqkv, const void* wo,
                                       const void* bo, const void* rpb, void* y, void* workspace,
                                       size_t workspace_bytes, int B, int H, int W, int heads, int dh, int ksize,
                                       na_dtype dt, void* stream) {
  Shape s;
  na_status st = check_dtype(dt);
  if (st == NA_OK) st = check_shape(B, heads, H, W, dh, ksize, true, &s);
  if (st != NA_OK) return st;
  if (s.queries() == 0) return NA_OK;
  if ((long long)B * H * W >= (1ll << 31) || (long long)heads * dh * 3 >= (1ll << 31)) return NA_ERR_INVALID_ARG;
  for (const void* ptr : {x, wqkv, wo, (const void*)y})
    if (!ptr || !aligned16(ptr)) return NA_ERR_INVALID_ARG;
  for (const void* ptr : {bqkv, bo, rpb})
    if (ptr && !aligned16(ptr)) return NA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return NA_ERR_INVALID_ARG;
  if (workspace_bytes < block_workspace_bytes(B, H, W, heads, dh, elem_size(dt))) return NA_ERR_INVALID_ARG;
  return run_block(x, wqkv, bqkv, wo, bo, rpb, y, workspace, B, H, W, heads, dh, ksize, dt, (cudaStream_t)stream);
}

NA_EXPORT na_status na_forward_nd(const void* q, const void* k, const void* v, const void* rpb, void* out, int B,
                                  int heads, int L0, int L1, int L2, int d, int k0, int k1, int k2, int dil0,
                                  int dil1, int dil2, na_dtype dt, void* stream) {
  na_status st = check_dtype(dt);
  if (st != NA_OK) return st;
  const int L[3] = {L0, L1, L2}, ks[3] = {k0, k1, k2}, dil[3] = {dil0, dil1, dil2};
  if (B < 0 || heads < 0 || (d != 16 && d != 32 && d != 64 && d != 128)) return NA_ERR_INVALID_ARG;
  long double n = (long double)B * heads;
  for (int a = 0; a < 3; ++a) {
    if (L[a] < 1 || ks[a] < 1 || (ks[a] & 1) == 0 || ks[a] > 63 || dil[a] < 1) return NA_ERR_INVALID_ARG;
    if (L[a] / dil[a] < ks[a]) return NA_ERR_INVALID_ARG;  // every sub-grid holds a window
    n *= L[a];
  }
  if (n * (long double)(d > ks[0] * ks[1] * ks[2] ? d : ks[0] * ks[1] * ks[2]) >= (long double)(1ll << 62))
    return NA_ERR_INVALID_ARG;
  if (n == 0) return NA_OK;
  for (const void* ptr : {q, k, v, (const void*)out})
    if (!ptr || !aligned16(ptr)) return NA_ERR_INVALID_ARG;
  if (rpb && !aligned16(rpb)) return NA_ERR_INVALID_ARG;
  return from_cuda(launch_forward_nd(q, k, v, rpb, out, B, heads, L, d, ks, dil, dt, (cudaStream_t)stream));
}

namespace {
struct HostLayout {
  size_t q, k, v, rpb, out, total, tensor_bytes, rpb_bytes;
};
// The workspace always reserves room for the bias table, so its size does
// not depend on whether the caller passes one.
HostLayout host_layout(const Shape& s, na_dtype dt) {
  HostLayout L{};
  const size_t es = elem_size(dt);
  L.tensor_bytes = (size_t)s.queries() * (size_t)s.d * es;
  L.rpb_bytes = (size_t)s.heads * (2 * s.ks - 1) * (2 * s.ks - 1) * es;
  size_t off = 0;
  L.q = off; off = round_up(off + L.tensor_bytes, 256);
  L.k = off; off = round_up(off + L.tensor_bytes, 256);
  L.v = off; off = round_up(off + L.tensor_bytes, 256);
  L.out = off; off = round_up(off + L.tensor_bytes, 256);
  L.rpb = off; off = round_up(off + L.rpb_bytes, 256);
  L.total = off;
  return L;
}
}  // namespace

NA_EXPORT size_t na2d_forward_host_workspace_bytes(int B, int heads, int H, int W, int d, int ksize,
                                                   na_dtype dt) {
  Shape s;
  if (check_dtype(dt) != NA_OK || check_shape(B, heads, H, W, d, ksize, true, &s) != NA_OK) return 0;
  return host_layout(s, dt).total;
}

namespace {
// Streams per device on which na2d_forward_host runs batch chunks side by
// side, one chunk per stream -- the host-to-device copies of one chunk
// overlap the kernel and the device-to-host copy of the previous ones, and
// no stream holds a chunk's input copy behind another chunk's output copy --
// and the events that fork them from, and join them back to, the caller's
// stream.  Created by the first such call on the device and kept for the
// life of the process; calls are enqueued one at a time (a host mutex), so
// the shared events are never recorded by two calls at once.
constexpr int kLanes = 4;
struct Lanes {
  cudaStream_t s[kLanes];
  cudaEvent_t fork, join[kLanes], in_done[kLanes];
  bool ready;
};
constexpr int kMaxDevices = 64;
std::mutex g_lanes_mu;
Lanes g_lanes[kMaxDevices];

cudaError_t lanes_for_current_device(Lanes** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  Lanes& L = g_lanes[dev];
  if (!L.ready) {
    for (int i = 0; i < kLanes && e == cudaSuccess; ++i) e = cudaStreamCreateWithFlags(&L.s[i], cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming);
    for (int i = 0; i < kLanes && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&L.join[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L.in_done[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return e;
    L.ready = true;
  }
  *out = &L;
  return cudaSuccess;
}

// The host-buffer forward.  serial: every copy and the kernel in order on
// the caller's stream.  Otherwise the batch is cut into up to kLanes chunks
// of whole batch entries, chunk c going to lane c: its inputs'
// host-to-device copies, its forward and its output's device-to-host copy,
// so that one chunk's copies overlap another's kernel and copies in the two
// directions overlap each other.
na_status forward_host_impl(const void* q_host, const void* k_host, const void* v_host, const void* rpb_host,
                            void* out_host, void* workspace, size_t workspace_bytes, int B, int heads, int H,
                            int W, int d, int ksize, na_dtype dt, void* stream, bool serial) {
  Shape s;
  na_status st = check_dtype(dt);
  if (st == NA_OK) st = check_shape(B, heads, H, W, d, ksize, true, &s);
  if (st != NA_OK) return st;
  if (s.queries() == 0) return NA_OK;
  if (!q_host || !k_host || !v_host || !out_host || !workspace) return NA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return NA_ERR_INVALID_ARG;
  const HostLayout L = host_layout(s, dt);
  if (workspace_bytes < L.total) return NA_ERR_INVALID_ARG;
  cudaStream_t cs = (cudaStream_t)stream;
  char* ws = static_cast<char*>(workspace);
  const char* qh = static_cast<const char*>(q_host);
  const char* kh = static_cast<const char*>(k_host);
  const char* vh = static_cast<const char*>(v_host);
  char* oh = static_cast<char*>(out_host);
  cudaError_t e = cudaSuccess;
  if (rpb_host) e = cudaMemcpyAsync(ws + L.rpb, rpb_host, L.rpb_bytes, cudaMemcpyHostToDevice, cs);
  if (e != cudaSuccess) return NA_ERR_CUDA;
  const void* rpb_dev = rpb_host ? ws + L.rpb : nullptr;
  const int chunks = serial ? 1 : (B < kLanes ? B : kLanes);
  if (chunks <= 1) {
    e = cudaMemcpyAsync(ws + L.q, qh, L.tensor_bytes, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ws + L.k, kh, L.tensor_bytes, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ws + L.v, vh, L.tensor_bytes, cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return NA_ERR_CUDA;
    st = na2d_forward(ws + L.q, ws + L.k, ws + L.v, rpb_dev, ws + L.out, B, heads, H, W, d, ksize, dt, stream);
    if (st != NA_OK) return st;
    return from_cuda(cudaMemcpyAsync(oh, ws + L.out, L.tensor_bytes, cudaMemcpyDeviceToHost, cs));
  }
  std::lock_guard<std::mutex> lk(g_lanes_mu);
  Lanes* ln = nullptr;
  if (lanes_for_current_device(&ln) != cudaSuccess) return NA_ERR_CUDA;
  e = cudaEventRecord(ln->fork, cs);
  for (int i = 0; i < chunks && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(ln->s[i], ln->fork, 0);
  if (e != cudaSuccess) return NA_ERR_CUDA;
  const size_t per_b = L.tensor_bytes / (size_t)B;
  for (int c = 0; c < chunks && st == NA_OK; ++c) {
    const int b0 = (int)((long long)B * c / chunks), b1 = (int)((long long)B * (c + 1) / chunks);
    const size_t off = per_b * (size_t)b0, bytes = per_b * (size_t)(b1 - b0);
    cudaStream_t ls = ln->s[c];
    // the chunks' input copies run one after another, each at the link's
    // full rate, so that chunk c's kernel starts as soon as its own inputs
    // are in (copies running side by side would share the link and land
    // together)
    e = c > 0 ? cudaStreamWaitEvent(ls, ln->in_done[c - 1], 0) : cudaSuccess;
    if (e == cudaSuccess) e = cudaMemcpyAsync(ws + L.q + off, qh + off, bytes, cudaMemcpyHostToDevice, ls);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ws + L.k + off, kh + off, bytes, cudaMemcpyHostToDevice, ls);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ws + L.v + off, vh + off, bytes, cudaMemcpyHostToDevice, ls);
    if (e == cudaSuccess) e = cudaEventRecord(ln->in_done[c], ls);
    if (e != cudaSuccess) {
      st = NA_ERR_CUDA;
      break;
    }
    st = na2d_forward(ws + L.q + off, ws + L.k + off, ws + L.v + off, rpb_dev, ws + L.out + off, b1 - b0, heads, H,
                      W, d, ksize, dt, (void*)ls);
    if (st == NA_OK && cudaMemcpyAsync(oh + off, ws + L.out + off, bytes, cudaMemcpyDeviceToHost, ls) != cudaSuccess)
      st = NA_ERR_CUDA;
  }
  // the caller's stream waits for every lane used, also after a failed enqueue
  for (int i = 0; i < chunks; ++i)
    if (cudaEventRecord(ln->join[i], ln->s[i]) != cudaSuccess || cudaStreamWaitEvent(cs, ln->join[i], 0) != cudaSuccess)
      st = NA_ERR_CUDA;
  return st;
}
}  // namespace

NA_EXPORT na_status na2d_forward_host(const void* q_host, const void* k_host, const void* v_host,
                                      const void* rpb_host, void* out_host, void* workspace,
                                      size_t workspace_bytes, int B, int heads, int H, int W, int d,
                                      int ksize, na_dtype dt, void* stream) {
  return forward_host_impl(q_host, k_host, v_host, rpb_host, out_host, workspace, workspace_bytes, B, heads, H, W,
                           d, ksize, dt, stream, false);
}

// For na2d_noalloc.cu: the same call with every step on the caller's stream.
namespace na2d {
na_status forward_host_serial(const void* q_host, const void* k_host, const void* v_host, const void* rpb_host,
                              void* out_host, void* workspace, size_t workspace_bytes, int B, int heads, int H,
                              int W, int d, int ksize, na_dtype dt, void* stream) {
  return forward_host_impl(q_host, k_host, v_host, rpb_host, out_host, workspace, workspace_bytes, B, heads, H, W,
                           d, ksize, dt, stream, true);
}
}  // namespace na2d

NA_EXPORT na_status na2d_device_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return NA_ERR_CUDA;
  unsigned* p = nullptr;
  if (status_ptr(&p) != cudaSuccess) return NA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return NA_ERR_CUDA;
  if (v && cudaMemset(p, 0, sizeof(v)) != cudaSuccess) return NA_ERR_CUDA;
  return (v & kStatusTimeout) ? NA_ERR_DEVICE_TIMEOUT : NA_OK;
}

NA_EXPORT na_status na2d_debug_timeout_probe(unsigned int timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000u) return NA_ERR_INVALID_ARG;
  unsigned* p = nullptr;
  if (status_ptr(&p) != cudaSuccess) return NA_ERR_CUDA;
  timeout_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(p, 1000ull * timeout_us);
  return from_cuda(cudaGetLastError());
}
