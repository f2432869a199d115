// na2d_common.cuh -- helpers shared by the CUDA kernels of the 2D
// Neighborhood Attention library (element traits, the window rule, bounded
// waits).  Device code only; nothing here allocates.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "na2d.h"

#define NA_DEVICE __device__ __forceinline__

namespace na2d {

// Bits of the per-device status word.
constexpr unsigned kStatusTimeout = 1u;

// Wall-clock limit of every device-side wait (ns): far above any legitimate
// wait of these kernels, far below a watchdog.
constexpr unsigned long long kWaitLimitNs = 2000ull * 1000ull * 1000ull;

// Start of the ks-wide window of position i on an axis of length L: the
// window keeps its full span and is shifted inward at the borders
// (Neighborhood Attention Transformer, Sec. 3.1 and App. C).
NA_DEVICE int window_start(int i, int L, int ks) {
  int s = i - (ks >> 1);
  s = s < 0 ? 0 : s;
  return s > L - ks ? L - ks : s;
}

NA_DEVICE unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- elements
template <typename T> struct Elem;

template <> struct Elem<float> {
  static constexpr int kVec = 4;  // elements per 16-byte vector
  using Acc = double;
  NA_DEVICE static void load(const float* p, Acc (&o)[kVec]) {
    float4 x = __ldg(reinterpret_cast<const float4*>(p));
    o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
  }
  NA_DEVICE static void store(float* p, const Acc (&o)[kVec]) {
    float4 x = make_float4((float)o[0], (float)o[1], (float)o[2], (float)o[3]);
    *reinterpret_cast<float4*>(p) = x;
  }
  NA_DEVICE static Acc scalar(const float* p) { return (Acc)__ldg(p); }
};

template <> struct Elem<__nv_bfloat16> {
  static constexpr int kVec = 8;
  using Acc = float;
  NA_DEVICE static void load(const __nv_bfloat16* p, Acc (&o)[kVec]) {
    uint4 x = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float2 f = __bfloat1622float2(h[t]);
      o[2 * t] = f.x; o[2 * t + 1] = f.y;
    }
  }
  NA_DEVICE static void store(__nv_bfloat16* p, const Acc (&o)[kVec]) {
    uint4 x;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&x);
#pragma unroll
    for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(o[2 * t], o[2 * t + 1]);
    *reinterpret_cast<uint4*>(p) = x;
  }
  NA_DEVICE static Acc scalar(const __nv_bfloat16* p) { return __bfloat162float(p[0]); }
};

template <> struct Elem<__half> {
  static constexpr int kVec = 8;
  using Acc = float;
  NA_DEVICE static void load(const __half* p, Acc (&o)[kVec]) {
    uint4 x = __ldg(reinterpret_cast<const uint4*>(p));
    const __half2* h = reinterpret_cast<const __half2*>(&x);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float2 f = __half22float2(h[t]);
      o[2 * t] = f.x; o[2 * t + 1] = f.y;
    }
  }
  NA_DEVICE static void store(__half* p, const Acc (&o)[kVec]) {
    uint4 x;
    __half2* h = reinterpret_cast<__half2*>(&x);
#pragma unroll
    for (int t = 0; t < 4; ++t) h[t] = __floats2half2_rn(o[2 * t], o[2 * t + 1]);
    *reinterpret_cast<uint4*>(p) = x;
  }
  NA_DEVICE static Acc scalar(const __half* p) { return __half2float(p[0]); }
};

NA_DEVICE double acc_exp(double x) { return exp(x); }
NA_DEVICE float acc_exp(float x) { return expf(x); }

}  // namespace na2d
