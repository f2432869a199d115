// na2d_tc.cu -- tensor-core fused forward of 2D Neighborhood Attention for
// fp16 / bf16 on sm_100a (Neighborhood Attention Transformer, Sec. 3.1,
// Eqs. (2)-(4); the tiling follows the "tiled NA" idea of Sec. 3.2 and
// App. A.4: a query tile plus its key/value halo staged in shared memory).
//
// One persistent CTA per SM walks a list of 8 x 16 query tiles.  Per tile:
//   * TMA loads the query tile (four 4 x 8 patches) and the K and V halo --
//     the (8+k-1) x (16+k-1, rounded up to 8) keys every window of the tile
//     lies in -- into swizzled shared memory (double-buffered).
//   * One thread issues tcgen05.mma: S = Q_tile . K_halo^T (M = 128 queries,
//     N = halo keys, float32 in tensor memory).
//   * Four softmax warps, each owning one 4 x 8 patch (32 TMEM lanes), read
//     only the union of their 32 windows from tensor memory, add the bias
//     (and -inf outside each query's clamped window) from a per-head table in
//     shared memory, take the row maximum, then write exp2((s - m) * log2e /
//     sqrt(d)) rounded to 16 bits back over S as the P operand (zeros outside
//     the union).
//   * tcgen05.mma: O = P . V_halo (A = P from tensor memory, B = V in shared
//     memory, N = d), then the softmax warps divide by the row sum and store.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "na2d_common.cuh"
#include "na2d_internal.h"
#include "na2d_sm100.cuh"

namespace na2d {
namespace {

using namespace sm100;

constexpr int TH = 8, TW = 16;  // query tile (rows x columns), 128 queries = MMA M
constexpr int PH = 4, PW = 8;   // query patch of one softmax warp (32 TMEM lanes)
constexpr int kSoftmaxWarps = 4;
constexpr int kThreads = 32 * (2 + kSoftmaxWarps);
constexpr int kTmemCols = 512;
constexpr int kMinSmem = 116 * 1024;  // keeps one CTA per SM (it holds all of tensor memory)

template <int KS, int D>
struct Cfg {
  static constexpr int HH = TH + KS - 1;                    // halo rows
  static constexpr int HW = (TW + KS - 1 + 7) / 8 * 8;      // halo columns, multiple of 8
  static constexpr int NS = HH * HW;                        // halo keys = S columns
  static constexpr int NP = HW / 8;                         // 8-key pieces per halo row
  static constexpr int ROWB = D * 2;                        // bytes per key / query row
  static constexpr int Q_BYTES = TH * TW * ROWB;
  static constexpr int KV_BYTES = NS * ROWB;
  static constexpr int STAGE_BYTES = Q_BYTES + 2 * KV_BYTES;
  // bias / mask table: rows 0..2KS-2 are bias rows, row 2KS-1 is all -inf.
  // Row layout: KS blocks of stride KS+PAD, block dc = [PAD x -inf][bias
  // row, columns dc .. dc+KS-1][shared with the next block's -inf pad].
  static constexpr int PAD = (PW - 1) + 7;
  static constexpr int TBL_W0 = KS * (KS + PAD) + PAD;
  static constexpr int TBL_W = TBL_W0 + ((8 - TBL_W0 % 32) + 32) % 32;  // = 8 mod 32: no bank conflicts
  static constexpr int TBL_ROWS = 2 * KS;
  static constexpr int TBL_BYTES = TBL_ROWS * TBL_W * 4;
  static constexpr int STAGES = (2 * STAGE_BYTES + TBL_BYTES + 4096 <= 200 * 1024) ? 2 : 1;
  static constexpr int S_COL = 0;
  static constexpr int O_COL = (NS + 31) / 32 * 32;
  static constexpr int SMEM_BYTES_RAW = 1024 + STAGES * STAGE_BYTES + TBL_BYTES + 256;
  static constexpr int SMEM_BYTES = SMEM_BYTES_RAW > kMinSmem ? SMEM_BYTES_RAW : kMinSmem;
  static constexpr uint32_t LAYOUT = ROWB == 64 ? kLayoutSW64 : kLayoutSW128;
  static_assert(O_COL + D <= kTmemCols, "S and O must fit in tensor memory");
  static_assert(NS % 16 == 0, "halo keys must be a multiple of the MMA K step");
  static_assert(Q_BYTES % 1024 == 0 && KV_BYTES % 1024 == 0, "swizzle atoms must stay aligned");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct Params {
  const void* rpb;  // [heads][2KS-1][2KS-1] or nullptr
  void* out;
  int B, heads, H, W;
  int n_tr, n_tc, total_tiles;
  float scale_log2;  // log2(e) / sqrt(d)
  unsigned* status;
};

struct Tile {
  int b, h, i0, j0, r0, c0;
};

template <int KS>
NA_DEVICE Tile decode_tile(int t, const Params& p) {
  Tile tl;
  const int tc = t % p.n_tc;
  int rest = t / p.n_tc;
  const int tr = rest % p.n_tr;
  rest /= p.n_tr;
  tl.b = rest % p.B;
  tl.h = rest / p.B;
  tl.i0 = tr * TH;
  tl.j0 = tc * TW;
  // Halo origin: every window of the tile's queries lies in
  // [r0, r0 + HH) x [c0, c0 + HW); out-of-map parts are zero-filled by TMA.
  tl.r0 = window_start(tl.i0, p.H, KS);
  const int cj = window_start(tl.j0, p.W, KS);
  tl.c0 = min(tl.j0 - KS / 2, cj);
  return tl;
}

template <typename T> NA_DEVICE float to_f(T x);
template <> NA_DEVICE float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <> NA_DEVICE float to_f(__half x) { return __half2float(x); }

template <typename T> NA_DEVICE uint32_t pack2(float lo, float hi);
template <> NA_DEVICE uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <> NA_DEVICE uint32_t pack2<__half>(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <typename T, int KS, int D>
__global__ void __launch_bounds__(kThreads, 1)
na2d_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<KS, D>;
  constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  float* tbl = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::TBL_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar_full = [&](int s) { return smem_addr(bars + s); };
  auto bar_empty = [&](int s) { return smem_addr(bars + C::STAGES + s); };
  const uint32_t bar_s_full = smem_addr(bars + 2 * C::STAGES);
  const uint32_t bar_p_full = smem_addr(bars + 2 * C::STAGES + 1);
  const uint32_t bar_o_full = smem_addr(bars + 2 * C::STAGES + 2);
  auto q_smem = [&](int s) { return sbase + s * C::STAGE_BYTES; };
  auto k_smem = [&](int s) { return sbase + s * C::STAGE_BYTES + C::Q_BYTES; };
  auto v_smem = [&](int s) { return sbase + s * C::STAGE_BYTES + C::Q_BYTES + C::KV_BYTES; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_p_full, 32 * kSoftmaxWarps);
    mbar_init(bar_o_full, 1);
    *abort_flag = 0;
    mbar_init_fence();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int n = 0;
      for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++n) {
        const int s = n % C::STAGES;
        if (!mbar_wait(bar_empty(s), ((n / C::STAGES) & 1) ^ 1, abort_flag, p.status)) break;
        const Tile tl = decode_tile<KS>(t, p);
        mbar_expect_tx(bar_full(s), C::STAGE_BYTES);
        for (int pq = 0; pq < 4; ++pq)
          tma_load_5d(q_smem(s) + pq * PH * PW * C::ROWB, &tm_q, bar_full(s), 0, tl.j0 + (pq & 1) * PW,
                      tl.i0 + (pq >> 1) * PH, tl.h, tl.b);
        tma_load_5d(k_smem(s), &tm_k, bar_full(s), 0, tl.c0, tl.r0, tl.h, tl.b);
        tma_load_5d(v_smem(s), &tm_v, bar_full(s), 0, tl.c0, tl.r0, tl.h, tl.b);
      }
      // drain: every stage's last use must have been released before exit
      for (int e = 0; e < C::STAGES && !*abort_flag; ++e, ++n)
        mbar_wait(bar_empty(n % C::STAGES), ((n / C::STAGES) & 1) ^ 1, abort_flag, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_f16(kBF16, 128, D, true);
      int n = 0;
      for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++n) {
        const int s = n % C::STAGES;
        if (!mbar_wait(bar_full(s), (n / C::STAGES) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        // S = Q . K_halo^T, in chunks of at most 256 keys
#pragma unroll
        for (int n0 = 0; n0 < C::NS; n0 += 256) {
          const int N = C::NS - n0 < 256 ? C::NS - n0 : 256;
          const uint32_t idesc = idesc_f16(kBF16, 128, N, false);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = smem_desc(q_smem(s) + kk * 32, 16, 8 * C::ROWB, C::LAYOUT);
            const uint64_t bd = smem_desc(k_smem(s) + n0 * C::ROWB + kk * 32, 16, 8 * C::ROWB, C::LAYOUT);
            mma_ss(tmem + C::S_COL + n0, ad, bd, idesc, kk > 0);
          }
        }
        mma_commit(bar_s_full);
        if (!mbar_wait(bar_p_full, n & 1, abort_flag, p.status)) break;
        tc_fence_after();
        // O = P . V_halo; P (16-bit, two keys per column) overlays S
#pragma unroll 4
        for (int kk = 0; kk < C::NS / 16; ++kk) {
          const uint64_t bd = smem_desc(v_smem(s) + kk * 16 * C::ROWB, 16, 8 * C::ROWB, C::LAYOUT);
          mma_ts(tmem + C::O_COL, tmem + C::S_COL + kk * 8, bd, idesc_pv, kk > 0);
        }
        mma_commit(bar_o_full);
        mma_commit(bar_empty(s));
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------- softmax and epilogue
    const int wq = warp & 3;  // tensor-memory lane quarter of this warp
    const int pr0 = (wq >> 1) * PH, pc0 = (wq & 1) * PW;
    const int qr = lane / PW, qc = lane % PW;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const int tid = threadIdx.x - 64;  // 0 .. 127
    const float c = p.scale_log2;
    const T* rpb = static_cast<const T*>(p.rpb);
    T* out = static_cast<T*>(p.out);
    int cur_h = -1;
    int n = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++n) {
      const Tile tl = decode_tile<KS>(t, p);
      if (tl.h != cur_h) {
        // (re)build the bias / mask table of this head
        named_barrier(1, 32 * kSoftmaxWarps);
        constexpr int span = 2 * KS - 1;
        for (int idx = tid; idx < C::TBL_ROWS * C::TBL_W; idx += 32 * kSoftmaxWarps) {
          const int row = idx / C::TBL_W, col = idx % C::TBL_W;
          const int blk = col / (KS + C::PAD), off = col % (KS + C::PAD);
          float v = -INFINITY;
          if (row < span && blk < KS && off >= C::PAD) {
            const int bc = blk + (off - C::PAD);
            v = rpb ? to_f(rpb[((size_t)tl.h * span + row) * span + bc]) : 0.f;
          }
          tbl[idx] = v;
        }
        named_barrier(1, 32 * kSoftmaxWarps);
        cur_h = tl.h;
      }
      const int i = tl.i0 + pr0 + qr, j = tl.j0 + pc0 + qc;
      const bool valid = i < p.H && j < p.W;
      const int ic = min(i, p.H - 1), jc = min(j, p.W - 1);
      const int si = window_start(ic, p.H, KS), sj = window_start(jc, p.W, KS);
      const int wr0 = si - tl.r0, wc0 = sj - tl.c0;         // window origin in the halo
      const int er = tl.r0 - ic + KS - 1;                   // bias row of halo row 0
      const int colbase = (sj - jc + KS - 1) * (KS + C::PAD) + C::PAD - wc0;
      const int u_r0 = __reduce_min_sync(0xffffffffu, wr0);
      const int u_r1 = __reduce_max_sync(0xffffffffu, wr0 + KS);
      const int pbeg = __reduce_min_sync(0xffffffffu, wc0) >> 3;
      const int pend = (__reduce_max_sync(0xffffffffu, wc0 + KS) + 7) >> 3;

      if (!mbar_wait(bar_s_full, n & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t srow0 = tmem + lane_base + C::S_COL;

      // pass 1: row maximum of the logits over the window
      float m = -INFINITY;
      for (int hr = u_r0; hr < u_r1; ++hr) {
        uint32_t sv[C::NP][8];
#pragma unroll
        for (int pp = 0; pp < C::NP; ++pp)
          if (pp >= pbeg && pp < pend) tmem_ld8(srow0 + hr * C::HW + pp * 8, sv[pp]);
        tmem_wait_ld();
        const float* trow = tbl + ((unsigned)(hr - wr0) < (unsigned)KS ? hr + er : 2 * KS - 1) * C::TBL_W + colbase;
#pragma unroll
        for (int pp = 0; pp < C::NP; ++pp)
          if (pp >= pbeg && pp < pend) {
#pragma unroll
            for (int e = 0; e < 8; ++e) m = fmaxf(m, __uint_as_float(sv[pp][e]) + trow[pp * 8 + e]);
          }
      }
      const float mc = m * c;

      // pass 2: weights, row sum, P over S (every halo row, zeros outside the union)
      float l = 0.f;
      for (int hr = 0; hr < C::HH; ++hr) {
        uint32_t pk[C::NP][4];
        if (hr >= u_r0 && hr < u_r1) {
          uint32_t sv[C::NP][8];
#pragma unroll
          for (int pp = 0; pp < C::NP; ++pp)
            if (pp >= pbeg && pp < pend) tmem_ld8(srow0 + hr * C::HW + pp * 8, sv[pp]);
          tmem_wait_ld();
          const float* trow =
              tbl + ((unsigned)(hr - wr0) < (unsigned)KS ? hr + er : 2 * KS - 1) * C::TBL_W + colbase;
#pragma unroll
          for (int pp = 0; pp < C::NP; ++pp) {
            if (pp >= pbeg && pp < pend) {
#pragma unroll
              for (int e = 0; e < 8; e += 2) {
                const float x0 = __uint_as_float(sv[pp][e]) + trow[pp * 8 + e];
                const float x1 = __uint_as_float(sv[pp][e + 1]) + trow[pp * 8 + e + 1];
                const float p0 = ex2(fmaf(x0, c, -mc));
                const float p1 = ex2(fmaf(x1, c, -mc));
                l += p0 + p1;
                pk[pp][e >> 1] = pack2<T>(p0, p1);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) pk[pp][e] = 0u;
            }
          }
        } else {
#pragma unroll
          for (int pp = 0; pp < C::NP; ++pp)
#pragma unroll
            for (int e = 0; e < 4; ++e) pk[pp][e] = 0u;
        }
        const uint32_t prow = srow0 + hr * (C::HW / 2);
#pragma unroll
        for (int pp = 0; pp < C::NP; ++pp) tmem_st4(prow + pp * 4, pk[pp]);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_full);

      // epilogue: O / l, rounded to T
      if (!mbar_wait(bar_o_full, n & 1, abort_flag, p.status)) break;
      tc_fence_after();
      uint32_t ov[D];
#pragma unroll
      for (int cc = 0; cc < D; cc += 32) tmem_ld32(tmem + lane_base + C::O_COL + cc, ov + cc);
      tmem_wait_ld();
      if (valid) {
        const float inv = 1.f / l;
        T* dst = out + ((((size_t)tl.b * p.heads + tl.h) * p.H + i) * p.W + j) * D;
#pragma unroll
        for (int x = 0; x < D; x += 8) {
          uint4 w;
          w.x = pack2<T>(__uint_as_float(ov[x + 0]) * inv, __uint_as_float(ov[x + 1]) * inv);
          w.y = pack2<T>(__uint_as_float(ov[x + 2]) * inv, __uint_as_float(ov[x + 3]) * inv);
          w.z = pack2<T>(__uint_as_float(ov[x + 4]) * inv, __uint_as_float(ov[x + 5]) * inv);
          w.w = pack2<T>(__uint_as_float(ov[x + 6]) * inv, __uint_as_float(ov[x + 7]) * inv);
          *reinterpret_cast<uint4*>(dst + x) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// [B][heads][H][W][d] as a 5-D map with a box of (d, bw, bh, 1, 1).
bool make_map(CUtensorMap* m, const void* base, const Shape& s, bool bf16, int bw, int bh) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t es = 2;
  cuuint64_t dims[5] = {(cuuint64_t)s.d, (cuuint64_t)s.W, (cuuint64_t)s.H, (cuuint64_t)s.heads, (cuuint64_t)s.B};
  cuuint64_t strides[4] = {s.d * es, (cuuint64_t)s.W * s.d * es, (cuuint64_t)s.H * s.W * s.d * es,
                           (cuuint64_t)s.heads * s.H * s.W * s.d * es};
  cuuint32_t box[5] = {(cuuint32_t)s.d, (cuuint32_t)bw, (cuuint32_t)bh, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   s.d == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  static int counts[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!counts[dev]) cudaDeviceGetAttribute(&counts[dev], cudaDevAttrMultiProcessorCount, dev);
  return counts[dev];
}

template <typename T, int KS, int D>
cudaError_t launch(const void* q, const void* k, const void* v, const void* rpb, void* out, const Shape& s,
                   unsigned* status, cudaStream_t st) {
  using C = Cfg<KS, D>;
  constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, s, bf16, PW, PH) || !make_map(&mk, k, s, bf16, C::HW, C::HH) ||
      !make_map(&mv, v, s, bf16, C::HW, C::HH))
    return cudaErrorInvalidValue;
  auto kern = na2d_fwd_tc_kernel<T, KS, D>;
  static std::mutex mu;
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_set[dev]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  Params p;
  p.rpb = rpb;
  p.out = out;
  p.B = s.B;
  p.heads = s.heads;
  p.H = s.H;
  p.W = s.W;
  p.n_tr = (s.H + TH - 1) / TH;
  p.n_tc = (s.W + TW - 1) / TW;
  const long long tiles = (long long)p.n_tr * p.n_tc * s.B * s.heads;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  p.total_tiles = (int)tiles;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s.d));
  p.status = status;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = p.total_tiles < sms ? p.total_tiles : sms;
  kern<<<grid, kThreads, C::SMEM_BYTES, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_ks(const void* q, const void* k, const void* v, const void* rpb, void* out, const Shape& s,
                      unsigned* status, cudaStream_t st) {
  switch (s.ks) {
    case 3: return launch<T, 3, D>(q, k, v, rpb, out, s, status, st);
    case 5: return launch<T, 5, D>(q, k, v, rpb, out, s, status, st);
    case 7: return launch<T, 7, D>(q, k, v, rpb, out, s, status, st);
    case 9: return launch<T, 9, D>(q, k, v, rpb, out, s, status, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool forward_tc_supported(const Shape& s, na_dtype dt) {
  if (dt != NA_F16 && dt != NA_BF16) return false;
  if (s.d != 32 && s.d != 64) return false;
  if (s.ks != 3 && s.ks != 5 && s.ks != 7 && s.ks != 9) return false;
  return true;
}

cudaError_t launch_forward_tc(const void* q, const void* k, const void* v, const void* rpb, void* out,
                              const Shape& s, na_dtype dt, unsigned* status, cudaStream_t st) {
  if (!forward_tc_supported(s, dt)) return cudaErrorInvalidValue;
  if (dt == NA_BF16)
    return s.d == 32 ? launch_ks<__nv_bfloat16, 32>(q, k, v, rpb, out, s, status, st)
                     : launch_ks<__nv_bfloat16, 64>(q, k, v, rpb, out, s, status, st);
  return s.d == 32 ? launch_ks<__half, 32>(q, k, v, rpb, out, s, status, st)
                   : launch_ks<__half, 64>(q, k, v, rpb, out, s, status, st);
}

}  // namespace na2d
