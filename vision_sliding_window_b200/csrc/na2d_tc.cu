// na2d_tc.cu -- tensor-core fused forward of 2D Neighborhood Attention for
// fp16 / bf16 on sm_100a (Neighborhood Attention Transformer, Sec. 3.1,
// Eqs. (2)-(4)).  The data movement follows the "tiled NA" idea of Sec. 3.2
// and App. A.4 -- a query tile plus the key/value halo its windows cover,
// staged in shared memory -- re-planned for TMA, tcgen05 and tensor memory.
//
// Work unit: a "pair" of 8x8 query tiles stacked vertically (16 x 8
// queries), one M = 128 MMA: tile A's queries are tensor-memory lanes 0-15
// of every 32-lane quarter, tile B's lanes 16-31.  The query operand is
// block-structured (tile A's queries in K block 0, tile B's in K block 1),
// so each tile's S row is taken against its own halo: the pair's K and V
// halo -- (16+k-1) rows x (8+k-1, rounded up to 8) columns -- is one TMA
// box each, and tile B's halo starts rB rows further down inside the same
// buffer.  Two single tiles of a map's last tile row share a pair that way.
//
// Roles of one persistent CTA per SM:
//   warp 0          TMA producer of the Q/K ring (query tiles, K halo)
//   warp 3          TMA producer of the V ring
//   warps 1..NBUF   one MMA issuer each, for its own tensor-memory buffer
//                   (warp 1 also allocates and frees tensor memory)
//   warpgroups 1..NBUF  softmax groups: group g owns buffer g and every
//                   NBUF-th pair of the CTA
//   last warpgroup  the epilogue of every pair, in order
// Per pair:  S = Q K_halo^T (fp32, tensor memory) -> each softmax warp reads
// the union of the windows of its two 4x4 patches (one per tile), adds the
// bias and the -inf mask from a per-head 16-bit table, keeps x = s + bias in
// place, takes the row maximum, then writes P = exp2((x - max) log2e /
// sqrt(d)) in 16 bits over S (zeros outside the union) -> O = P V_halo, in
// the dead columns of S -> O / rowsum, rounded, stored by the epilogue.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>
#include <type_traits>

#include "na2d_common.cuh"
#include "na2d_internal.h"
#include "na2d_sm100.cuh"

namespace na2d {
namespace {

using namespace sm100;

constexpr int TT = 8;  // 8 x 8 query tile
constexpr int PQ = 4;  // 4 x 4 patch: the 16 lanes of one tile a softmax warp owns
constexpr int kTmemCols = 512;
constexpr int kMaxSmem = 227 * 1024;
constexpr int kMinSmem = 116 * 1024;  // one CTA per SM: it holds all of tensor memory

__host__ __device__ constexpr int round_up(int x, int a) { return (x + a - 1) / a * a; }

template <int KS, int D>
struct Cfg {
  static constexpr int HH = TT + KS - 1;               // halo rows of one tile
  static constexpr int HHP = 2 * TT + KS - 1;          // halo rows of the pair buffer
  static constexpr int HS = TT + KS / 2;               // halo rows of a bottom single tile
  static_assert(2 * HS == HHP, "two single-tile halos fill a pair buffer");
  static constexpr int HW = round_up(TT + KS - 1, 8);  // halo columns
  static constexpr int NS = HH * HW;                   // keys of one tile = S columns
  static constexpr int NPC = HW / 4;                   // 4-key pieces per halo row
  static constexpr int NPU = (PQ - 1 + KS + 3) / 4;    // pieces of an interior patch's window union
  static constexpr int ROWB = 2 * D;                   // bytes per key / query row
  static constexpr int QBLK = 2 * TT * TT * ROWB;      // one K block of the query operand (128 rows)
  static constexpr int Q_BYTES = 2 * QBLK;
  static constexpr int KV_BYTES = HHP * HW * ROWB;
  static constexpr int QK_BYTES = Q_BYTES + KV_BYTES;  // one stage of the Q/K ring
  // tensor memory: per buffer S (NS columns); P (16-bit) overlays its first
  // NS/2 columns; O (2d columns: tile A's d, then tile B's d) sits in the
  // dead part of S after P.
  static constexpr int NBUF = NS <= kTmemCols / 2 ? 2 : 1;
  static constexpr int BUF_COLS = kTmemCols / NBUF;
  static constexpr int PO = round_up(NS / 2, 32);
  static constexpr int s_col(int b) { return b * BUF_COLS; }
  static constexpr int o_col(int b) { return b * BUF_COLS + PO; }
  // bias / mask table (one per softmax group), 16-bit entries of the input
  // type, exactly the bias values given: rows 0..2KS-2 hold bias rows, row
  // 2KS-1 is all -inf.  A row is KS blocks of stride KS+PAD; block dc holds
  // the bias row's columns dc..dc+KS-1 after PAD entries of -inf, and its
  // tail is the next block's -inf head.  PAD covers a whole halo row around
  // any window.
  static constexpr int PAD = HW - KS;
  static constexpr int TBL_W0 = KS * (KS + PAD) + PAD;
  static constexpr int TBL_W = TBL_W0 + ((4 - TBL_W0 % 64) + 64) % 64;  // = 4 mod 64 entries
  static constexpr int TBL_ROWS = 2 * KS;
  static constexpr int TBL_N = TBL_ROWS * TBL_W;  // entries of one copy
  static_assert(TBL_W % 4 == 0 && TBL_N % 4 == 0, "table rows keep a column's offset mod 4");
  // Copies of the table, copy q shifted left by q entries: every lane reads
  // its entries 4 at a time with 8-byte loads (2 at a time with 4-byte loads
  // when only two copies are kept) from the copy that makes them aligned.
  // Copy q starts tbl_off(q) entries past a 64-entry boundary: offsets that
  // spread the 16 lanes of a tile over distinct banks for the softmax's
  // lane-to-query layout.  Four copies are kept where they cost no stage.
  static constexpr int TBL_CS = round_up(TBL_N, 64);
  static constexpr int tbl_off(int q) { return q == 0 ? 0 : q == 1 ? 16 : KS % 4 == 1 ? 16 * q : 16 * q + 4; }
  static constexpr int tbl_base(int q) { return q * TBL_CS + tbl_off(q); }
  static constexpr int tbl_bytes(int copies) { return round_up((tbl_base(copies - 1) + TBL_N) * 2, 16); }
  static constexpr int RAW = (2 * KS - 1) * (2 * KS - 1);  // one head's bias table
  static constexpr int RAW_BYTES = round_up(RAW * 2, 16);
  static constexpr int LSUM_BYTES = 2 * 128 * 4;  // row sums handed to the epilogue, per buffer and use parity
  // A stage holds Q, K and V.  Where not even one such stage fits (large k
  // with d = 64), V is loaded into the K slot once S = Q K^T has read K
  // (KV_ALIAS): a stage is then Q and one K-or-V slot.
  static constexpr int FULL_STAGE = QK_BYTES + KV_BYTES;
  static constexpr bool KV_ALIAS =
      (kMaxSmem - (1024 + NBUF * (tbl_bytes(2) + RAW_BYTES + LSUM_BYTES) + 512)) / FULL_STAGE < 1;
  static constexpr int STAGE_BYTES = KV_ALIAS ? QK_BYTES : FULL_STAGE;
  static constexpr int stages_with(int copies) {
    return (kMaxSmem - (1024 + NBUF * (tbl_bytes(copies) + RAW_BYTES + LSUM_BYTES) + 512)) / STAGE_BYTES;
  }
  static constexpr int TBL_COPIES = (stages_with(4) >= 3 || stages_with(4) == stages_with(2)) ? 4 : 2;
  static constexpr int TBL_BYTES = tbl_bytes(TBL_COPIES);
  static constexpr int FIXED = 1024 + NBUF * (TBL_BYTES + RAW_BYTES + LSUM_BYTES) + 512;  // + barriers, TMEM slot
  static constexpr int STAGES_FIT = (kMaxSmem - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT >= 3 ? 3 : STAGES_FIT;
  static constexpr int SMEM_RAW = FIXED + STAGES * STAGE_BYTES;
  static constexpr int SMEM_BYTES = SMEM_RAW > kMinSmem ? SMEM_RAW : kMinSmem;
  // Warpgroup 0: TMA producers (warps 0 and 3) and MMA issuers (warps
  // 1..NBUF); warpgroups 1..NBUF: softmax groups, one per buffer; the last
  // warpgroup: the epilogue of every pair.  The register file is re-split at
  // run time (setmaxnreg) within what the CTA is launched with.
  static constexpr int THREADS = 128 * (2 + NBUF);
  static constexpr int LAUNCH_REGS = NBUF == 2 ? 128 : 168;  // 65536 / THREADS in steps of 8
  static constexpr bool kWideCtrl = D == 64 && KS > 9;
  static constexpr int REGS_CTRL = NBUF == 2 ? 64 : (kWideCtrl ? 80 : 72);
  static constexpr int REGS_EPI = NBUF == 2 ? 56 : 80;
  static constexpr int REGS_SOFTMAX = NBUF == 2 ? 192 : 232;
  static_assert(REGS_CTRL * 128 + REGS_EPI * 128 + REGS_SOFTMAX * 128 * NBUF <= LAUNCH_REGS * THREADS,
                "the register split must fit the launch allocation");
  static constexpr uint32_t LAYOUT = ROWB == 64 ? kLayoutSW64 : kLayoutSW128;
  static_assert(NS <= BUF_COLS && PO + 2 * D <= BUF_COLS, "S, P and O of a buffer must fit in tensor memory");
  static_assert(STAGES >= 1, "a pipeline stage must fit in shared memory");
  static_assert(NS % 16 == 0, "halo keys must be a multiple of the MMA K step");
  static_assert(QBLK % 1024 == 0 && KV_BYTES % 1024 == 0 && (TT * HW * ROWB) % 1024 == 0,
                "swizzle atoms must stay aligned");
  static_assert(SMEM_BYTES <= kMaxSmem, "shared memory");
};

// Division by a divisor fixed at launch: q = (umulhi(n, m) + n) >> s for
// 0 <= n < 2^31, with s = ceil(log2 d) and m = ceil(2^(32+s) / d) - 2^32.
struct FastDiv {
  uint32_t d, m, s;
  FastDiv() = default;
  explicit FastDiv(uint32_t div) : d(div), m(0), s(0) {
    while ((1ull << s) < div) ++s;
    m = (uint32_t)((((1ull << (32 + s)) + div - 1) / div) - (1ull << 32));
  }
  NA_DEVICE int div(int n) const { return (int)((__umulhi((uint32_t)n, m) + (uint32_t)n) >> s); }
};

// Work units.  A map's rows are cut into pairs of 8x8 tiles stacked
// vertically (16 rows).  Where the last tile row of a map is a single tile
// (1 to 8 rows left over), that tile's clamped halo is only TT + KS/2 rows,
// so two such single tiles -- of the same head, any maps and columns --
// share one pair: each gets its own halo box, tile A's in buffer rows
// [0, HS) and tile B's in [HHP - HS, HHP), which fill the pair's buffer
// exactly.  Per head: the full pairs (column fastest, then pair row, then
// batch), then the packed pairs of single tiles in (batch, column) order.
// Unit t is pair t / heads of head t % heads: with the head fastest, the
// pairs a softmax group takes (2 x gridDim apart) keep one head, and its
// bias table, whenever the head count divides 2 x gridDim.
struct Params {
  const void* rpb;  // [heads][2KS-1][2KS-1] or nullptr
  void* out;
  int B, heads, H, W;
  int n_pc, n_fpr;                   // tile columns; full pair rows per map
  int full_per_head, singles_per_head, per_head, total;
  FastDiv div_head, div_pc, div_fpr;
  float scale_log2;       // log2(e) / sqrt(d)
  unsigned* status;
};

// One work unit: per tile t (0 = A, TMEM lanes 0-15 of each quarter; 1 = B,
// lanes 16-31) the map b[t], first query row i0[t] and column j0[t], the
// halo box origin (R0[t], c0[t]) and rt[t], the map row of the tile's
// S-space row 0.  Tile B's S-space starts rB buffer rows into the halo.
struct Pair {
  int h;
  bool packed, has_b;
  int b[2], i0[2], j0[2], c0[2], R0[2], rt[2];
  int rB;
};

template <int KS>
NA_DEVICE Pair decode_pair(int t, const Params& p) {
  constexpr int HHP = 2 * TT + KS - 1, HS = TT + KS / 2;
  Pair q;
  const int r = p.div_head.div(t);  // the head varies fastest
  q.h = t - r * p.heads;
  if (r < p.full_per_head) {
    const int rr = p.div_pc.div(r);
    const int pc = r - rr * p.n_pc;
    const int b = p.div_fpr.div(rr);
    const int pr = rr - b * p.n_fpr;
    q.packed = false;
    q.has_b = true;
    q.b[0] = q.b[1] = b;
    q.i0[0] = pr * 2 * TT;
    q.i0[1] = q.i0[0] + TT;
    q.j0[0] = q.j0[1] = pc * TT;
    q.R0[0] = q.R0[1] = window_start(q.i0[0], p.H, KS);
    q.c0[0] = q.c0[1] = min(q.j0[0] - KS / 2, window_start(q.j0[0], p.W, KS));
    q.rB = window_start(min(q.i0[1], p.H - 1), p.H, KS) - q.R0[0];  // 0 .. 8
    q.rt[0] = q.R0[0];
    q.rt[1] = q.R0[0] + q.rB;
  } else {
    const int u = r - p.full_per_head;
    q.packed = true;
    q.has_b = 2 * u + 1 < p.singles_per_head;
#pragma unroll
    for (int tl = 0; tl < 2; ++tl) {
      const int sidx = q.has_b ? 2 * u + tl : 2 * u;  // a missing tile B repeats tile A
      const int b = p.div_pc.div(sidx);
      const int pc = sidx - b * p.n_pc;
      q.b[tl] = b;
      q.i0[tl] = p.n_fpr * 2 * TT;
      q.j0[tl] = pc * TT;
      q.R0[tl] = window_start(q.i0[tl], p.H, KS);
      q.c0[tl] = min(q.j0[tl] - KS / 2, window_start(q.j0[tl], p.W, KS));
    }
    q.rB = TT;
    q.rt[0] = q.R0[0];
    q.rt[1] = q.R0[1] - (HHP - HS - TT);
  }
  return q;
}

template <typename T> NA_DEVICE uint32_t pack2(float lo, float hi);
template <> NA_DEVICE uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <> NA_DEVICE uint32_t pack2<__half>(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Stores N (a multiple of 4) consecutive 32-bit columns from registers.
template <int N>
NA_DEVICE void tmem_st_row(uint32_t taddr, const uint32_t (&r)[N]) {
  static_assert(N % 4 == 0, "row stores go by 4 columns");
#pragma unroll
  for (int c = 0; c < N; c += 4) {
    const uint32_t v[4] = {r[c], r[c + 1], r[c + 2], r[c + 3]};
    tmem_st4(taddr + c, v);
  }
}

// Largest access width (4, 8 or 16 columns) that a start column known to be
// a multiple of `align` allows; every tensor-memory access starts at a
// multiple of its own width.
__host__ __device__ constexpr int span_width(int align) { return align % 16 == 0 ? 16 : align % 8 == 0 ? 8 : 4; }
__host__ __device__ constexpr int low_pow2(int x) { return x & -x; }

// N consecutive 32-bit columns starting at a column that is a multiple of A.
template <int N, int A>
NA_DEVICE void ld_span(uint32_t addr, uint32_t* v) {
  static_assert(N % 4 == 0 && A % 4 == 0, "spans go by 4 columns");
  constexpr int W = span_width(A) < span_width(N) ? span_width(A) : span_width(N);  // divides N and A
#pragma unroll
  for (int c = 0; c < N; c += W) {
    if constexpr (W == 16) tmem_ld16(addr + c, *reinterpret_cast<uint32_t(*)[16]>(v + c));
    else if constexpr (W == 8) tmem_ld8(addr + c, *reinterpret_cast<uint32_t(*)[8]>(v + c));
    else tmem_ld4(addr + c, *reinterpret_cast<uint32_t(*)[4]>(v + c));
  }
}
template <int N, int A>
NA_DEVICE void st_span(uint32_t addr, const uint32_t* v) {
  static_assert(N % 4 == 0 && A % 4 == 0, "spans go by 4 columns");
  constexpr int W = span_width(A) < span_width(N) ? span_width(A) : span_width(N);  // divides N and A
#pragma unroll
  for (int c = 0; c < N; c += W) {
    if constexpr (W == 16) tmem_st16(addr + c, v + c);
    else if constexpr (W == 8) tmem_st8(addr + c, v + c);
    else tmem_st4(addr + c, *reinterpret_cast<const uint32_t(*)[4]>(v + c));
  }
}

// exp2 of a float pair, rounded to T: two results per MUFU operation.  The
// exponent argument is rounded to T first; for bf16 that adds at most about
// 0.3% relative error to each weight, inside the bf16 rounding of P itself.
template <typename T> NA_DEVICE uint32_t exp2_pair(float a0, float a1);
template <> NA_DEVICE uint32_t exp2_pair<__nv_bfloat16>(float a0, float a1) {
  return ex2_bf16x2(pack2<__nv_bfloat16>(a0, a1));
}
template <> NA_DEVICE uint32_t exp2_pair<__half>(float a0, float a1) { return ex2_f16x2(pack2<__half>(a0, a1)); }
// s0 += low half of w, s1 += high half, each taken exactly as a float (one
// mixed-precision add per element, no unpacking).
template <typename T> NA_DEVICE void acc_pair(float& s0, float& s1, uint32_t w);
template <> NA_DEVICE void acc_pair<__nv_bfloat16>(float& s0, float& s1, uint32_t w) {
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n add.rn.f32.bf16 %0, lo, %0;\n add.rn.f32.bf16 %1, hi, %1;\n}"
      : "+f"(s0), "+f"(s1)
      : "r"(w));
}
template <> NA_DEVICE void acc_pair<__half>(float& s0, float& s1, uint32_t w) {
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n add.rn.f32.f16 %0, lo, %0;\n add.rn.f32.f16 %1, hi, %1;\n}"
      : "+f"(s0), "+f"(s1)
      : "r"(w));
}

// d0 = s0 + low half of w, d1 = s1 + high half, each half taken exactly as
// a float (mixed-precision adds, no unpacking).
template <typename T> NA_DEVICE void add_pair(float& d0, float& d1, float s0, float s1, uint32_t w);
template <> NA_DEVICE void add_pair<__nv_bfloat16>(float& d0, float& d1, float s0, float s1, uint32_t w) {
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n add.rn.f32.bf16 %0, lo, %3;\n add.rn.f32.bf16 %1, hi, %4;\n}"
      : "=f"(d0), "=f"(d1)
      : "r"(w), "f"(s0), "f"(s1));
}
template <> NA_DEVICE void add_pair<__half>(float& d0, float& d1, float s0, float s1, uint32_t w) {
  asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n add.rn.f32.f16 %0, lo, %3;\n add.rn.f32.f16 %1, hi, %4;\n}"
      : "=f"(d0), "=f"(d1)
      : "r"(w), "f"(s0), "f"(s1));
}
NA_DEVICE uint32_t bits16(__nv_bfloat16 x) { return __bfloat16_as_ushort(x); }
NA_DEVICE uint32_t bits16(__half x) { return __half_as_ushort(x); }
template <typename T> NA_DEVICE T neg_inf();
template <> NA_DEVICE __nv_bfloat16 neg_inf() { return __ushort_as_bfloat16((unsigned short)0xff80u); }
template <> NA_DEVICE __half neg_inf() { return __ushort_as_half((unsigned short)0xfc00u); }

// Arrives on `bar` once for the whole warp, after every lane's earlier
// memory operations: the barrier counts warps, not threads, which keeps
// shared-memory atomics off the hot path.
NA_DEVICE void warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// A bounded meeting point of a fixed set of warps: an mbarrier that each
// arrives on once per meeting, then waits for (with the kernel's time limit
// and abort flag), so no thread can be left waiting by one that gave up.
struct Meeting {
  uint32_t bar;
  uint32_t phase;
  volatile int* abort_flag;
  unsigned* status;
  NA_DEVICE bool sync() {
    warp_arrive(bar);
    const bool ok = mbar_wait(bar, phase, abort_flag, status);
    phase ^= 1;
    return ok;
  }
};

// Softmax of one warp's 32 queries (two 4x4 patches, one per tile) over the
// union rows [u_r0, u_r1) and pieces [PB, PB+NU) of their windows, RB rows
// at a time: each batch's tensor-memory loads are issued together and the RB
// rows are independent streams of arithmetic.  Pass 1 writes
// y = s + table (the bias, -inf outside the window) back over S and takes
// the row maximum m; pass 2 writes P = exp2((y - m) log2e/sqrt(d)) as
// 16-bit pairs over S -- P row hr covers the S columns of row hr / 2, read by
// an earlier or the same batch -- zeros outside the pieces, and returns the
// sum of the rounded P.  Rows past u_r1 in the last batch repeat row u_r1-1:
// they store the same values again and are left out of the sum.
template <typename T, int KS, int D, int PB, int NU>
NA_DEVICE float softmax_rows(uint32_t sbuf, const T* tl, int u_r0, int u_r1, int wr0, int er, float c) {
  using C = Cfg<KS, D>;
  constexpr int HW = C::HW, PW = HW / 2, NV = NU * 4, RB = 2;
  // start-column alignment of a piece window (row hr * HW + PB * 4) and of a P row (hr * PW)
  constexpr int AS = PB == 0 ? low_pow2(HW) : (low_pow2(HW) < low_pow2(PB * 4) ? low_pow2(HW) : low_pow2(PB * 4));
  constexpr int AP = low_pow2(PW);
  const int last = u_r1 - 1;
  float mx[RB];
#pragma unroll
  for (int j = 0; j < RB; ++j) mx[j] = -INFINITY;
#pragma unroll 1
  for (int r0 = u_r0; r0 < u_r1; r0 += RB) {
    uint32_t v[RB][NV];
#pragma unroll
    for (int j = 0; j < RB; ++j) ld_span<NV, AS>(sbuf + min(r0 + j, last) * HW + PB * 4, v[j]);
#pragma unroll
    for (int j = 0; j < RB; ++j) tmem_wait_ld_regs(v[j]);
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      const int hr = min(r0 + j, last);
      const T* tr = tl + ((unsigned)(hr - wr0) < (unsigned)KS ? hr + er : 2 * KS - 1) * C::TBL_W + PB * 4;
#pragma unroll
      for (int e = 0; e < NV; e += 4) {
        uint32_t b01, b23;  // entries e, e+1 and e+2, e+3
        if constexpr (C::TBL_COPIES == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(tr + e);
          b01 = w.x;
          b23 = w.y;
        } else {
          b01 = *reinterpret_cast<const uint32_t*>(tr + e);
          b23 = *reinterpret_cast<const uint32_t*>(tr + e + 2);
        }
        float y0, y1, y2, y3;
        add_pair<T>(y0, y1, __uint_as_float(v[j][e]), __uint_as_float(v[j][e + 1]), b01);
        add_pair<T>(y2, y3, __uint_as_float(v[j][e + 2]), __uint_as_float(v[j][e + 3]), b23);
        mx[j] = max3(mx[j], max3(y0, y1, y2), y3);
        v[j][e] = __float_as_uint(y0);
        v[j][e + 1] = __float_as_uint(y1);
        v[j][e + 2] = __float_as_uint(y2);
        v[j][e + 3] = __float_as_uint(y3);
      }
      st_span<NV, AS>(sbuf + hr * HW + PB * 4, v[j]);
    }
  }
  tmem_wait_st();
  float m = mx[0];
#pragma unroll
  for (int j = 1; j < RB; ++j) m = fmaxf(m, mx[j]);
  const float cm = -c * m;

  uint32_t z[PW];
#pragma unroll
  for (int e = 0; e < PW; ++e) z[e] = 0u;
#pragma unroll 1
  for (int hr = 0; hr < u_r0; ++hr) st_span<PW, AP>(sbuf + hr * PW, z);
  float l = 0.f;
#pragma unroll 1
  for (int r0 = u_r0; r0 < u_r1; r0 += RB) {
    uint32_t v[RB][NV];
#pragma unroll
    for (int j = 0; j < RB; ++j) ld_span<NV, AS>(sbuf + min(r0 + j, last) * HW + PB * 4, v[j]);
#pragma unroll
    for (int j = 0; j < RB; ++j) tmem_wait_ld_regs(v[j]);
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      uint32_t pk[PW];
#pragma unroll
      for (int e = 0; e < PW; ++e) pk[e] = 0u;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int e = 0; e < NV; e += 4) {
        float a0, a1, a2, a3;
        fma2(a0, a1, __uint_as_float(v[j][e]), __uint_as_float(v[j][e + 1]), c, c, cm, cm);
        fma2(a2, a3, __uint_as_float(v[j][e + 2]), __uint_as_float(v[j][e + 3]), c, c, cm, cm);
        const uint32_t pa = exp2_pair<T>(a0, a1), pb = exp2_pair<T>(a2, a3);
        acc_pair<T>(s0, s1, pa);
        acc_pair<T>(s0, s1, pb);
        pk[PB * 2 + e / 2] = pa;
        pk[PB * 2 + e / 2 + 1] = pb;
      }
      st_span<PW, AP>(sbuf + min(r0 + j, last) * PW, pk);
      if (r0 + j < u_r1) l += s0 + s1;
    }
  }
#pragma unroll 1
  for (int hr = u_r1; hr < C::HH; ++hr) st_span<PW, AP>(sbuf + hr * PW, z);
  return l;
}

// Runs softmax_rows over the pieces [pb, pb + NPU) of an interior patch's
// window union, fixed at compile time, or over whole rows when the union is
// wider (patches at the map border).
template <typename T, int KS, int D, int PB = 0>
NA_DEVICE float softmax_dispatch(int pb, int pe, uint32_t sbuf, const T* tl, int u_r0, int u_r1, int wr0,
                                 int er, float c) {
  using C = Cfg<KS, D>;
  if constexpr (PB + C::NPU <= C::NPC) {
    if (pe - pb <= C::NPU && min(pb, C::NPC - C::NPU) == PB)
      return softmax_rows<T, KS, D, PB, C::NPU>(sbuf, tl, u_r0, u_r1, wr0, er, c);
    return softmax_dispatch<T, KS, D, PB + 1>(pb, pe, sbuf, tl, u_r0, u_r1, wr0, er, c);
  } else {
    return softmax_rows<T, KS, D, 0, C::NPC>(sbuf, tl, u_r0, u_r1, wr0, er, c);
  }
}

template <typename T, int KS, int D>
__global__ void __launch_bounds__(Cfg<KS, D>::THREADS, 1)
na2d_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k1,
                   const __grid_constant__ CUtensorMap tm_v1, const Params p) {
  using C = Cfg<KS, D>;
  constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int NB = C::NBUF, ST = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  T* tables = reinterpret_cast<T*>(smem + ST * C::STAGE_BYTES);
  T* raws = reinterpret_cast<T*>(smem + ST * C::STAGE_BYTES + NB * C::TBL_BYTES);
  float* lsums = reinterpret_cast<float*>(smem + ST * C::STAGE_BYTES + NB * (C::TBL_BYTES + C::RAW_BYTES));
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(smem + ST * C::STAGE_BYTES + NB * (C::TBL_BYTES + C::RAW_BYTES + C::LSUM_BYTES));
  // Two shared-memory rings of ST stages: Q and K (released when S = Q K^T
  // has read them) and V (released when P.V has read it), each fed by its
  // own producer thread, so the next pairs' Q and K arrive while this
  // pair's softmax runs.
  // barrier slots: kfull[ST][NB] vfull[ST][NB] kempty[ST] vempty[ST]
  //                s_full[NB] p_full[NB] o_full[NB] o_empty[NB].
  // A stage's "full" barriers are split by buffer: each is waited on by one
  // issuer only, one phase per use, so a parity wait can never see a phase
  // of a pair that belongs to the other buffer.  Pair n uses
  // kfull[n % ST][n % NB] and vfull[n % ST][n % NB] for the (n / LCM)-th time.
  constexpr int LCM = (ST % NB == 0) ? ST : ST * NB;
  constexpr int B0 = 2 * ST * NB + 2 * ST;
  // then: the table meeting of each softmax group [NB]
  // and l_full [NB][2]: row sums of a buffer's use posted for the epilogue,
  // one barrier per use parity (a group may run one use ahead of the epilogue)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B0 + 7 * NB);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_addr(bars + i); };
  auto bar_kfull = [&](int n) { return bar((n % ST) * NB + n % NB); };
  auto bar_vfull = [&](int n) { return bar(ST * NB + (n % ST) * NB + n % NB); };
  auto bar_kempty = [&](int s) { return bar(2 * ST * NB + s); };
  auto bar_vempty = [&](int s) { return bar(2 * ST * NB + ST + s); };
  auto bar_s_full = [&](int b) { return bar(B0 + b); };
  auto bar_p_full = [&](int b) { return bar(B0 + NB + b); };
  auto bar_o_full = [&](int b) { return bar(B0 + 2 * NB + b); };
  auto bar_o_empty = [&](int b) { return bar(B0 + 3 * NB + b); };
  auto bar_tbl = [&](int g) { return bar(B0 + 4 * NB + g); };
  auto bar_l_full = [&](int b, int par) { return bar(B0 + 5 * NB + 2 * b + par); };
  auto q_smem = [&](int s) { return sbase + s * C::QK_BYTES; };
  auto k_smem = [&](int s) { return sbase + s * C::QK_BYTES + C::Q_BYTES; };
  auto v_smem = [&](int s) { return C::KV_ALIAS ? k_smem(s) : sbase + ST * C::QK_BYTES + s * C::KV_BYTES; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The query operand of S = Q K^T is block structured: K block 0 holds
  // tile A's queries (TMEM lanes 0-15 of every quarter), K block 1 tile B's
  // (lanes 16-31); the other rows of each block stay zero.
  for (int s = 0; s < ST; ++s)
    for (int i = threadIdx.x; i < C::Q_BYTES / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(smem + s * C::QK_BYTES)[i] = make_uint4(0u, 0u, 0u, 0u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * ST * NB + 2 * ST; ++i) mbar_init(bar(i), 1);
    for (int b = 0; b < NB; ++b) {
      mbar_init(bar_s_full(b), 1);
      mbar_init(bar_p_full(b), 4);  // barriers a warpgroup meets count its 4 warps
      mbar_init(bar_o_full(b), 1);
      mbar_init(bar_o_empty(b), 4);
    }
    for (int g = 0; g < NB; ++g) mbar_init(bar_tbl(g), 4);
    for (int i = 0; i < 2 * NB; ++i) mbar_init(bar_l_full(i >> 1, i & 1), 4);
    *abort_flag = 0;
    mbar_init_fence();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_k1);
    tma_prefetch_desc(&tm_v1);
  }
  if (warp == 1) tmem_alloc(smem_addr(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
  regs_dec<C::REGS_CTRL>();
  if (warp == 0 || warp == 3) {
    // ------------------------------------- TMA producers (Q/K ring; V ring)
    const bool qk = warp == 0;
    if (lane == 0) {
      int n = 0;
      for (int t = blockIdx.x; t < p.total; t += gridDim.x, ++n) {
        const int s = n % ST;
        bool ok;
        if constexpr (C::KV_ALIAS)  // Q/K: the slot's previous V is consumed; V: this pair's K is
          ok = qk ? mbar_wait(bar_vempty(s), ((n / ST) & 1) ^ 1, abort_flag, p.status)
                  : mbar_wait(bar_kempty(s), (n / ST) & 1, abort_flag, p.status);
        else
          ok = mbar_wait(qk ? bar_kempty(s) : bar_vempty(s), ((n / ST) & 1) ^ 1, abort_flag, p.status);
        if (!ok) break;
        const Pair pr = decode_pair<KS>(t, p);
        if (qk) {
          const uint32_t full = bar_kfull(n);
          mbar_expect_tx(full, C::Q_BYTES / 2 + C::KV_BYTES);
#pragma unroll
          for (int tile = 0; tile < 2; ++tile)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              tma_load_5d(q_smem(s) + tile * C::QBLK + (32 * q + 16 * tile) * C::ROWB, &tm_q, full, 0,
                          pr.j0[tile] + (q & 1) * PQ, pr.i0[tile] + (q >> 1) * PQ, pr.h, pr.b[tile]);
          if (pr.packed) {
            tma_load_5d(k_smem(s), &tm_k1, full, 0, pr.c0[0], pr.R0[0], pr.h, pr.b[0]);
            tma_load_5d(k_smem(s) + (C::HHP - C::HS) * C::HW * C::ROWB, &tm_k1, full, 0, pr.c0[1], pr.R0[1],
                        pr.h, pr.b[1]);
          } else {
            tma_load_5d(k_smem(s), &tm_k, full, 0, pr.c0[0], pr.R0[0], pr.h, pr.b[0]);
          }
        } else {
          const uint32_t full = bar_vfull(n);
          mbar_expect_tx(full, C::KV_BYTES);
          if (pr.packed) {
            tma_load_5d(v_smem(s), &tm_v1, full, 0, pr.c0[0], pr.R0[0], pr.h, pr.b[0]);
            tma_load_5d(v_smem(s) + (C::HHP - C::HS) * C::HW * C::ROWB, &tm_v1, full, 0, pr.c0[1], pr.R0[1],
                        pr.h, pr.b[1]);
          } else {
            tma_load_5d(v_smem(s), &tm_v, full, 0, pr.c0[0], pr.R0[0], pr.h, pr.b[0]);
          }
        }
      }
      for (int e = 0; e < ST && !*abort_flag; ++e, ++n)
        mbar_wait((qk != C::KV_ALIAS) ? bar_kempty(n % ST) : bar_vempty(n % ST), ((n / ST) & 1) ^ 1, abort_flag,
                  p.status);
    }
    __syncwarp();
  } else if (warp <= NB) {
    // -------------------------------------------- MMA issuer of buffer b
    // Buffer b takes the CTA's pairs b, b + NB, ...; its issuer runs
    // S = Q K^T, then (after the softmax) O = P V, in that order, so the
    // two buffers never wait on each other's barriers.
    const int b = warp - 1;
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_f16(kBF16, 128, 2 * D, true);
      // Stages are contiguous, so a stage's descriptor is the first one plus
      // s * QK_BYTES / 16 in the start-address field.
      const uint64_t dq0 = smem_desc(q_smem(0), 16, 8 * C::ROWB, C::LAYOUT);
      const uint64_t dk0 = smem_desc(k_smem(0), 16, 8 * C::ROWB, C::LAYOUT);
      constexpr uint64_t kStageDesc = C::QK_BYTES >> 4;
      const uint32_t d = tmem + C::s_col(b), o = tmem + C::o_col(b);
      int n = b, use = 0;
      for (int t = blockIdx.x + b * gridDim.x; t < p.total; t += NB * gridDim.x, n += NB, ++use) {
        const Pair pr = decode_pair<KS>(t, p);
        const int s = n % ST;
        if (!mbar_wait(bar_kfull(n), (n / LCM) & 1, abort_flag, p.status)) break;
        // S of this buffer is free once the epilogue has read the buffer's
        // previous O, which overlays the dead part of S (after P.V read P).
        if (!mbar_wait(bar_o_empty(b), (use & 1) ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint64_t qA = dq0 + s * kStageDesc, qB = qA + (C::QBLK >> 4);
        const uint64_t kA = dk0 + s * kStageDesc, kB = kA + (uint64_t)(pr.rB * C::HW * C::ROWB >> 4);
#pragma unroll
        for (int n0 = 0; n0 < C::NS; n0 += 256) {
          const int N = C::NS - n0 < 256 ? C::NS - n0 : 256;
          const uint32_t idesc = idesc_f16(kBF16, 128, N, false);
          const uint64_t no = (uint64_t)(n0 * C::ROWB >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(d + n0, qA + kk * 2, kA + no + kk * 2, idesc, kk > 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(d + n0, qB + kk * 2, kB + no + kk * 2, idesc, 1u);
        }
        mma_commit(bar_s_full(b));
        mma_commit(bar_kempty(s));

        if (!mbar_wait(bar_p_full(b), use & 1, abort_flag, p.status)) break;
        if (!mbar_wait(bar_vfull(n), (n / LCM) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        // B = [V_A | V_B]: two MN blocks of d columns, tile B's rows rB halo rows further on
        const uint64_t vd = smem_desc(v_smem(s), (uint32_t)(pr.rB * C::HW * C::ROWB), 8 * C::ROWB, C::LAYOUT);
        constexpr uint64_t kstep = 16 * C::ROWB >> 4;
        mma_ts(o, d, vd, idesc_pv, 0u);
#pragma unroll
        for (int kk = 1; kk < C::NS / 16; ++kk) mma_ts(o, d + kk * 8, vd + kk * kstep, idesc_pv, 1u);
        mma_commit(bar_o_full(b));
        mma_commit(bar_vempty(s));
      }
    }
    __syncwarp();
  }
  } else if (warp < 4 + 4 * NB) {
    regs_inc<C::REGS_SOFTMAX>();
    // --------------------------------------------------------- softmax groups
    const int g = (warp - 4) >> 2;  // group = tensor-memory buffer
    const int wq = warp & 3;        // lane quarter
    const int gtid = threadIdx.x - 128 - 128 * g;
    const int tile = lane >> 4, l16 = lane & 15;
    const int pr0 = (wq >> 1) * PQ + (l16 >> 2);  // query row inside the tile
    const int pc0 = (wq & 1) * PQ + (l16 & 3);    // query column inside the tile
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const uint32_t sbuf = tmem + lane_base + C::s_col(g);
    T* tbl = tables + g * (C::TBL_BYTES / 2);
    T* raw = raws + g * (C::RAW_BYTES / 2);
    const float c = p.scale_log2;
    const T* rpb = static_cast<const T*>(p.rpb);
    Meeting tmeet{bar_tbl(g), 0u, abort_flag, p.status};
    int cur_h = -1;
    int use = 0;
    for (int t = blockIdx.x + g * gridDim.x; t < p.total; t += NB * gridDim.x, ++use) {
      const Pair pr = decode_pair<KS>(t, p);
      if (pr.h != cur_h) {
        // New head: stage its bias with all loads in flight at once, then
        // expand it into every copy of the group's table.
        constexpr int span = 2 * KS - 1;
        constexpr int PER = (C::RAW + 127) / 128;
        T rv[PER];
#pragma unroll
        for (int m = 0; m < PER; ++m) {
          const int idx = gtid + 128 * m;
          rv[m] = (idx < C::RAW && rpb) ? rpb[(size_t)pr.h * C::RAW + idx] : T(0.f);
        }
#pragma unroll
        for (int m = 0; m < PER; ++m)
          if (gtid + 128 * m < C::RAW) raw[gtid + 128 * m] = rv[m];
        if (!tmeet.sync()) break;  // raw is visible; the previous pair's table reads are done
        // copy 0, one table column per thread
        for (int col = gtid; col < C::TBL_W; col += 128) {
          const int blk = col / (KS + C::PAD), off = col % (KS + C::PAD);
          const bool live = blk < KS && off >= C::PAD;
          const int bc = blk + (off - C::PAD);
#pragma unroll
          for (int row = 0; row < C::TBL_ROWS; ++row)
            tbl[row * C::TBL_W + col] = (live && row < span) ? raw[row * span + bc] : neg_inf<T>();
        }
        if (!tmeet.sync()) break;  // copy 0 is complete
        // copies 1..: entry y of copy q is entry y + q of copy 0 (-inf past
        // its end), four entries per 8-byte store, shifted out of two
        // aligned 8-byte loads of copy 0
        {
          constexpr int QUADS = C::TBL_N / 4;
          const uint32_t ninf2 = bits16(neg_inf<T>()) * 0x10001u;
          for (int u = gtid; u < (C::TBL_COPIES - 1) * QUADS; u += 128) {
            const int q = 1 + u / QUADS, y = (u - (q - 1) * QUADS) * 4;
            const uint2 lo = *reinterpret_cast<const uint2*>(tbl + y);
            const uint2 hi = y + 4 < C::TBL_N ? *reinterpret_cast<const uint2*>(tbl + y + 4) : make_uint2(ninf2, ninf2);
            const uint32_t w[4] = {lo.x, lo.y, hi.x, hi.y};
            const int k = q >> 1, sh = (q & 1) * 16;
            *reinterpret_cast<uint2*>(tbl + C::tbl_base(q) + y) =
                make_uint2(__funnelshift_r(w[k], w[k + 1], sh), __funnelshift_r(w[k + 1], w[k + 2], sh));
          }
        }
        if (!tmeet.sync()) break;
        cur_h = pr.h;
      }
      const int i = (tile ? pr.i0[1] : pr.i0[0]) + pr0, j = (tile ? pr.j0[1] : pr.j0[0]) + pc0;
      const int ic = min(i, p.H - 1), jc = min(j, p.W - 1);
      const int si = window_start(ic, p.H, KS), sj = window_start(jc, p.W, KS);
      const int rt = tile ? pr.rt[1] : pr.rt[0];                // map row of this tile's S-space row 0
      const int wr0 = si - rt, wc0 = sj - (tile ? pr.c0[1] : pr.c0[0]);  // window origin in S-space
      const int er = rt - ic + KS - 1;                         // bias row of halo row 0
      const int colbase = (sj - jc + KS - 1) * (KS + C::PAD) + C::PAD - wc0;
      const int u_r0 = __reduce_min_sync(0xffffffffu, wr0);
      const int u_r1 = __reduce_max_sync(0xffffffffu, wr0 + KS);
      const int pb = __reduce_min_sync(0xffffffffu, wc0) >> 2;
      const int pe = (__reduce_max_sync(0xffffffffu, wc0 + KS) + 3) >> 2;

      if (!mbar_wait(bar_s_full(g), use & 1, abort_flag, p.status)) break;
      tc_fence_after();
      // this lane's table origin, in the copy where its entries are aligned
      const int cq = colbase & (C::TBL_COPIES - 1);
      const T* tl = tbl + C::tbl_base(cq) + colbase - cq;
      const float l = softmax_dispatch<T, KS, D>(pb, pe, sbuf, tl, u_r0, u_r1, wr0, er, c);
      // the row sum goes to the epilogue warpgroup through shared memory
      lsums[(g * 2 + (use & 1)) * 128 + wq * 32 + lane] = l;
      warp_arrive(bar_l_full(g, use & 1));
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(bar_p_full(g));
    }
  } else {
    if constexpr (C::REGS_EPI < C::LAUNCH_REGS) regs_dec<C::REGS_EPI>();
    // ------------------------------------------------------------ epilogue
    // Every pair of the CTA in order: O / l, rounded to T, stored.  O holds
    // tile A's d columns, then tile B's.
    const int wq = warp & 3;
    const int tile = lane >> 4, l16 = lane & 15;
    const int pr0 = (wq >> 1) * PQ + (l16 >> 2);
    const int pc0 = (wq & 1) * PQ + (l16 & 3);
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    T* out = static_cast<T*>(p.out);
    int n = 0;
    for (int t = blockIdx.x; t < p.total; t += gridDim.x, ++n) {
      const int b = n % NB, use = n / NB;
      const Pair pr = decode_pair<KS>(t, p);
      const int i = (tile ? pr.i0[1] : pr.i0[0]) + pr0, j = (tile ? pr.j0[1] : pr.j0[0]) + pc0;
      const bool valid = i < p.H && j < p.W && (tile == 0 || pr.has_b);
      T* dst = out + ((((size_t)(tile ? pr.b[1] : pr.b[0]) * p.heads + pr.h) * p.H + min(i, p.H - 1)) * p.W +
                      min(j, p.W - 1)) * D;
      if (!mbar_wait(bar_l_full(b, use & 1), (use >> 1) & 1, abort_flag, p.status)) break;
      const float inv = 1.f / lsums[(b * 2 + (use & 1)) * 128 + wq * 32 + lane];
      if (!mbar_wait(bar_o_full(b), use & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t obuf = tmem + lane_base + C::o_col(b);
#pragma unroll
      for (int cc = 0; cc < D; cc += 16) {
        uint32_t oa[16], ob[16];
        tmem_ld16(obuf + cc, oa);
        tmem_ld16(obuf + D + cc, ob);
        tmem_wait_ld_regs(oa);
        tmem_wait_ld_regs(ob);
        if (cc + 16 >= D) {
          tc_fence_before();
          warp_arrive(bar_o_empty(b));
        }
        if (valid) {
#pragma unroll
          for (int x = 0; x < 16; x += 8) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(tile ? ob[x + e] : oa[x + e]) * inv;
            uint4 w;
            w.x = pack2<T>(f[0], f[1]);
            w.y = pack2<T>(f[2], f[3]);
            w.z = pack2<T>(f[4], f[5]);
            w.w = pack2<T>(f[6], f[7]);
            *reinterpret_cast<uint4*>(dst + cc + x) = w;
          }
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
  CUtensorMap mq, mk, mv, mk1, mv1;
  if (!make_map(&mq, q, s, bf16, PQ, PQ) || !make_map(&mk, k, s, bf16, C::HW, C::HHP) ||
      !make_map(&mv, v, s, bf16, C::HW, C::HHP) || !make_map(&mk1, k, s, bf16, C::HW, C::HS) ||
      !make_map(&mv1, v, s, bf16, C::HW, C::HS))
    return cudaErrorInvalidValue;
  auto kern = na2d_fwd_tc_kernel<T, KS, D>;
  static std::mutex mu;
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_set[dev]) {
      // The run-time register split (setmaxnreg) must fit what the CTA is
      // launched with, or its warpgroups would wait for registers forever.
      cudaFuncAttributes fa;
      cudaError_t e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return e;
      if (C::REGS_CTRL * 128 + C::REGS_EPI * 128 + C::REGS_SOFTMAX * 128 * C::NBUF > fa.numRegs * C::THREADS)
        return cudaErrorInvalidConfiguration;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
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
  // A last tile row of 1..8 rows is made of single tiles, packed two per
  // pair; a last pair row of 9..15 rows stays a (ragged) pair.
  p.n_pc = (s.W + TT - 1) / TT;
  const int rem = s.H % (2 * TT);
  const bool singles = rem > 0 && rem <= TT;
  p.n_fpr = singles ? s.H / (2 * TT) : (s.H + 2 * TT - 1) / (2 * TT);
  const long long full = (long long)s.B * p.n_fpr * p.n_pc;
  const long long single = singles ? (long long)s.B * p.n_pc : 0;
  const long long per_head = full + (single + 1) / 2;
  const long long pairs = per_head * s.heads;
  if (pairs > 0x7fffffffLL) return cudaErrorInvalidValue;
  p.full_per_head = (int)full;
  p.singles_per_head = (int)single;
  p.per_head = (int)per_head;
  p.total = (int)pairs;
  p.div_head = FastDiv((uint32_t)s.heads);
  p.div_pc = FastDiv((uint32_t)p.n_pc);
  p.div_fpr = FastDiv((uint32_t)(p.n_fpr > 0 ? p.n_fpr : 1));
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s.d));
  p.status = status;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = p.total < sms ? p.total : sms;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(mq, mk, mv, mk1, mv1, p);
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
    case 11: return launch<T, 11, D>(q, k, v, rpb, out, s, status, st);
    case 13: return launch<T, 13, D>(q, k, v, rpb, out, s, status, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool forward_tc_supported(const Shape& s, na_dtype dt) {
  if (dt != NA_F16 && dt != NA_BF16) return false;
  if (s.d != 32 && s.d != 64) return false;
  if (s.ks < 3 || s.ks > 13 || (s.ks & 1) == 0) return false;

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
