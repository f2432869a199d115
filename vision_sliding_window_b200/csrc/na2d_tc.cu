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
// A tile's S (its halo rows x halo columns) is computed in chunks of CR halo
// rows.  Chunks go through a ring of S slots in tensor memory, so the MMA of
// later chunks runs while a softmax group works on earlier ones:
//   S_c = Q K_c^T  ->  softmax of chunk c, P_c written over S_c (16 bits)
//   ->  O += P_c V_c  (O in one of two O slots, apart from the S slots).
// The softmax needs no maximum across chunks: every row of P is taken as
// exp2((y - f) log2e/sqrt(d)) with f = the row's own maximum rounded up to an
// integer in those units, then multiplied by the exact power of two
// 2^(f - sigma).  P is therefore exp2(y log2e/sqrt(d) - sigma) for every
// entry, i.e. softmax numerators with one fixed shift sigma, while the 16-bit
// exponent argument stays in (-1, 0] for each row's largest entries.  Rows
// of a query whose sum leaves the range where that is exact (huge or tiny
// logits) are recomputed by the epilogue from global memory (exact_query).
//
// Roles of one persistent CTA per SM:
//   warp 0          TMA producer of the Q/K ring (query tiles, K halo) and of
//                   the V ring
//   warp 1          issuer of S = Q K^T (also allocates and frees tensor memory)
//   warps 2, 3      issuers of O += P V for even and odd pairs
//   warpgroups 1..NG  softmax groups: group g takes every NG-th pair
//   last warpgroup  the epilogue of every pair, in order
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
  static constexpr int NPC = HW / 4;                   // 4-key pieces per halo row
  static constexpr int NPU = (PQ - 1 + KS + 3) / 4;    // pieces of an interior patch's window union
  static constexpr int ROWB = 2 * D;                   // bytes per key / query row
  static constexpr int QBLK = 2 * TT * TT * ROWB;      // one K block of the query operand (128 rows)
  static constexpr int Q_BYTES = 2 * QBLK;
  static constexpr int KV_BYTES = HHP * HW * ROWB;
  static constexpr int QK_BYTES = Q_BYTES + KV_BYTES;  // one stage of the Q/K ring
  // ---------------------------------------------------------- tensor memory
  // NO slots of O (2d columns each: tile A's d, then tile B's d), then NSLOT
  // slots of S, each holding one chunk of CR halo rows (CR x HW columns of
  // fp32 S; P overlays the first CR x HW/2 columns as 16-bit pairs).
  static constexpr int NG = 2;  // softmax groups
  static constexpr int NO = 2;
  static constexpr int O_COLS = 2 * D;
  static constexpr int CR = HW == 16 ? 8 : 4;
  static constexpr int NCH = (HH + CR - 1) / CR;
  static constexpr int SLOT_COLS = CR * HW;
  static constexpr int NSLOT_FIT = (kTmemCols - NO * O_COLS) / SLOT_COLS;
  static constexpr int NSLOT = NSLOT_FIT > 4 ? 4 : NSLOT_FIT;
  static constexpr int PW = HW / 2;  // 32-bit columns of one P row
  static constexpr int o_col(int o) { return o * O_COLS; }
  static constexpr int s_col(int s) { return NO * O_COLS + s * SLOT_COLS; }
  static constexpr int chunk_rows(int c) { return (c + 1) * CR <= HH ? CR : HH - c * CR; }
  static_assert(NSLOT >= 2, "two S slots must fit next to the O slots");
  static_assert(SLOT_COLS % 16 == 0 && (chunk_rows(NCH - 1) * HW) % 16 == 0,
                "chunk widths must be multiples of the MMA's N and K steps");
  static_assert(SLOT_COLS <= 256, "one MMA covers a chunk");
  // ---------------------------------------------------- bias / mask table
  // One per CTA (the grid is chosen so that a CTA meets one head), 16-bit
  // entries of the input type, exactly the
  // bias values given: rows 0..2KS-2 hold bias rows, row 2KS-1 is all -inf.
  // A row is KS blocks of stride KS+PAD; block dc holds the bias row's
  // columns dc..dc+KS-1 after PAD entries of -inf, and its tail is the next
  // block's -inf head.  PAD covers a whole halo row around any window.
  static constexpr int PAD = HW - KS;
  static constexpr int TBL_W0 = KS * (KS + PAD) + PAD;
  static constexpr int TBL_W = TBL_W0 + ((4 - TBL_W0 % 64) + 64) % 64;  // = 4 mod 64 entries
  static constexpr int TBL_ROWS = 2 * KS;
  static constexpr int TBL_N = TBL_ROWS * TBL_W;  // entries of one copy
  static_assert(TBL_W % 4 == 0 && TBL_N % 4 == 0, "table rows keep a column's offset mod 4");
  // Copies of the table, copy q shifted left by q entries: every lane reads
  // its entries 4 at a time with 8-byte loads (2 at a time with 4-byte loads
  // when only two copies are kept, one at a time from a single copy) from the
  // copy that makes them aligned.
  // Copy q starts tbl_off(q) entries past a 64-entry boundary: offsets that
  // spread the 16 lanes of a tile over distinct banks for the softmax's
  // lane-to-query layout.
  static constexpr int TBL_CS = round_up(TBL_N, 64);
  static constexpr int tbl_off(int q) { return q == 0 ? 0 : q == 1 ? 16 : KS % 4 == 1 ? 16 * q : 16 * q + 4; }
  static constexpr int tbl_base(int q) { return q * TBL_CS + tbl_off(q); }
  static constexpr int tbl_bytes(int copies) { return round_up((tbl_base(copies - 1) + TBL_N) * 2, 16); }
  static constexpr int RAW = (2 * KS - 1) * (2 * KS - 1);  // one head's bias table
  static constexpr int RAW_BYTES = round_up(RAW * 2, 16);
  static constexpr int LSUM_BYTES = NG * 2 * 128 * 4;  // row sums handed to the epilogue, per group and use parity
  static constexpr int BAR_BYTES = 512;
  // Shared memory: a ring of STQ stages of Q and K, a ring of STV stages of
  // V, one bias table (TBL_COPIES copies) for the CTA's head, the staged raw
  // table, the row sums and the barriers.  The first plan of (STQ, STV,
  // copies) that fits, in this order: deeper rings first, then the table
  // copies that let a lane read 4 entries per load.
  static constexpr int fixed_with(int copies) {
    return 1024 + tbl_bytes(copies) + RAW_BYTES + LSUM_BYTES + BAR_BYTES;
  }
  static constexpr int need(int stq, int stv, int copies) {
    return fixed_with(copies) + stq * QK_BYTES + stv * KV_BYTES;
  }
  static constexpr int kPlans[9][3] = {{3, 3, 4}, {3, 3, 2}, {2, 2, 4}, {2, 2, 2}, {2, 1, 4},
                                        {2, 1, 2}, {1, 1, 4}, {1, 1, 2}, {1, 1, 1}};
  static constexpr int plan() {
    for (int i = 0; i < 9; ++i)
      if (need(kPlans[i][0], kPlans[i][1], kPlans[i][2]) <= kMaxSmem) return i;
    return -1;
  }
  static_assert(plan() >= 0, "a Q/K stage, a V stage and a table must fit in shared memory");
  static constexpr int STQ = kPlans[plan()][0];
  static constexpr int STV = kPlans[plan()][1];
  static constexpr int TBL_COPIES = kPlans[plan()][2];
  static constexpr int TBL_BYTES = tbl_bytes(TBL_COPIES);
  static constexpr int SMEM_RAW = need(STQ, STV, TBL_COPIES);
  static constexpr int SMEM_BYTES = SMEM_RAW > kMinSmem ? SMEM_RAW : kMinSmem;
  // Warpgroup 0: the TMA producer (warp 0) and the MMA issuers (warps 1-3);
  // warpgroups 1..NG: softmax groups; the last warpgroup: the epilogue.  The
  // register file is re-split at run time (setmaxnreg) within what the CTA
  // is launched with.
  static constexpr int THREADS = 128 * (2 + NG);
  static constexpr int LAUNCH_REGS = 128;  // 65536 / THREADS
  static constexpr int REGS_CTRL = 88;
  static constexpr int REGS_SOFTMAX = 160;
  static constexpr int REGS_EPI = 104;
  static_assert(REGS_CTRL * 128 + REGS_EPI * 128 + REGS_SOFTMAX * 128 * NG <= LAUNCH_REGS * THREADS,
                "the register split must fit the launch allocation");
  static constexpr uint32_t LAYOUT = ROWB == 64 ? kLayoutSW64 : kLayoutSW128;
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
// Unit t is pair t / heads of head t % heads: with the head fastest and a
// grid that is a multiple of the head count, all the units of a CTA share
// one head, and so its bias table.
struct Params {
  const void* q;  // the inputs again, for the exact path of out-of-range rows
  const void* k;
  const void* v;
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
// argument is rounded to T first: for arguments in (-1, 0] (the largest
// entries of a row, after its own shift) that moves the result by at most
// 2^-9 ln2 relative in bf16 and 2^-12 ln2 in fp16; smaller entries carry a
// larger relative but a negligible absolute error.
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
// Both halves of w times both halves of s (a power of two: exact unless the
// product leaves T's normal range).
template <typename T> NA_DEVICE uint32_t mul_pair(uint32_t w, uint32_t s);
template <> NA_DEVICE uint32_t mul_pair<__nv_bfloat16>(uint32_t w, uint32_t s) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(s));
  return r;
}
template <> NA_DEVICE uint32_t mul_pair<__half>(uint32_t w, uint32_t s) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(s));
  return r;
}

// The fixed shift sigma of P = exp2(a - sigma) and the bit layout of a
// power of two in T.  P's range decides sigma: bf16 has fp32's exponent
// range, fp16 tops out at 65504, so fp16 probabilities are shifted down by
// 2^4 to leave room above the largest logits seen in practice.  A query's
// row sum l decides whether the fast path was exact: it must lie in
// [kLo, kHi] (finite, and large enough that entries lost to T's underflow
// are negligible against it); otherwise the epilogue recomputes the query.
template <typename T> struct Shift;
template <> struct Shift<__nv_bfloat16> {
  static constexpr int kSigma = 0, kBias = 127, kMax = 255, kShift = 7;
  static constexpr float kLo = 0x1p-64f, kHi = 0x1p64f;
};
template <> struct Shift<__half> {
  static constexpr int kSigma = 4, kBias = 15, kMax = 31, kShift = 10;
  static constexpr float kLo = 0x1p-6f, kHi = 0x1p30f;
};

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

// Softmax numerators of one chunk -- S-space rows [r_lo, r_hi) of a slot --
// for one warp's 32 queries (two 4x4 patches, one per tile), over the union
// rows [u_r0, u_r1) and pieces [PB, PB+NU) of their windows, RB rows at a
// time: each batch's tensor-memory loads are issued together and the RB
// rows are independent streams of arithmetic.  Per batch: y = s + table (the
// bias, -inf outside the window), the batch maximum m and an integer shift f
// in [m c, m c + 1] with c = log2e/sqrt(d); per row e = exp2(y c - f) in T
// and P = e * 2^(f - sigma) written as 16-bit pairs over S -- P row t of the chunk covers the S
// columns of chunk row t / 2, read by an earlier or the same batch -- with
// zeros outside the pieces and in the chunk's rows outside the union.
// Returns the chunk's part of the row sum, sum(P).  Rows past the union's
// end in the last batch repeat its last row: they store the same values
// again and are left out of the sum.
template <typename T, int KS, int D, int PB, int NU>
NA_DEVICE float softmax_chunk(uint32_t sbuf, const T* tl, int r_lo, int r_hi, int u_r0, int u_r1, int wr0,
                              int er, float c) {
  using C = Cfg<KS, D>;
  using E = Shift<T>;
  constexpr int HW = C::HW, PW = C::PW, NV = NU * 4, RB = 1;
  // start-column alignment of a piece window (row t * HW + PB * 4) and of a P row (t * PW)
  constexpr int AS = PB == 0 ? low_pow2(HW) : (low_pow2(HW) < low_pow2(PB * 4) ? low_pow2(HW) : low_pow2(PB * 4));
  constexpr int AP = low_pow2(PW);
  const int c0 = max(r_lo, u_r0), c1 = min(r_hi, u_r1);
  uint32_t z[PW];
#pragma unroll
  for (int e = 0; e < PW; ++e) z[e] = 0u;
#pragma unroll 1
  for (int hr = r_lo; hr < min(c0, r_hi); ++hr) st_span<PW, AP>(sbuf + (hr - r_lo) * PW, z);
  float l = 0.f;
#pragma unroll 1
  for (int r0 = c0; r0 < c1; r0 += RB) {
    uint32_t v[RB][NV];
#pragma unroll
    for (int j = 0; j < RB; ++j) ld_span<NV, AS>(sbuf + (min(r0 + j, c1 - 1) - r_lo) * HW + PB * 4, v[j]);
#pragma unroll
    for (int j = 0; j < RB; ++j) tmem_wait_ld_regs(v[j]);
    // y = s + table in place, and the batch's maximum
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      const int hr = min(r0 + j, c1 - 1);
      const T* tr = tl + ((unsigned)(hr - wr0) < (unsigned)KS ? hr + er : 2 * KS - 1) * C::TBL_W + PB * 4;
#pragma unroll
      for (int e = 0; e < NV; e += 4) {
        uint32_t b01, b23;  // entries e, e+1 and e+2, e+3
        if constexpr (C::TBL_COPIES == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(tr + e);
          b01 = w.x;
          b23 = w.y;
        } else if constexpr (C::TBL_COPIES == 2) {
          b01 = *reinterpret_cast<const uint32_t*>(tr + e);
          b23 = *reinterpret_cast<const uint32_t*>(tr + e + 2);
        } else {
          const unsigned short* t16 = reinterpret_cast<const unsigned short*>(tr + e);
          b01 = (uint32_t)t16[0] | ((uint32_t)t16[1] << 16);
          b23 = (uint32_t)t16[2] | ((uint32_t)t16[3] << 16);
        }
        float y0, y1, y2, y3;
        add_pair<T>(y0, y1, __uint_as_float(v[j][e]), __uint_as_float(v[j][e + 1]), b01);
        add_pair<T>(y2, y3, __uint_as_float(v[j][e + 2]), __uint_as_float(v[j][e + 3]), b23);
        mx = max3(mx, max3(y0, y1, y2), y3);
        v[j][e] = __float_as_uint(y0);
        v[j][e + 1] = __float_as_uint(y1);
        v[j][e + 2] = __float_as_uint(y2);
        v[j][e + 3] = __float_as_uint(y3);
      }
    }
    // The batch's shift f: the integer round(m c + 1/2) in [m c, m c + 1],
    // kept in [-100, 200] (rows outside every window give exp2(-inf) = 0
    // rather than NaN, and the exponent arithmetic cannot overflow).  Adding
    // 1.5 * 2^23 leaves that integer in the float's low mantissa bits.  Any
    // shift at most one above the query's maximum keeps its largest entries'
    // arguments in [-1, 0], so one shift serves all rows of the batch.  Then
    // the power of two 2^(f - sigma) in T (both halves) and as a float: the
    // float saturates exactly where T does, so a power of two T cannot hold
    // makes the row sum infinite (the query goes to the exact path) and one
    // below T's normal range zeroes the rows' P and their share of the sum
    // alike.
    constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
    const float t = fminf(fmaxf(fmaf(mx, c, 0.5f), -100.f), 200.f) + kMagic;
    const int eb = __float_as_int(t) - __float_as_int(kMagic) - E::kSigma + E::kBias;
    const float nf = kMagic - t;  // -f
    const uint32_t s16 = (uint32_t)min(max(eb, 0), E::kMax) << E::kShift;
    const uint32_t s2 = s16 * 0x10001u;
    float sf;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) sf = __uint_as_float(s16 << 16);
    else sf = __half2float(__ushort_as_half((unsigned short)s16));
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      const int hr = min(r0 + j, c1 - 1);
      uint32_t pk[PW];
#pragma unroll
      for (int e = 0; e < PW; ++e) pk[e] = 0u;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int e = 0; e < NV; e += 4) {
        float a0, a1, a2, a3;
        fma2(a0, a1, __uint_as_float(v[j][e]), __uint_as_float(v[j][e + 1]), c, c, nf, nf);
        fma2(a2, a3, __uint_as_float(v[j][e + 2]), __uint_as_float(v[j][e + 3]), c, c, nf, nf);
        const uint32_t pa = exp2_pair<T>(a0, a1), pb = exp2_pair<T>(a2, a3);
        acc_pair<T>(s0, s1, pa);
        acc_pair<T>(s0, s1, pb);
        pk[PB * 2 + e / 2] = mul_pair<T>(pa, s2);
        pk[PB * 2 + e / 2 + 1] = mul_pair<T>(pb, s2);
      }
      st_span<PW, AP>(sbuf + (hr - r_lo) * PW, pk);
      if (r0 + j < c1) l = fmaf(s0 + s1, sf, l);
    }
  }
#pragma unroll 1
  for (int hr = max(c0, c1); hr < r_hi; ++hr) st_span<PW, AP>(sbuf + (hr - r_lo) * PW, z);
  return l;
}

// Runs softmax_chunk over the pieces [pb, pb + NPU) of an interior patch's
// window union, fixed at compile time, or over whole rows when the union is
// wider (patches at the map border).
template <typename T, int KS, int D, int PB = 0>
NA_DEVICE float softmax_dispatch(int pb, int pe, uint32_t sbuf, const T* tl, int r_lo, int r_hi, int u_r0,
                                 int u_r1, int wr0, int er, float c) {
  using C = Cfg<KS, D>;
  if constexpr (PB + C::NPU <= C::NPC) {
    if (pe - pb <= C::NPU && min(pb, C::NPC - C::NPU) == PB)
      return softmax_chunk<T, KS, D, PB, C::NPU>(sbuf, tl, r_lo, r_hi, u_r0, u_r1, wr0, er, c);
    return softmax_dispatch<T, KS, D, PB + 1>(pb, pe, sbuf, tl, r_lo, r_hi, u_r0, u_r1, wr0, er, c);
  } else {
    return softmax_chunk<T, KS, D, 0, C::NPC>(sbuf, tl, r_lo, r_hi, u_r0, u_r1, wr0, er, c);
  }
}

// 8 consecutive elements of T as floats (one 16-byte load).
template <typename T>
NA_DEVICE void load8(const T* p, float (&f)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[t]));
      f[2 * t] = x.x;
      f[2 * t + 1] = x.y;
    } else {
      const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&u[t]));
      f[2 * t] = x.x;
      f[2 * t + 1] = x.y;
    }
  }
}

// The exact path for one query whose fast-path row sum left its range: the
// output of Eqs. (2)-(4) straight from global memory, in float with the
// exact row maximum subtracted, rounded to T.  Logits are recomputed for
// each 8-column group of the output rather than kept, so the path needs few
// registers; it runs only for queries with extreme logits.
template <typename T, int KS, int D>
__device__ __noinline__ void exact_query(const Params& p, int b, int h, int i, int j, T* dst) {
  const size_t map = ((size_t)b * p.heads + h) * p.H * p.W;
  const T* qv = static_cast<const T*>(p.q) + (map + (size_t)i * p.W + j) * D;
  const T* kb = static_cast<const T*>(p.k) + map * D;
  const T* vb = static_cast<const T*>(p.v) + map * D;
  const T* rpb = static_cast<const T*>(p.rpb);
  const int si = window_start(i, p.H, KS), sj = window_start(j, p.W, KS);
  constexpr int span = 2 * KS - 1;
  auto logit = [&](int a, int cc) {  // (q . k + bias) log2(e) / sqrt(d)
    const T* kv = kb + ((size_t)(si + a) * p.W + sj + cc) * D;
    float dot = 0.f;
#pragma unroll 1
    for (int x = 0; x < D; x += 8) {
      float fq[8], fk[8];
      load8(qv + x, fq);
      load8(kv + x, fk);
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(fq[e], fk[e], dot);
    }
    const float bias =
        rpb ? (float)rpb[((size_t)h * span + (si + a - i + KS - 1)) * span + (sj + cc - j + KS - 1)] : 0.f;
    return (dot + bias) * p.scale_log2;
  };
  float m = -INFINITY;
#pragma unroll 1
  for (int a = 0; a < KS; ++a)
#pragma unroll 1
    for (int cc = 0; cc < KS; ++cc) m = fmaxf(m, logit(a, cc));
  float l = 0.f;
#pragma unroll 1
  for (int x0 = 0; x0 < D; x0 += 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int a = 0; a < KS; ++a)
#pragma unroll 1
      for (int cc = 0; cc < KS; ++cc) {
        const float w = exp2f(logit(a, cc) - m);
        if (x0 == 0) l += w;
        float fv[8];
        load8(vb + ((size_t)(si + a) * p.W + sj + cc) * D + x0, fv);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, fv[e], acc[e]);
      }
    const float inv = 1.f / l;
    uint4 o;
    o.x = pack2<T>(acc[0] * inv, acc[1] * inv);
    o.y = pack2<T>(acc[2] * inv, acc[3] * inv);
    o.z = pack2<T>(acc[4] * inv, acc[5] * inv);
    o.w = pack2<T>(acc[6] * inv, acc[7] * inv);
    *reinterpret_cast<uint4*>(dst + x0) = o;
  }
}

template <typename T, int KS, int D>
__global__ void __launch_bounds__(Cfg<KS, D>::THREADS, 1)
na2d_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k1,
                   const __grid_constant__ CUtensorMap tm_v1, const Params p) {
  using C = Cfg<KS, D>;
  constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int STQ = C::STQ, STV = C::STV, NSL = C::NSLOT, NO = C::NO, NG = C::NG, NCH = C::NCH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  constexpr int RINGS = STQ * C::QK_BYTES + STV * C::KV_BYTES;
  T* tbl = reinterpret_cast<T*>(smem + RINGS);
  T* raw = reinterpret_cast<T*>(smem + RINGS + C::TBL_BYTES);
  float* lsums = reinterpret_cast<float*>(smem + RINGS + C::TBL_BYTES + C::RAW_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RINGS + C::TBL_BYTES + C::RAW_BYTES + C::LSUM_BYTES);
  // Two shared-memory rings: Q and K (STQ stages, released when the last
  // chunk of S = Q K^T has read them) and V (STV stages, released when the
  // last chunk of P.V has), fed by one producer thread in pair order.
  // barrier slots: kfull[STQ] kempty[STQ] vfull[STV][2] vempty[STV]
  //                s_full[NSL][NG] p_full[NSL][2] slot_free[NSL]
  //                o_full[2] o_empty[2]
  //                tbl  l_full[NG][2] l_empty[NG][2]  mma_done[3]
  // The "V loaded" and "P written" barriers are per P.V issuer and the "S
  // ready" ones per softmax group: where two threads take turns on a slot,
  // each waits on a barrier of its own, so one that runs ahead never sees
  // the other's phase.
  constexpr int B_V = 2 * STQ, B_S = B_V + 3 * STV, B_O = B_S + (NG + 3) * NSL, B_G = B_O + 4,
                N_BARS = B_G + 4 * NG + 4;
  static_assert(NG == 2 && NO == 2, "softmax groups, P.V issuers and O slots go by pair parity");
  static_assert(N_BARS * 8 + 8 <= C::BAR_BYTES, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_addr(bars + i); };
  auto bar_kfull = [&](int s) { return bar(s); };
  auto bar_kempty = [&](int s) { return bar(STQ + s); };
  auto bar_vfull = [&](int s, int u) { return bar(B_V + 2 * s + u); };
  auto bar_vempty = [&](int s) { return bar(B_V + 2 * STV + s); };
  auto bar_s_full = [&](int sl, int g) { return bar(B_S + sl * NG + g); };
  auto bar_p_full = [&](int sl, int u) { return bar(B_S + NG * NSL + 2 * sl + u); };
  auto bar_slot_free = [&](int sl) { return bar(B_S + (NG + 2) * NSL + sl); };
  auto bar_o_full = [&](int o) { return bar(B_O + o); };
  auto bar_o_empty = [&](int o) { return bar(B_O + 2 + o); };
  auto bar_tbl = [&]() { return bar(B_G); };
  auto bar_l_full = [&](int g, int par) { return bar(B_G + 1 + 2 * g + par); };
  auto bar_l_empty = [&](int g, int par) { return bar(B_G + 1 + 2 * NG + 2 * g + par); };
  auto bar_mma_done = [&](int which) { return bar(B_G + 1 + 4 * NG + which); };
  auto q_smem = [&](int s) { return sbase + s * C::QK_BYTES; };
  auto k_smem = [&](int s) { return sbase + s * C::QK_BYTES + C::Q_BYTES; };
  auto v_smem = [&](int s) { return sbase + STQ * C::QK_BYTES + s * C::KV_BYTES; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's pairs: n = 0, 1, ... is work unit blockIdx.x + n * gridDim.x
  const int n_mine = (p.total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  auto unit = [&](int n) { return (int)blockIdx.x + n * (int)gridDim.x; };
  // The query operand of S = Q K^T is block structured: K block 0 holds
  // tile A's queries (TMEM lanes 0-15 of every quarter), K block 1 tile B's
  // (lanes 16-31); the other rows of each block stay zero.
  for (int s = 0; s < STQ; ++s)
    for (int i = threadIdx.x; i < C::Q_BYTES / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(smem + s * C::QK_BYTES)[i] = make_uint4(0u, 0u, 0u, 0u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int i = 0; i < B_S; ++i) mbar_init(bar(i), 1);
    for (int sl = 0; sl < NSL; ++sl) {
      for (int g = 0; g < NG; ++g) mbar_init(bar_s_full(sl, g), 1);
      for (int u = 0; u < 2; ++u) mbar_init(bar_p_full(sl, u), 4);  // barriers a warpgroup meets count its 4 warps
      mbar_init(bar_slot_free(sl), 1);
    }
    for (int o = 0; o < 2; ++o) {
      mbar_init(bar_o_full(o), 1);
      mbar_init(bar_o_empty(o), 4);
    }
    mbar_init(bar_tbl(), 4 * NG);  // every warp of every softmax group
    for (int g = 0; g < NG; ++g)
      for (int par = 0; par < 2; ++par) {
        mbar_init(bar_l_full(g, par), 4);
        mbar_init(bar_l_empty(g, par), 4);
      }
    for (int w = 0; w < 3; ++w) mbar_init(bar_mma_done(w), 1);
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
  if (warp == 0) {
    // -------------------------------------------- TMA producer (both rings)
    // Pair by pair: Q and K into the Q/K ring once that stage's previous
    // pair has left it, then V into the V ring likewise.
    if (lane == 0) {
      int n = 0;
      bool ok = true, qk_loaded = false;
      for (; n < n_mine; ++n) {
        qk_loaded = false;
        const Pair pr = decode_pair<KS>(unit(n), p);
        {
          const int s = n % STQ;
          if (!(ok = mbar_wait(bar_kempty(s), ((n / STQ) & 1) ^ 1, abort_flag, p.status))) break;
          const uint32_t full = bar_kfull(s);
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
          qk_loaded = true;
        }
        {
          const int s = n % STV;
          if (!(ok = mbar_wait(bar_vempty(s), ((n / STV) & 1) ^ 1, abort_flag, p.status))) break;
          const uint32_t full = bar_vfull(s, n & 1);
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
      if (ok) {
        // every load issued was consumed: the MMAs' release commits have all arrived
        for (int e = 0, m = n; e < STQ; ++e, ++m)
          mbar_wait(bar_kempty(m % STQ), ((m / STQ) & 1) ^ 1, abort_flag, p.status);
        for (int e = 0, m = n; e < STV; ++e, ++m)
          mbar_wait(bar_vempty(m % STV), ((m / STV) & 1) ^ 1, abort_flag, p.status);
      } else {
        // gave up: still let the loads in flight land before the CTA exits
        const int nq = qk_loaded ? n + 1 : n;  // Q/K loads issued: pairs [0, nq); V loads: [0, n)
        for (int m = nq - 1; m >= 0 && m >= nq - STQ; --m) mbar_wait_settle(bar_kfull(m % STQ), (m / STQ) & 1);
        uint32_t seen = 0;  // the latest V load of each stage
        for (int m = n - 1; m >= 0 && m >= n - STV; --m)
          if (!(seen & (1u << (m % STV)))) {
            seen |= 1u << (m % STV);
            // the k-th load of stage m % STV for issuer m & 1: phase parity of that issuer's uses
            int uses = 0;
            for (int x = m % STV; x <= m; x += STV) uses += (x & 1) == (m & 1);
            mbar_wait_settle(bar_vfull(m % STV, m & 1), (uses - 1) & 1);
          }
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- MMA issuers
    // Warp 1 issues S = Q K^T of every chunk j = n * NCH + c in order, into
    // slot j % NSL once P.V of chunk j - NSL has finished reading that
    // slot's P (the two write and read different accumulators, so nothing
    // else orders them).  Warps 2 and 3 issue O += P V for the pairs of
    // their parity u, into O slot u.  Each tcgen05.mma holds its thread for
    // a fixed time whatever its size, and MMAs of different threads overlap
    // in the tensor pipe, so the work is spread over three threads.  A
    // commit tracks the MMAs of the thread that issues it.
    if (lane == 0) {
      const int total = n_mine * NCH;
      bool ok = true;
      if (warp == 1) {
        // Stages are contiguous, so a stage's descriptor is the first one plus
        // s * QK_BYTES / 16 in the start-address field.
        const uint64_t dq0 = smem_desc(q_smem(0), 16, 8 * C::ROWB, C::LAYOUT);
        const uint64_t dk0 = smem_desc(k_smem(0), 16, 8 * C::ROWB, C::LAYOUT);
        constexpr uint64_t kStageDesc = C::QK_BYTES >> 4;
        int rB = 0;
        for (int i = 0; i < total; ++i) {
          const int n = i / NCH, c = i - n * NCH, sl = i % NSL, s = n % STQ;
          if (c == 0) {
            if (!(ok = mbar_wait(bar_kfull(s), (n / STQ) & 1, abort_flag, p.status))) break;
            rB = decode_pair<KS>(unit(n), p).rB;
          }
          if (i >= NSL && !(ok = mbar_wait(bar_slot_free(sl), ((i / NSL) - 1) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint64_t qA = dq0 + s * kStageDesc, qB = qA + (C::QBLK >> 4);
          const uint64_t ko = (uint64_t)((c * C::CR * C::HW * C::ROWB) >> 4);
          const uint64_t kA = dk0 + s * kStageDesc + ko, kB = kA + (uint64_t)(rB * C::HW * C::ROWB >> 4);
          const uint32_t idesc = idesc_f16(kBF16, 128, C::chunk_rows(c) * C::HW, false);
          const uint32_t d = tmem + C::s_col(sl);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(d, qA + kk * 2, kA + kk * 2, idesc, kk > 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(d, qB + kk * 2, kB + kk * 2, idesc, 1u);
          mma_commit(bar_s_full(sl, n % NG));
          if (c == NCH - 1) mma_commit(bar_kempty(s));
        }
      } else {
        const int u = warp - 2;  // pairs u, u + 2, ...; O slot u
        constexpr uint32_t idesc_pv = idesc_f16(kBF16, 128, 2 * D, true);
        constexpr uint64_t kstep = 16 * C::ROWB >> 4;
        uint32_t vph = 0, pph = 0;  // parity of this issuer's next wait on each V stage / S slot
        for (int n = u; n < n_mine && ok; n += 2) {
          const int s = n % STV;
          int rB = 0;
          for (int c = 0; c < NCH; ++c) {
            const int j = n * NCH + c, sl = j % NSL;
            if (!(ok = mbar_wait(bar_p_full(sl, u), (pph >> sl) & 1, abort_flag, p.status))) break;
            pph ^= 1u << sl;
            if (c == 0) {
              if (!(ok = mbar_wait(bar_vfull(s, u), (vph >> s) & 1, abort_flag, p.status))) break;
              vph ^= 1u << s;
              if (!(ok = mbar_wait(bar_o_empty(u), ((n >> 1) & 1) ^ 1, abort_flag, p.status))) break;
              rB = decode_pair<KS>(unit(n), p).rB;
            }
            tc_fence_after();
            // B = [V_A | V_B]: two MN blocks of d columns, tile B's rows rB halo rows further on
            const uint64_t vd = smem_desc(v_smem(s) + c * C::CR * C::HW * C::ROWB,
                                          (uint32_t)(rB * C::HW * C::ROWB), 8 * C::ROWB, C::LAYOUT);
            const uint32_t od = tmem + C::o_col(u), pd = tmem + C::s_col(sl);
            const int ksteps = C::chunk_rows(c) * C::HW / 16;
#pragma unroll 1
            for (int kk = 0; kk < ksteps; ++kk)
              mma_ts(od, pd + kk * 8, vd + kk * kstep, idesc_pv, (c > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar_slot_free(sl));
            if (c == NCH - 1) {
              mma_commit(bar_o_full(u));
              mma_commit(bar_vempty(s));
            }
          }
        }
      }
      // every MMA this thread issued has finished, and its commits have
      // arrived, before tensor memory is freed -- also when a role gave up
      mma_commit(bar_mma_done(warp - 1));
      mbar_wait_settle(bar_mma_done(warp - 1), 0);
    }
    __syncwarp();
  }
  } else if (warp < 4 + 4 * NG) {
    regs_inc<C::REGS_SOFTMAX>();
    // --------------------------------------------------------- softmax groups
    const int g = (warp - 4) >> 2;  // group: pairs g, g + NG, ... of the CTA
    const int wq = warp & 3;        // lane quarter
    const int stid = threadIdx.x - 128;  // thread of the softmax warpgroups, 0 .. 128 NG - 1
    const int tile = lane >> 4, l16 = lane & 15;
    const int pr0 = (wq >> 1) * PQ + (l16 >> 2);  // query row inside the tile
    const int pc0 = (wq & 1) * PQ + (l16 & 3);    // query column inside the tile
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const float c = p.scale_log2;
    const T* rpb = static_cast<const T*>(p.rpb);
    Meeting tmeet{bar_tbl(), 0u, abort_flag, p.status};
    // The table holds the bias of one head.  It is (re)built by both groups
    // together before the first pair and before every pair whose head
    // differs from the previous pair's; every group takes part in every
    // rebuild, in pair order, after finishing its pairs before that point.
    // With a grid that is a multiple of the head count a CTA meets one head
    // and builds the table once.
    int next_change = 0, prev_h = -1;
    auto rebuild_until = [&](int last) -> bool {
      for (; next_change <= last; ++next_change) {
        const int h = decode_pair<KS>(unit(next_change), p).h;
        if (h == prev_h) continue;
        prev_h = h;
        constexpr int span = 2 * KS - 1;
        constexpr int PER = (C::RAW + 128 * NG - 1) / (128 * NG);
        T rv[PER];
#pragma unroll
        for (int m = 0; m < PER; ++m) {
          const int idx = stid + 128 * NG * m;
          rv[m] = (idx < C::RAW && rpb) ? rpb[(size_t)h * C::RAW + idx] : T(0.f);
        }
        if (!tmeet.sync()) return false;  // every read of the previous table is done
#pragma unroll
        for (int m = 0; m < PER; ++m)
          if (stid + 128 * NG * m < C::RAW) raw[stid + 128 * NG * m] = rv[m];
        if (!tmeet.sync()) return false;  // raw is visible
        // copy 0, one table column per thread
        for (int col = stid; col < C::TBL_W; col += 128 * NG) {
          const int blk = col / (KS + C::PAD), off = col % (KS + C::PAD);
          const bool live = blk < KS && off >= C::PAD;
          const int bc = blk + (off - C::PAD);
#pragma unroll 1
          for (int row = 0; row < C::TBL_ROWS; ++row)
            tbl[row * C::TBL_W + col] = (live && row < span) ? raw[row * span + bc] : neg_inf<T>();
        }
        if (!tmeet.sync()) return false;  // copy 0 is complete
        // copies 1..: entry y of copy q is entry y + q of copy 0 (-inf past
        // its end), four entries per 8-byte store, shifted out of two
        // aligned 8-byte loads of copy 0
        if constexpr (C::TBL_COPIES > 1) {
          constexpr int QUADS = C::TBL_N / 4;
          const uint32_t ninf2 = bits16(neg_inf<T>()) * 0x10001u;
          for (int u = stid; u < (C::TBL_COPIES - 1) * QUADS; u += 128 * NG) {
            const int q = 1 + u / QUADS, y = (u - (q - 1) * QUADS) * 4;
            const uint2 lo = *reinterpret_cast<const uint2*>(tbl + y);
            const uint2 hi = y + 4 < C::TBL_N ? *reinterpret_cast<const uint2*>(tbl + y + 4) : make_uint2(ninf2, ninf2);
            const uint32_t w[4] = {lo.x, lo.y, hi.x, hi.y};
            const int k = q >> 1, sh = (q & 1) * 16;
            *reinterpret_cast<uint2*>(tbl + C::tbl_base(q) + y) =
                make_uint2(__funnelshift_r(w[k], w[k + 1], sh), __funnelshift_r(w[k + 1], w[k + 2], sh));
          }
          if (!tmeet.sync()) return false;
        }
      }
      return true;
    };
    uint32_t sphase = 0;  // parity of this group's next wait on each slot's s_full
    int use = 0;
    bool ok = true;
    for (int n = g; n < n_mine && ok; n += NG, ++use) {
      if (!(ok = rebuild_until(n))) break;
      const Pair pr = decode_pair<KS>(unit(n), p);
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
      // this lane's table origin, in the copy where its entries are aligned
      const int cq = colbase & (C::TBL_COPIES - 1);
      const T* tl = tbl + C::tbl_base(cq) + colbase - cq;
      float l = 0.f;
#pragma unroll 1
      for (int ch = 0; ch < NCH; ++ch) {
        const int jj = n * NCH + ch, sl = jj % NSL;
        if (!(ok = mbar_wait(bar_s_full(sl, g), (sphase >> sl) & 1, abort_flag, p.status))) break;
        sphase ^= 1u << sl;
        tc_fence_after();
        const uint32_t sbuf = tmem + lane_base + C::s_col(sl);
        l += softmax_dispatch<T, KS, D>(pb, pe, sbuf, tl, ch * C::CR, ch * C::CR + C::chunk_rows(ch), u_r0, u_r1,
                                        wr0, er, c);
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(bar_p_full(sl, n & 1));
      }
      if (!ok) break;
      // the row sum goes to the epilogue warpgroup through shared memory
      if (!(ok = mbar_wait(bar_l_empty(g, use & 1), ((use >> 1) & 1) ^ 1, abort_flag, p.status))) break;
      lsums[(g * 2 + (use & 1)) * 128 + wq * 32 + lane] = l;
      warp_arrive(bar_l_full(g, use & 1));
    }
    // take part in the table rebuilds of the other groups' remaining pairs
    if (ok) rebuild_until(n_mine - 1);
  } else {
    if constexpr (C::REGS_EPI < C::LAUNCH_REGS) regs_dec<C::REGS_EPI>();
    else regs_inc<C::REGS_EPI>();
    // ------------------------------------------------------------ epilogue
    // Every pair of the CTA in order: O / l, rounded to T, stored.  O holds
    // tile A's d columns, then tile B's.  A query whose row sum left the
    // fast path's range is recomputed exactly instead.
    using E = Shift<T>;
    const int wq = warp & 3;
    const int tile = lane >> 4, l16 = lane & 15;
    const int pr0 = (wq >> 1) * PQ + (l16 >> 2);
    const int pc0 = (wq & 1) * PQ + (l16 & 3);
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    T* out = static_cast<T*>(p.out);
    for (int n = 0; n < n_mine; ++n) {
      const int g = n % NG, use = n / NG, o = n & 1;
      const Pair pr = decode_pair<KS>(unit(n), p);
      const int i = (tile ? pr.i0[1] : pr.i0[0]) + pr0, j = (tile ? pr.j0[1] : pr.j0[0]) + pc0;
      const bool valid = i < p.H && j < p.W && (tile == 0 || pr.has_b);
      const int bq = tile ? pr.b[1] : pr.b[0];
      T* dst = out + ((((size_t)bq * p.heads + pr.h) * p.H + min(i, p.H - 1)) * p.W + min(j, p.W - 1)) * D;
      if (!mbar_wait(bar_l_full(g, use & 1), (use >> 1) & 1, abort_flag, p.status)) break;
      const float l = lsums[(g * 2 + (use & 1)) * 128 + wq * 32 + lane];
      warp_arrive(bar_l_empty(g, use & 1));
      const bool fast = l >= E::kLo && l <= E::kHi;  // false for NaN too
      const float inv = 1.f / l;
      if (!mbar_wait(bar_o_full(o), (n >> 1) & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t obuf = tmem + lane_base + C::o_col(o);
#pragma unroll
      for (int cc = 0; cc < D; cc += 16) {
        uint32_t oa[16], ob[16];
        tmem_ld16(obuf + cc, oa);
        tmem_ld16(obuf + D + cc, ob);
        tmem_wait_ld_regs(oa);
        tmem_wait_ld_regs(ob);
        if (cc + 16 >= D) {
          tc_fence_before();
          warp_arrive(bar_o_empty(o));
        }
        if (valid && fast) {
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
      if (valid && !fast) exact_query<T, KS, D>(p, bq, pr.h, i, j, dst);
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

// The five tensor maps of a launch (q tiles; k and v pair halos; k and v
// single-tile halos).  A map is a pure function of the base address, the
// shape, the element type and the box, so encoded maps are kept in a small
// cache keyed by exactly those and reused by later calls on the same
// buffers; eager callers then skip five encodings per call.
struct MapSet {
  CUtensorMap q, k, v, k1, v1;
};
struct MapKey {
  int dev;
  const void *q, *k, *v;
  int B, heads, H, W, d, ks;
  bool bf16;
  bool operator==(const MapKey& o) const {
    return dev == o.dev && q == o.q && k == o.k && v == o.v && B == o.B && heads == o.heads && H == o.H &&
           W == o.W && d == o.d && ks == o.ks && bf16 == o.bf16;
  }
};
constexpr int kMapCache = 16;
std::mutex g_map_mu;
MapKey g_map_keys[kMapCache];
MapSet g_map_vals[kMapCache];
int g_map_used = 0, g_map_next = 0;

template <int KS, int D>
bool get_maps(MapSet* out, int dev, const void* q, const void* k, const void* v, const Shape& s, bool bf16) {
  using C = Cfg<KS, D>;
  const MapKey key{dev, q, k, v, s.B, s.heads, s.H, s.W, s.d, s.ks, bf16};
  std::lock_guard<std::mutex> lk(g_map_mu);
  for (int e = 0; e < g_map_used; ++e)
    if (g_map_keys[e] == key) {
      *out = g_map_vals[e];
      return true;
    }
  MapSet m;
  if (!make_map(&m.q, q, s, bf16, PQ, PQ) || !make_map(&m.k, k, s, bf16, C::HW, C::HHP) ||
      !make_map(&m.v, v, s, bf16, C::HW, C::HHP) || !make_map(&m.k1, k, s, bf16, C::HW, C::HS) ||
      !make_map(&m.v1, v, s, bf16, C::HW, C::HS))
    return false;
  const int e = g_map_next;
  g_map_keys[e] = key;
  g_map_vals[e] = m;
  g_map_next = (g_map_next + 1) % kMapCache;
  if (g_map_used < kMapCache) ++g_map_used;
  *out = m;
  return true;
}

int sm_count(int dev) {
  static int counts[64] = {};
  if (dev < 0 || dev >= 64) return 0;
  if (!counts[dev]) cudaDeviceGetAttribute(&counts[dev], cudaDevAttrMultiProcessorCount, dev);
  return counts[dev];
}

template <typename T, int KS, int D>
cudaError_t launch(const void* q, const void* k, const void* v, const void* rpb, void* out, const Shape& s,
                   unsigned* status, cudaStream_t st) {
  using C = Cfg<KS, D>;
  constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  MapSet maps;
  if (!get_maps<KS, D>(&maps, dev, q, k, v, s, bf16)) return cudaErrorInvalidValue;
  auto kern = na2d_fwd_tc_kernel<T, KS, D>;
  static std::mutex mu;
  static bool attr_set[64] = {};
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_set[dev]) {
      // The run-time register split (setmaxnreg) must fit what the CTA is
      // launched with, or its warpgroups would wait for registers forever.
      cudaFuncAttributes fa;
      cudaError_t e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return e;
      if (C::REGS_CTRL * 128 + C::REGS_EPI * 128 + C::REGS_SOFTMAX * 128 * C::NG > fa.numRegs * C::THREADS)
        return cudaErrorInvalidConfiguration;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  Params p;
  p.q = q;
  p.k = k;
  p.v = v;
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
  const int sms = sm_count(dev);
  if (sms <= 0) return cudaErrorInvalidDevice;
  // CTA c takes units c, c + G, ...; with G a multiple of the head count
  // every unit of a CTA has head c % heads, so each CTA builds its bias
  // table once (G = 144 of 148 SMs for 8 or 16 heads).
  const int G = s.heads <= sms ? sms / s.heads * s.heads : sms;
  const int grid = p.total < G ? p.total : G;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(maps.q, maps.k, maps.v, maps.k1, maps.v1, p);
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
