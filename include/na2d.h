/*
 * na2d.h -- C ABI of the B200 (sm_100a) 2D Neighborhood Attention library.
 *
 * The operator (Neighborhood Attention Transformer, Sec. 3.1, Eqs. (2)-(4);
 * restated in the Qiita write-up "NAT: sliding-window attention", section
 * "Neighborhood Attention (NA)"): for every query pixel (i, j) of an H x W
 * map, per batch entry and head,
 *
 *   A_n    = q(i,j) . k(r_n,t_n) + B[h][r_n - i + ks - 1][t_n - j + ks - 1]   Eq. (2)
 *   out    = sum_n softmax(A / sqrt(d))_n * v(r_n,t_n)                      Eqs. (3)-(4)
 *
 * over the ks x ks window r_n in [si, si+ks), t_n in [sj, sj+ks) with
 * si = clamp(i - ks/2, 0, H - ks) and sj = clamp(j - ks/2, 0, W - ks)
 * (Sec. 1 and App. C: every pixel keeps the same span, corner pixels get a
 * window that is not centred on them).  The scale 1/sqrt(d) applies to the
 * bias too, as Eq. (4) divides all of A.  Window entries are numbered
 * row-major, n = a*ks + c for key (si + a, sj + c).
 *
 * Layouts (contiguous, C order, innermost last):
 *   q, k, v, out : [B][heads][H][W][d]      element type given by na_dtype
 *   rpb          : [heads][2*ks-1][2*ks-1]  same element type as q; may be NULL (zero bias,
 *                                           the "no RPB" setting of App. B.1)
 *   attn         : [B][heads][H][W][ks*ks]  always float32
 *
 * Ownership: the caller allocates and owns every buffer.  Device pointers
 * must point to device memory of the current CUDA device and be 16-byte
 * aligned.  The library allocates no memory in any call (cuBLAS allocates
 * its handle's state at the first na2d_block_forward on a device); it keeps only a
 * per-device status word (a static device variable), encoded TMA
 * descriptors passed by value to its kernels, and the fixed staging array
 * of na2d_forward_host_noalloc (a static device variable).
 *
 * Streams: every call that takes `stream` (a cudaStream_t passed as void*,
 * NULL meaning the legacy default stream) only enqueues work on it and
 * returns; results are ready once the stream has been synchronised.
 *
 * An empty batch (B == 0 or heads == 0) is a no-op that returns NA_OK
 * without looking at the buffer pointers (they may be NULL).
 *
 * Errors: argument errors are detected on the host before anything is
 * enqueued and returned synchronously (NA_ERR_INVALID_ARG); shapes the
 * library does not handle return NA_ERR_UNSUPPORTED; a failed launch or
 * copy returns NA_ERR_CUDA.  Kernels never trap: a device-side wait that
 * exceeds its time limit records NA_ERR_DEVICE_TIMEOUT in the status word,
 * the kernel cleans up and returns, and na2d_device_status() reports it.
 */
#ifndef NA2D_H
#define NA2D_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NA_OK = 0,
    NA_ERR_INVALID_ARG = 1,
    NA_ERR_UNSUPPORTED = 2,
    NA_ERR_CUDA = 3,
    NA_ERR_DEVICE_TIMEOUT = 4
} na_status;

typedef enum { NA_F32 = 0, NA_F16 = 1, NA_BF16 = 2 } na_dtype;

/* Argument rules shared by the calls below: B >= 0 and heads >= 0 (either 0
 * is an empty batch and a no-op); H, W >= 1; d in {16, 32, 64, 128}; ksize odd,
 * 1 <= ksize <= min(H, W, 63); B*heads*H*W*max(d, ksize^2) < 2^62. */

/*
 * QK + B -- Eq. (2), the "QK+RPB" step of NATTEN (NAT paper Sec. 3.2;
 * Qiita section "NATTEN": the library computes QK+B and AV separately).
 * Writes the UNSCALED logits A (bias included, not divided by sqrt(d)) as
 * float32 to attn [B][heads][H][W][ks*ks].  q, k, rpb are read-only.
 */
na_status na2d_qk_rpb(const void *q, const void *k, const void *rpb, float *attn,
                      int B, int heads, int H, int W, int d, int ksize,
                      na_dtype dt, void *stream);

/*
 * Softmax of Eq. (4), in place: each row of ksize*ksize entries of attn
 * [B][heads][H][W][ks*ks] becomes softmax(scale * row) (the maximum is
 * subtracted first).  Call with scale = 1/sqrt(d) between na2d_qk_rpb and
 * na2d_av to obtain Eq. (4).
 */
na_status na2d_softmax(float *attn, int B, int heads, int H, int W, int ksize,
                       float scale, void *stream);

/*
 * AV -- Eqs. (3)-(4) with given weights: out(i,j) = sum_n attn[i][j][n] * v(r_n, t_n),
 * attn float32 [B][heads][H][W][ks*ks], v and out [B][heads][H][W][d] of type dt.
 * Accumulates in float32 (float64 for NA_F32) and rounds to dt (nearest-even).
 */
na_status na2d_av(const float *attn, const void *v, void *out,
                  int B, int heads, int H, int W, int d, int ksize,
                  na_dtype dt, void *stream);

/*
 * Fused NA forward -- Eqs. (2)-(4) in one pass, out = NA_ks(q, k, v, rpb).
 * fp16/bf16: tensor-core (tcgen05) logits and weighted sum with float32
 * accumulation, softmax in float32, probabilities rounded to dt for the
 * weighted sum, output rounded to dt.  fp32: float64 accumulation, output
 * rounded to float32.  Nothing is materialised in global memory but out.
 */
na_status na2d_forward(const void *q, const void *k, const void *v, const void *rpb, void *out,
                       int B, int heads, int H, int W, int d, int ksize,
                       na_dtype dt, void *stream);

/*
 * Backward of na2d_forward: the gradients of a scalar loss L with respect to
 * q, k, v and the bias table, given dout = dL/d(out).  NATTEN provides these
 * for its "QK+B" and "AV" steps (Qiita write-up, section "NATTEN"); the NAT
 * paper, Sec. 3.2, makes the operator an autograd function.  With
 * P = softmax(A / sqrt(d)) over each query's window (Eqs. (2)-(4)):
 *
 *   dP_n = dout . v_n,  dA_n = P_n (dP_n - sum_m P_m dP_m) / sqrt(d),
 *   dq = sum_n dA_n k_n,  dk(key) and dv(key) = sums over the queries whose
 *   window holds the key of dA q and P dout,  drpb[h][displacement] = sum of
 *   dA over all queries and window entries at that displacement.
 *
 * dout, dq, dk, dv: [B][heads][H][W][d] of type dt; dq, dk, dv are written,
 * not accumulated into.  drpb: float32 [heads][2*ks-1][2*ks-1], written; NULL
 * skips the bias gradient (which is defined whether rpb is NULL or not: a
 * NULL rpb is a zero bias).  workspace: a 16-byte aligned device buffer of
 * at least na2d_backward_workspace_bytes() bytes that the caller owns; its
 * contents on entry do not matter (it holds two float64 per query between
 * the passes).  Accumulation is float64 for NA_F32 and float32 for the
 * 16-bit types; results are rounded to dt (drpb to float32).  The logits are
 * recomputed from q, k and rpb: nothing from the forward call is needed.
 */
size_t na2d_backward_workspace_bytes(int B, int heads, int H, int W, int d, int ksize, na_dtype dt);
na_status na2d_backward(const void *q, const void *k, const void *v, const void *rpb, const void *dout,
                        void *dq, void *dk, void *dv, float *drpb, void *workspace, size_t workspace_bytes,
                        int B, int heads, int H, int W, int d, int ksize, na_dtype dt, void *stream);

/*
 * SASA (stand-alone self-attention): every query attends to its CENTRED
 * ks x ks window, positions outside the map being zero padding (zero key
 * and value; the table's bias still applies at every window position).
 * The NAT paper, Sec. 3.2, calls SASA NA on a zero-padded input, and the
 * Qiita write-up's SASA/NA drawing shows the two windows at the borders;
 * that is how this call computes it: q, k and v are padded by ks/2 zero
 * pixels on every side into the workspace, na2d_forward runs on the padded
 * map, and the original pixels' outputs are written to out.
 *
 * Layouts, dtypes, rpb and errors as na2d_forward, except that ksize may
 * exceed H and W (odd, 1 .. 63).  workspace: a 256-byte aligned device
 * buffer of at least na2d_sasa_workspace_bytes() bytes that the caller owns
 * (the padded q, k, v and output); its contents on entry do not matter.
 */
size_t na2d_sasa_workspace_bytes(int B, int heads, int H, int W, int d, int ksize, na_dtype dt);
na_status na2d_sasa_forward(const void *q, const void *k, const void *v, const void *rpb, void *out,
                            void *workspace, size_t workspace_bytes,
                            int B, int heads, int H, int W, int d, int ksize,
                            na_dtype dt, void *stream);

/*
 * An NA block: the query/key/value projection, neighborhood attention, and
 * the output projection (NAT App. A.1: linear projections for queries,
 * keys and values followed by a final linear projection; the Qiita
 * write-up's "計算量" counts the block as 4hwd^2 + 2hwdk^2):
 *
 *   qkv = x Wqkv + bqkv,  q | k | v = its three C-channel thirds (each heads x dh),
 *   o = NA_ks(q, k, v, rpb) per head,  y = o Wo + bo,   C = heads * dh.
 *
 * x, y: [B][H][W][C]; wqkv: [C][3C]; bqkv: [3C] or NULL; wo: [C][C]; bo: [C]
 * or NULL; rpb as na2d_forward; all of type dt (dh and ksize as na2d_forward's
 * d and ksize).  The projections run in cuBLAS with float32 accumulation;
 * q, k, v and o are stored in dt between the steps, y is rounded to dt.
 * workspace: a 256-byte aligned device buffer of at least
 * na2d_block_workspace_bytes() bytes that the caller owns (it also serves
 * as cuBLAS's workspace); its contents on entry do not matter.  The first
 * call on a device creates a cuBLAS handle for it (cuBLAS allocates its
 * own small state then) and keeps it; make that call before any stream
 * capture.
 */
size_t na2d_block_workspace_bytes(int B, int H, int W, int heads, int dh, int ksize, na_dtype dt);
na_status na2d_block_forward(const void *x, const void *wqkv, const void *bqkv, const void *wo, const void *bo,
                             const void *rpb, void *y, void *workspace, size_t workspace_bytes,
                             int B, int H, int W, int heads, int dh, int ksize,
                             na_dtype dt, void *stream);

/*
 * Neighborhood attention over 1, 2 or 3 axes with dilation: NATTEN's NA
 * "from 1D to 3D" (Qiita write-up, section "NATTEN"; NAT Sec. 3.2) and the
 * dilated NA of DiNAT.  The pages give no formula for dilation; this call
 * reads a dilation dl as splitting an axis into dl interleaved sub-grids
 * (positions congruent mod dl), a query attending within its own sub-grid
 * with NA's clamped window of k positions:
 *
 *   r = i mod dl, i' = i div dl, L' = ceil((L - r) / dl),
 *   start' = clamp(i' - k/2, 0, L' - k), keys at r + (start' + t) dl,
 *   bias index (start' + t) - i' + k - 1 on that axis.
 *
 * q, k, v, out: [B][heads][L0][L1][L2][d]; rpb: [heads][2k0-1][2k1-1][2k2-1]
 * or NULL; all of type dt.  1D and 2D NA are the cases L0 = k0 = 1 (and
 * L1 = k1 = 1); with every dilation 1 and L0 = k0 = 1 this is na2d_forward.
 * Arguments: every k odd, 1 .. 63; every dilation >= 1; L / dilation >= k on
 * every axis (each sub-grid holds a window); d in {16, 32, 64, 128}.
 * CUDA-core kernel with the exact row maximum; float64 accumulation for
 * NA_F32, float32 otherwise.
 */
na_status na_forward_nd(const void *q, const void *k, const void *v, const void *rpb, void *out,
                        int B, int heads, int L0, int L1, int L2, int d,
                        int k0, int k1, int k2, int dil0, int dil1, int dil2,
                        na_dtype dt, void *stream);

/*
 * na2d_forward from HOST buffers: copies q, k, v (and rpb when not NULL)
 * host-to-device into the caller's device workspace, runs na2d_forward and
 * copies the result back to out_host, one cudaMemcpyAsync per buffer and
 * batch chunk.  With B >= 2 the batch is cut into up to four chunks of whole
 * batch entries, each on a stream of the library's own, forked from and
 * joined back to `stream` with events; the chunks' input copies run one
 * after another, so that one chunk's kernel and output copy overlap the next
 * chunk's input copies.  The call is still ordered on `stream` as one
 * operation.  The library creates those four streams and their events on
 * the first such call on a device and keeps them; make that first call
 * before any stream capture.  Pinned host memory makes the copies
 * asynchronous; the host buffers must stay valid until the stream is
 * synchronised.  workspace must be a 256-byte aligned device buffer of at
 * least na2d_forward_host_workspace_bytes() bytes.
 */
size_t na2d_forward_host_workspace_bytes(int B, int heads, int H, int W, int d, int ksize,
                                         na_dtype dt);
na_status na2d_forward_host(const void *q_host, const void *k_host, const void *v_host,
                            const void *rpb_host, void *out_host,
                            void *workspace, size_t workspace_bytes,
                            int B, int heads, int H, int W, int d, int ksize,
                            na_dtype dt, void *stream);

/*
 * na2d_forward_host without a workspace argument, for callers that cannot
 * allocate device memory: for example a plugin whose host framework owns
 * every device allocation, or a caller that must not enter the driver's
 * allocator on its path.  The pages have no counterpart to this call; it is
 * a convenience of this library.
 *
 * Instead of a caller's workspace it stages the inputs and the output in one
 * fixed device array that the library reserves, NA2D_NOALLOC_SCRATCH_BYTES
 * (64 MiB) on every device that loads the library, held until the process
 * exits.  Shapes whose na2d_forward_host_workspace_bytes() exceeds that are
 * rejected with NA_ERR_UNSUPPORTED; otherwise arguments, errors and results
 * are those of na2d_forward_host.  The call allocates nothing and creates
 * nothing: every copy and the kernel run in order on `stream`.
 *
 * Every call looks up the array's device address on the current device (a
 * host-side lookup in the CUDA runtime, so a device reset between calls is
 * harmless).  The first call on a device may load the library's kernels on
 * it; make that first call before any stream capture.  All calls on a
 * device share the one array: calls whose
 * work overlaps on the GPU (different streams, or host threads) race and may
 * return wrong results.  Each call writes everything it reads from the
 * array, so the contents left by an earlier call do not matter.
 */
#define NA2D_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
na_status na2d_forward_host_noalloc(const void *q_host, const void *k_host, const void *v_host,
                                    const void *rpb_host, void *out_host,
                                    int B, int heads, int H, int W, int d, int ksize,
                                    na_dtype dt, void *stream);

/*
 * Which kernel na2d_forward launches for these arguments: 1 = tensor-core
 * (tcgen05/TMEM/TMA) kernel, 0 = SIMT kernel, negative = the arguments are
 * rejected (the negated na_status).  Host-only; enqueues nothing.
 */
int na2d_forward_kernel(int B, int heads, int H, int W, int d, int ksize, na_dtype dt);

/*
 * Synchronises `stream`, then returns and clears the status word of the
 * current device: NA_ERR_DEVICE_TIMEOUT if any kernel gave up on a bounded
 * wait since the last call, NA_ERR_CUDA if the stream reports a CUDA error,
 * NA_OK otherwise.
 */
na_status na2d_device_status(void *stream);

/*
 * Test hook for the failure path: enqueues one kernel that waits on a
 * barrier nothing ever releases, with a wait limit of timeout_us
 * microseconds (1 .. 10^6).  The wait runs out, the kernel records
 * NA_ERR_DEVICE_TIMEOUT and returns; the context stays usable.
 */
na_status na2d_debug_timeout_probe(unsigned int timeout_us, void *stream);

/* Human-readable name of a status code (static string). */
const char *na_status_str(na_status s);

#ifdef __cplusplus
}
#endif

#endif /* NA2D_H */
