/*
 * pdssm.h -- C ABI of libpdssm.so, the B200 (sm_100a) forward pass of Flash PD-SSM.
 *
 * Method: "Flash PD-SSM: Memory-Optimized Structured Sparse State-Space Models"
 * (gist.science explainer of arXiv 2605.19150), Technical Summary:
 *   - Methodology 1 ("Novel Selection Mechanism"): the input gives K scores; the
 *     single highest-scoring matrix of a dictionary of K sparse matrices is
 *     used directly. Each is a one-hot column selector, so memory is O(L*N),
 *     not the O(L*N^2) of the original PD-SSM.
 *   - Methodology 2: the forward pass uses hard argmax.
 *   - Methodology 3 ("Hardware-Aware Implementation"): a three-phase chunked
 *     scan -- A: independent sequential recurrences inside chunks; B: a prefix
 *     scan over the chunks' dependencies gives the carry states; C: the carry
 *     corrections are applied.
 * The page prints no formula. This library computes the PD (one-hot-column
 * matrix times diagonal) recurrence those passages describe:
 *     s_t = argmax_k logits_t[k]          (lowest k on ties, first NaN wins)
 *     H_t = P_{s_t} diag(d_t) H_{t-1} + B_t x_t^T,   H_{-1} = h0 (or 0)
 *     y_t = H_t^T C_t                     (plain transpose, also for complex H)
 * where P_k[idx[k][j]][j] = 1 is the only nonzero of column j. Chunks are
 * combined with the associative composition of (index, value) pairs
 *     (idx, val) o (idx', val') = (idx[idx'], val[idx'] * val')
 * which is the pair of the matrix product A * A' (A' applied first); the
 * prefix-scan framing follows the abstract of "Sequential-Parallel Duality in
 * Prefix Scannable Models" (state updates by a parallel prefix scan with a
 * custom associative operator). No N x N matrix is ever formed.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Ownership: the caller allocates every buffer, inputs, outputs and the
 *   workspace, in device memory of the device that owns `stream`. The library
 *   never allocates, frees or synchronises (pdssm_read_device_check and the
 *   PDSSM_FLAG_DEVICE_CHECK flag are the documented exceptions: they
 *   synchronise the stream).
 * Streams: every call only enqueues work on `stream` and returns. A NULL
 *   stream is the legacy default stream of the calling thread's current
 *   device. Outputs are valid once the stream has reached the call.
 * Layouts (row-major, contiguous, element-aligned):
 *   logits [batch][seqlen][heads][K]          s    [batch][seqlen][heads] int32
 *   idx    [K][N] int32, shared by all heads  (idx[k][j] = row of the nonzero
 *                                              of column j of P_k, in [0, N));
 *          [heads][K][N] with PDSSM_FLAG_HEAD_DICTS
 *   d, B, C [batch][seqlen][heads][N]         x, y [batch][seqlen][heads][P]
 *   h0, h_final [batch][heads][N][P]          prod_idx, prod_val [batch][heads][N]
 *   Complex values (PDSSM_C64) are interleaved (re, im) float pairs, the
 *   layout of torch.complex64 / std::complex<float>.
 * Errors: argument errors are reported before anything is enqueued; a
 *   non-PDSSM_OK return means nothing was launched. Launch failures return
 *   PDSSM_ERR_CUDA. Index values that the host cannot see (idx entries outside
 *   [0, N), s entries outside [0, K)) never cause an out-of-bounds access: the
 *   kernels substitute 0, set a bit in the workspace's error word and carry
 *   on; pdssm_read_device_check reports it.
 */
#ifndef PDSSM_H_
#define PDSSM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
struct CUstream_st;
typedef struct CUstream_st *pdssm_stream_t;

typedef enum {
  PDSSM_OK = 0,
  PDSSM_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misalignment */
  PDSSM_ERR_UNSUPPORTED = 2,  /* N, P or K above the limits, dtype combination */
  PDSSM_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
  PDSSM_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
  PDSSM_ERR_DEVICE_CHECK = 5, /* a kernel met an out-of-range idx or s */
  PDSSM_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up */
} pdssm_status;

typedef enum { PDSSM_F32 = 0, PDSSM_BF16 = 1, PDSSM_C64 = 2 } pdssm_dtype;

#define PDSSM_MAX_N 128
#define PDSSM_MAX_P 128
#define PDSSM_MAX_K 64

/* flags */
#define PDSSM_FLAG_DEVICE_CHECK 1u   /* synchronise and return PDSSM_ERR_DEVICE_CHECK on bad idx/s */
#define PDSSM_FLAG_REFERENCE_PATH 2u /* use the plain three-kernel chunked path (no fused kernel) */
/* Failure-detection testing: the fused kernel's bounded device waits (one role
 * waiting for another) give up after about 1 microsecond instead of 2 seconds.
 * A wait that gives up records PDSSM_ERR_TIMEOUT in the workspace's error word,
 * every role leaves its loop and the kernel returns: nothing faults or hangs, and
 * the outputs of that call are unspecified. The final wait for the kernel's own
 * tensor-core work keeps its long limit. No effect on the three-kernel path. */
#define PDSSM_FLAG_SHORT_WAITS 4u
/* Per-head dictionaries (Flash PD-SSM page, Methodology 4: multi-head layers;
 * each head may hold its own dictionary): idx is [heads][K][N] instead of the
 * shared [K][N]; head h's step t uses P_{s_t} of its own dictionary
 * idx[h][s_t]. Workspace sizes grow by the dictionary's size only. */
#define PDSSM_FLAG_HEAD_DICTS 8u

/*
 * Problem description. Supported dtype combinations:
 *   real state:    state_t = F32; d_t in {F32, BF16}; in_t (B, C, x) in {F32, BF16};
 *                  out_t (y) in {F32, BF16}; logits_t in {F32, BF16};
 *                  h0 / h_final / prod_val are F32.
 *   complex state: state_t = C64; d_t = C64; in_t in {F32, BF16}; out_t = C64;
 *                  logits_t in {F32, BF16}; h0 / h_final / prod_val are C64.
 * Sizes: batch, seqlen, heads >= 0 (zero is an empty problem);
 *        1 <= N <= PDSSM_MAX_N, 1 <= P <= PDSSM_MAX_P, 1 <= K <= PDSSM_MAX_K.
 * chunk: the chunk length T of the three-phase scan; 0 picks a default. The
 *        results do not depend on T beyond floating-point rounding.
 */
typedef struct {
  int64_t batch, seqlen, heads, N, P, K;
  int32_t chunk;
  int32_t logits_t, in_t, d_t, state_t, out_t; /* pdssm_dtype values */
  uint32_t flags;
} pdssm_problem;

/* Human-readable name of a status code (static string, never NULL). */
const char *pdssm_status_string(int32_t status);

/* Library version as "major.minor.patch" (static string). */
const char *pdssm_version(void);

/*
 * Workspace bytes that pdssm_scan_fwd / pdssm_forward need for `pb`
 * (written to *bytes). The size follows the path the problem takes:
 *   - the fused single-kernel path (real state, N = P = 64, bf16 d/B/C/x,
 *     K * sizeof(logit) a multiple of 16, chunk 0 or 16, no
 *     PDSSM_FLAG_REFERENCE_PATH) needs only the 4-byte error word (256 bytes
 *     are reported), provided logits (or s), d, B, C and x are 16-byte aligned;
 *   - every other problem takes the three-kernel path, whose workspace grows as
 *     O(batch*heads*seqlen*(N+P)) -- the O(L*N) memory of Methodology 1 -- and
 *     never with N*N.
 * A fused-path problem whose inputs are not 16-byte aligned runs on the
 * three-kernel path and needs the size reported for the same problem with
 * PDSSM_FLAG_REFERENCE_PATH set; with a smaller workspace the call returns
 * PDSSM_ERR_WORKSPACE before anything is enqueued.
 * Errors: PDSSM_ERR_INVALID_ARG / PDSSM_ERR_UNSUPPORTED as for the calls.
 */
pdssm_status pdssm_workspace_size(const pdssm_problem *pb, size_t *bytes);

/*
 * Hard selection, Methodology 1 and 2: s[b][t][h] = the lowest k with
 * logits[b][t][h][k] == max_k' logits[b][t][h][k']. +0 and -0 compare equal;
 * a NaN counts as the maximum and the first NaN wins. Bit-exact.
 * logits: device, logits_t; s: device int32 output. No workspace.
 * One row is reduced by a group of lanes of a warp; rows whose size is a
 * multiple of 16 bytes (and a 16-byte aligned logits pointer) are read with
 * 128-bit loads.
 */
pdssm_status pdssm_select(const pdssm_problem *pb, const void *logits, int32_t *s,
                          pdssm_stream_t stream);

/*
 * The PD scan (Methodology 3) for given selections s.
 *   s        device int32 [batch][seqlen][heads], each in [0, K)
 *   idx      device int32 [K][N]
 *   d        device d_t    [batch][seqlen][heads][N]
 *   B, C     device in_t   [batch][seqlen][heads][N]
 *   x        device in_t   [batch][seqlen][heads][P]
 *   h0       device state  [batch][heads][N][P], or NULL for a zero state
 *   y        device out_t  [batch][seqlen][heads][P]            (output)
 *   h_final  device state  [batch][heads][N][P], or NULL         (output)
 *   prod_idx device int32  [batch][heads][N], or NULL            (output)
 *   prod_val device state  [batch][heads][N], or NULL            (output)
 *            (prod_idx, prod_val) is the pair of P_{s_{L-1}} diag(d_{L-1}) ...
 *            P_{s_0} diag(d_0): column j has its only nonzero, prod_val[j], at
 *            row prod_idx[j]. prod_idx is exact; prod_val may underflow to 0.
 *   workspace device, >= pdssm_workspace_size bytes, 16-byte aligned. Its
 *            contents are scratch, except the error word that
 *            pdssm_read_device_check reads after the call.
 * The output buffers must not overlap the inputs or each other.
 */
pdssm_status pdssm_scan_fwd(const pdssm_problem *pb, const int32_t *s, const int32_t *idx,
                            const void *d, const void *B, const void *C, const void *x,
                            const void *h0, void *y, void *h_final, int32_t *prod_idx,
                            void *prod_val, void *workspace, size_t workspace_bytes,
                            pdssm_stream_t stream);

/*
 * Selection and scan in one call: pdssm_select followed by pdssm_scan_fwd,
 * with the selection fused into the scan's input read where the fused path
 * applies. `logits` replaces `s`; `s_out` (device int32
 * [batch][seqlen][heads], or NULL) receives the selections.
 */
pdssm_status pdssm_forward(const pdssm_problem *pb, const void *logits, const int32_t *idx,
                           const void *d, const void *B, const void *C, const void *x,
                           const void *h0, void *y, void *h_final, int32_t *prod_idx,
                           void *prod_val, int32_t *s_out, void *workspace,
                           size_t workspace_bytes, pdssm_stream_t stream);

/*
 * pdssm_forward without a caller workspace, for callers that cannot allocate
 * device memory on their call path (a plug-in whose host application already
 * owns all device memory, or a latency-critical loop that cannot afford
 * cudaMalloc's implicit synchronisation). The paper has no counterpart to
 * this entry point.
 *   Arguments are those of pdssm_forward minus workspace / workspace_bytes.
 *   The workspace is a 32 MiB array inside this library's device image,
 *   held by every GPU that loads the library until the process exits.
 *   Problems whose pdssm_workspace_size exceeds 32 MiB return
 *   PDSSM_ERR_WORKSPACE before anything is enqueued.
 *   The first call on a device looks up the array's device address (with that
 *   device current) and keeps it; make that first call before any stream
 *   capture. A lookup that fails returns PDSSM_ERR_CUDA and is retried by the
 *   next call. Problems served by the fused kernel use only the array's error
 *   word; the 32 MiB limit matters for the three-kernel path.
 *   All calls on a device share the array and it keeps the last call's
 *   contents: calls that overlap on the GPU race and must be ordered by the
 *   caller (one stream, or events). pdssm_read_device_check cannot read this
 *   workspace; PDSSM_FLAG_DEVICE_CHECK still reports out-of-range values.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
pdssm_status pdssm_forward_noalloc(const pdssm_problem *pb, const void *logits, const int32_t *idx,
                                   const void *d, const void *B, const void *C, const void *x,
                                   const void *h0, void *y, void *h_final, int32_t *prod_idx,
                                   void *prod_val, int32_t *s_out, pdssm_stream_t stream);

/*
 * Dictionary construction (Flash PD-SSM page, Technical Summary, Methodology 1:
 * the dictionary's K sparse matrices are pre-computed; the original PD-SSM makes
 * a matrix sparse by a column-wise hardmax): for each dense matrix M_k and
 * column j, idx[k][j] = the lowest i with M[k][i][j] == max_i' M[k][i'][j]
 * (a NaN counts as the maximum and the first NaN wins). Bit-exact.
 *   M    device float [K][N][N], row-major (M[k][i][j] at (k * N + i) * N + j);
 *        K may count heads x entries to build per-head dictionaries [heads][K][N]
 *   idx  device int32 [K][N] output, in [0, N)
 * Errors: PDSSM_ERR_INVALID_ARG for null pointers, K < 0, N < 1, misaligned
 * pointers; PDSSM_ERR_UNSUPPORTED for N > PDSSM_MAX_N. No workspace.
 */
pdssm_status pdssm_dict_hardmax(int64_t K, int64_t N, const float *M, int32_t *idx, pdssm_stream_t stream);

/*
 * Fused projection and selection (Methodology 1: the input u_t generates the K
 * scores by a linear transformation; Methodology 2: hard argmax). For each row
 * r = b * seqlen + t and head h:
 *   logits[r][h][k] = sum_d u[r][d] * W[d][h * K + k]
 *   s[r][h]         = the lowest k with logits[r][h][k] == max_k' logits[r][h][k']
 * The products are exact (bf16 x bf16) and the sums are fp32, accumulated on the
 * tensor cores in tensor memory; the argmax runs in the epilogue that reads the
 * accumulator, so the logits need not be written at all.
 *   pb      batch, seqlen, heads, K (N, P, chunk and the dtypes are not used)
 *   D       width of u (the embedding dimension): a positive multiple of 64
 *   u       device bf16 [batch * seqlen][D], 16-byte aligned
 *   W       device bf16 [D][heads * K], 16-byte aligned
 *   s       device int32 [batch][seqlen][heads] output (the layout pdssm_scan_fwd reads)
 *   logits  device float [batch][seqlen][heads][K] output, or NULL
 *   workspace >= 256 bytes (error word; pdssm_read_device_check reads it)
 * Requirements: K a power of two; heads * K a multiple of 32 and either at most
 * 256 or a multiple of 256. Others return PDSSM_ERR_UNSUPPORTED.
 */
pdssm_status pdssm_select_proj(const pdssm_problem *pb, int64_t D, const void *u, const void *W, int32_t *s,
                               float *logits, void *workspace, size_t workspace_bytes, pdssm_stream_t stream);

/*
 * The original PD-SSM's selection (Flash PD-SSM page, Technical Summary,
 * Methodology 1, "Original PD-SSM"; Problem Statement: its O(L N^2) memory and
 * 40x slowdown are what Flash PD-SSM removes). Built here as the contrast the
 * pages measure against: each step's transition is the column-wise hardmax of a
 * convex combination of K dense dictionary matrices,
 *   pi_t = softmax(logits_t / tau),  idx_t[j] = argmax_i sum_k pi_t[k] M_k[i][j]
 * (lowest i on ties). The mixtures are never written to memory: for 128 steps of
 * one head they are one tensor-core product [steps x K] x [K x N^2] (pi and M
 * split into bf16 hi + lo, about 16 bits) whose epilogue takes the argmax.
 *   logits    device logits_t [batch][seqlen][heads][K]
 *   M         device float [K][N][N] ([heads][K][N][N] with PDSSM_FLAG_HEAD_DICTS)
 *   tau       > 0
 *   idx_steps device uint8 [batch][seqlen][heads][N] output: row of the nonzero
 *             of column j of step t's transition
 *   workspace pdssm_soft_select_workspace_size bytes, 256-byte aligned (the error
 *             word and the dictionary in the tensor cores' bf16 layout)
 * Requirements: N a power of two in [16, 128]; K <= 64. Near-ties of the
 * mixture (within its ~2^-16 relative precision) may resolve differently from an
 * exact computation.
 */
pdssm_status pdssm_soft_select_workspace_size(const pdssm_problem *pb, size_t *bytes);
pdssm_status pdssm_soft_select(const pdssm_problem *pb, const void *logits, const float *M, float tau,
                               uint8_t *idx_steps, void *workspace, size_t workspace_bytes,
                               pdssm_stream_t stream);

/*
 * The scan with a transition given for every step (the original PD-SSM's
 * per-step matrices from pdssm_soft_select, or any per-step one-hot-column
 * transitions): H_t = P_t diag(d_t) H_{t-1} + B_t x_t^T, y_t = H_t^T C_t with
 * P_t[idx_steps[t][j]][j] = 1. Arguments as pdssm_scan_fwd with idx_steps
 * (device uint8 [batch][seqlen][heads][N], 16-byte aligned; values >= N are
 * replaced by 0 and flagged) in place of s and idx; pb->K, pb->logits_t and
 * PDSSM_FLAG_HEAD_DICTS are not used. Served by the fused kernel only (N = P =
 * 64, bf16 d/B/C/x, real state): other problems return PDSSM_ERR_UNSUPPORTED.
 * The workspace is 256 bytes (the error word).
 */
pdssm_status pdssm_scan_fwd_steps(const pdssm_problem *pb, const uint8_t *idx_steps, const void *d,
                                  const void *B, const void *C, const void *x, const void *h0, void *y,
                                  void *h_final, int32_t *prod_idx, void *prod_val, void *workspace,
                                  size_t workspace_bytes, pdssm_stream_t stream);

/*
 * Backward pass: workspace bytes for pdssm_scan_bwd. Checkpoints of the state
 * every 16 steps (the carries of the chunked forward scan at chunk length 16, with
 * their chunk pairs) plus a 16-step scratch per (batch, head) slice:
 * E * N * P * batch * heads * (ceil(L / 16) + 16) bytes (E = 4 for a real state,
 * 8 for a complex one), batch * heads * ceil(L / 16) * N * (4 + E) bytes of pairs,
 * plus the dictionary's preimage lists. When there are
 * fewer than about two sequences per SM, a sequence's columns are split over
 * several blocks (a power of two nb dividing P) and the workspace also holds each
 * block's share of the sums over columns: nb * batch * seqlen * heads *
 * (N * (E + 8) + K * 4) bytes.
 * A block holds three N x (its columns) state buffers and the dictionary in
 * shared memory; where a whole row does not fit in 227 KiB the columns are split
 * further, so every problem up to N = P = 128, K = 64 is supported, real or complex.
 */
pdssm_status pdssm_bwd_workspace_size(const pdssm_problem *pb, size_t *bytes);

/*
 * Backward pass of the scan (Flash PD-SSM page, Technical Summary,
 * Methodology 2 "Gradient Propagation": hard argmax forward, tempered softmax
 * backward through a straight-through estimator). Gradients of
 *   Loss = Re[ sum_t <dy_t, y_t> + <dh_final, H_{L-1}> ],  <a, b> = sum conj(a) b,
 * where y, H are the forward pass of pdssm_scan_fwd on the same arguments. For
 * a complex quantity z = u + i v the gradient is dLoss/du + i dLoss/dv (for a
 * real state every conjugate and real part is the identity):
 *   dd          state type [batch][seqlen][heads][N]: exact derivative,
 *               dd_t[j] = sum_p Lam_t[idx[s_t][j]][p] conj(H_{t-1}[j][p]);
 *   dB, dC      float [batch][seqlen][heads][N]: exact derivatives (real parts);
 *   dx          float [batch][seqlen][heads][P]: exact derivative (real part);
 *   dh0         state type [batch][heads][N][P] or NULL: derivative in h0;
 *   dlogits     float [batch][seqlen][heads][K] or NULL (then `logits` is NULL
 *               too): with pit = softmax(logits_t / tau) and
 *               dpi_t[k] = Re sum_j conj((Lam_t H_{t-1}^H)[idx[k][j]][j]) d_t[j]
 *               (Lam_t = dLoss/dH_t), dlogits_t = pit * (dpi_t - <pit, dpi_t>) / tau.
 * "State type" is float for state_t = PDSSM_F32 and interleaved (re, im) float
 * pairs for state_t = PDSSM_C64.
 * Inputs: s (device int32 [batch][seqlen][heads], the forward's selections),
 * idx, d, B, C, x, h0 as for pdssm_scan_fwd (h0 of the state type or NULL); dy
 * in the problem's out_t ([batch][seqlen][heads][P]); dh_final of the state
 * type [batch][heads][N][P] or NULL (zero); logits in logits_t; tau > 0.
 * Errors as pdssm_scan_fwd; the workspace is pdssm_bwd_workspace_size bytes.
 */
pdssm_status pdssm_scan_bwd(const pdssm_problem *pb, const void *logits, const int32_t *s,
                            const int32_t *idx, const void *d, const void *B, const void *C,
                            const void *x, const void *h0, const void *dy, const void *dh_final,
                            float tau, float *dlogits, void *dd, float *dB, float *dC, float *dx,
                            void *dh0, void *workspace, size_t workspace_bytes,
                            pdssm_stream_t stream);

/*
 * Synchronises `stream` and reads the error word that the last pdssm_scan_fwd,
 * pdssm_forward or pdssm_scan_bwd call on `workspace` left: PDSSM_OK,
 * PDSSM_ERR_DEVICE_CHECK (an idx or s value was out of range) or PDSSM_ERR_TIMEOUT.
 */
pdssm_status pdssm_read_device_check(const void *workspace, pdssm_stream_t stream);

/*
 * Kernel tracing (observability; the pages describe none).
 * Between pdssm_trace_begin and pdssm_trace_end, every kernel the calling
 * thread's pdssm_* calls enqueue is bracketed by cudaEventRecord of
 * events[2*i] (before) and events[2*i+1] (after) on the launch stream, for
 * the first n_events/2 launches. `events` holds cudaEvent_t handles the caller
 * created (with timing enabled) and keeps alive until it has read them; the
 * library only records them.
 * pdssm_trace_end returns the number of launches recorded and stops tracing;
 * pdssm_trace_kernel_name(i) names launch i of the last trace (static
 * string, or NULL when i is out of range).
 */
pdssm_status pdssm_trace_begin(void *const *events, int32_t n_events);
int32_t pdssm_trace_end(void);
const char *pdssm_trace_kernel_name(int32_t i);

#ifdef __cplusplus
}
#endif

#endif /* PDSSM_H_ */
