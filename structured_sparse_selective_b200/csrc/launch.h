// Host-side launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace pdssm {

// Everything a scan launch needs; validated and laid out by the C-ABI layer.
struct ScanArgs {
  int64_t Bt, L, H, N, P, K;
  int64_t T, nC;  // chunk length and chunk count
  int d_t, in_t, out_t, logits_t;
  bool cplx;
  const int32_t *s;        // selections (device; null when the scan selects from logits)
  const int32_t *idx;      // caller's dictionary [K][N]
  const void *logits;      // logits when the scan selects by itself (may be null)
  const uint8_t *steps = nullptr;  // per-step transitions [Bt][L][H][N] (the original PD-SSM), or null
  int32_t *s_out;          // where a fused select stores s (may be null)
  const void *d, *B, *C, *x, *h0;
  void *y, *h_final;
  int32_t *prod_idx;
  void *prod_val;
  Workspace ws;
  bool short_waits = false;  // PDSSM_FLAG_SHORT_WAITS: the fused kernel's role waits give up after ~1 us
  bool head_dicts = false;   // PDSSM_FLAG_HEAD_DICTS: idx is [H][K][N]; head h's entry k is h * K + k
};

// Records the caller's trace events around a launch (no-op unless tracing).
cudaError_t trace_before(cudaStream_t st, const char *kernel_name);
cudaError_t trace_after(cudaStream_t st);

cudaError_t launch_select(int logits_t, const void *logits, int64_t rows, int K, int32_t *s,
                          cudaStream_t st);
cudaError_t launch_prep_dict(const int32_t *idx, int K, int N, const Workspace &ws,
                             cudaStream_t st);
// The plain three-kernel chunked scan (phases A, B, C as separate launches).
cudaError_t launch_chunked_scan(const ScanArgs &a, cudaStream_t st);
// The fused single-kernel forward pass (real state, N = P = 64, bf16 d/B/C/x).
// fused_scan_applies decides from the problem alone (shape, dtypes, chunk,
// flags); fused_scan_pointers_ok checks the 16-byte alignment its vector
// loads need. The fused kernel needs no workspace beyond the error word.
bool fused_scan_applies(const pdssm_problem *pb);
bool fused_scan_pointers_ok(const ScanArgs &a);
cudaError_t launch_fused_scan(const ScanArgs &a, cudaStream_t st);
// Outputs of an empty sequence (L == 0): h_final = h0 (or 0), prod = identity.
cudaError_t launch_empty_outputs(const ScanArgs &a, cudaStream_t st);
// Phases A and B of the chunked scan only: chunk_state[c] ends as the state after
// chunk c (the carry), h_final / prod_* written when given; no outputs, no y_loc
// (ws.y_loc may be null).
cudaError_t launch_chunked_carries(const ScanArgs &a, cudaStream_t st);

// Fused projection and selection on the tensor cores, and dictionary construction
// by column-wise hardmax (csrc/select_gemm.cu).
bool proj_select_supported(int64_t D, int64_t H, int64_t K);
size_t proj_select_smem_bytes(int64_t H, int64_t K);
cudaError_t launch_proj_select(int64_t rows, int64_t D, int64_t H, int64_t K, const void *u, const void *W,
                               int32_t *s, float *logits, uint32_t *err, cudaStream_t st);
cudaError_t launch_dict_hardmax(int64_t K, int N, const float *M, int32_t *idx, cudaStream_t st);
// The original PD-SSM's soft selection (convex mixture + column-wise hardmax) per step.
bool soft_select_supported(int64_t N, int64_t K);
size_t soft_select_ws_bytes(int64_t dicts, int64_t N, int64_t K);
cudaError_t launch_soft_select(int64_t rows, int64_t H, int64_t N, int64_t K, int logits_t, const void *logits,
                               const float *M, bool head_dicts, float tau, void *prep, uint8_t *steps, uint32_t *err,
                               cudaStream_t st);

// Everything a backward launch needs (real or complex state; h0, dh_final, dd,
// dh0 and the checkpoints are of the state type); validated by the C-ABI layer.
struct ScanBwdArgs {
  int64_t Bt, L, H, N, P, K;
  int d_t, in_t, out_t, logits_t;
  float tau;
  const int32_t *s;
  const void *logits, *d, *B, *C, *x, *dy;
  const void *h0, *dh_final;
  void *ckpt, *scratch;
  float *dlogits, *dB, *dC, *dx;
  void *dd, *dh0;
  Workspace ws;  // err, idx, csr_off, csr_src
  bool head_dicts = false;  // PDSSM_FLAG_HEAD_DICTS: dictionary entries h * K + k
  int64_t nPB = 1;          // column blocks per sequence (scan_bwd_column_blocks)
  void *pdd = nullptr;      // with nPB > 1: the blocks' shares [nPB][rows][N] (state type),
  float *pdB = nullptr, *pdC = nullptr;  // [nPB][rows][N]
  float *pdpi = nullptr;                 // [nPB][rows][K]
};
// Shared memory of one backward block, checkpoints of a sequence, and the steps
// between checkpoints (the per-sequence scratch holds that many states).
size_t scan_bwd_smem_bytes(int64_t N, int64_t P, int64_t K, bool cplx);
int64_t scan_bwd_checkpoints(int64_t L);
int64_t scan_bwd_scratch_steps();
// Blocks a sequence's columns are split over (a power of two dividing P).
int64_t scan_bwd_column_blocks(int64_t slices, int64_t P, bool cplx);
cudaError_t launch_scan_bwd(const ScanBwdArgs &a, cudaStream_t st);

}  // namespace pdssm
