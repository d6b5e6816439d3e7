// Hard selection and dictionary preparation kernels.
//
// Selection follows the Flash PD-SSM page, Technical Summary, Methodology 1
// and 2: each step's K scores pick the single highest-scoring dictionary
// matrix (hard argmax in the forward pass). Ties go to the lowest k, +0 and
// -0 compare equal and the first NaN wins, so the result is one exact integer
// per row.
//
// Dictionary preparation turns each one-hot-column matrix P_k (Methodology 1:
// "a one-hot column selector"), stored as idx[k][j], into its preimage lists:
// for every row i, the columns j with idx[k][j] == i in increasing j. With
// them the scan gathers H'[i] = sum_{j in pre(i)} d[j] H[j] instead of
// scattering, in a fixed summation order.
#include "launch.h"

namespace pdssm {

template <typename TL>
__global__ void __launch_bounds__(256) select_kernel(const TL *__restrict__ logits, int64_t rows,
                                                     int K, int32_t *__restrict__ s) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const TL *row = logits + r * K;
  float best = ldf(row);
  int bi = 0;
  if (!(best != best)) {
    for (int k = 1; k < K; ++k) {
      const float v = ldf(row + k);
      if (v != v) {  // NaN: the first one wins
        bi = k;
        break;
      }
      if (v > best) {
        best = v;
        bi = k;
      }
    }
  }
  s[r] = bi;
}

cudaError_t launch_select(int logits_t, const void *logits, int64_t rows, int K, int32_t *s,
                          cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (rows + threads - 1) / threads;
  cudaError_t e = trace_before(st, "select");
  if (e != cudaSuccess) return e;
  if (logits_t == PDSSM_BF16)
    select_kernel<<<(unsigned)blocks, threads, 0, st>>>((const __nv_bfloat16 *)logits, rows, K, s);
  else
    select_kernel<<<(unsigned)blocks, threads, 0, st>>>((const float *)logits, rows, K, s);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

// One block per dictionary entry k, one thread per row / column (N <= 128).
__global__ void __launch_bounds__(128) prep_dict_kernel(const int32_t *__restrict__ idx, int N,
                                                        int32_t *__restrict__ idx_out,
                                                        int32_t *__restrict__ off,
                                                        int32_t *__restrict__ src,
                                                        uint32_t *err) {
  __shared__ int32_t sidx[PDSSM_MAX_N];
  __shared__ int32_t soff[PDSSM_MAX_N + 1];
  const int k = blockIdx.x, i = threadIdx.x;
  if (i < N) {
    int v = idx[(int64_t)k * N + i];
    if (v < 0 || v >= N) {
      flag_error(err, kErrIdxRange);
      v = 0;
    }
    sidx[i] = v;
    idx_out[(int64_t)k * N + i] = v;
  }
  __syncthreads();
  int cnt = 0;
  if (i < N)
    for (int j = 0; j < N; ++j) cnt += (sidx[j] == i);
  // exclusive prefix sum of the counts over rows (N <= 128, two passes)
  if (i < N) soff[i + 1] = cnt;
  if (i == 0) soff[0] = 0;
  __syncthreads();
  if (i == 0)
    for (int r = 1; r <= N; ++r) soff[r] += soff[r - 1];
  __syncthreads();
  if (i < N) off[(int64_t)k * (N + 1) + i] = soff[i];
  if (i == 0) off[(int64_t)k * (N + 1) + N] = soff[N];
  if (i < N) {
    int o = soff[i];
    for (int j = 0; j < N; ++j)
      if (sidx[j] == i) src[(int64_t)k * N + o++] = j;
  }
}

cudaError_t launch_prep_dict(const int32_t *idx, int K, int N, const Workspace &ws,
                             cudaStream_t st) {
  cudaError_t e = trace_before(st, "prep_dict");
  if (e != cudaSuccess) return e;
  prep_dict_kernel<<<K, 128, 0, st>>>(idx, N, ws.idx, ws.csr_off, ws.csr_src, ws.err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

}  // namespace pdssm
