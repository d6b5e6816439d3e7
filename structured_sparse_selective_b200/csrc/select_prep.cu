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
#include <climits>

#include <algorithm>

#include "launch.h"

namespace pdssm {


// Warp-level selection. A row of K logits occupies G = 2^g lanes of a warp
// (32 / G rows per warp and pass). Vector form (kVec): the row is a whole
// number of 16-byte chunks, lane i of the group loads chunks i, i + G, ... with
// 128-bit loads, so a warp reads consecutive rows as one contiguous run.
// Scalar form: lane i of the group reads logits i, i + G, ... (any K).
// Each lane keeps its local winner, then the group merges by butterfly.
template <typename TL, bool kVec>
__global__ void __launch_bounds__(256) select_kernel(const TL *__restrict__ logits, int64_t rows,
                                                     int K, int lg, int32_t *__restrict__ s) {
  constexpr int kPer = 16 / (int)sizeof(TL);  // logits per 16-byte chunk
  const int G = 1 << lg;
  const int lane = threadIdx.x & 31, sub = lane & (G - 1);
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int rows_per_warp = 32 >> lg;
  for (int64_t r0 = warp * rows_per_warp; r0 < rows; r0 += nwarps * rows_per_warp) {
    const int64_t r = r0 + (lane >> lg);
    float bv = 0.f;
    int bk = INT_MAX;
    if (r < rows) {
      const TL *row = logits + r * K;
      if constexpr (kVec) {
        const int chunks = K / kPer;
        for (int c = sub; c < chunks; c += G) {
          const uint4 q = __ldg(reinterpret_cast<const uint4 *>(row) + c);
          const TL *e = reinterpret_cast<const TL *>(&q);
#pragma unroll
          for (int u = 0; u < kPer; ++u) sel_merge(bv, bk, to_f32(e[u]), c * kPer + u);
        }
      } else {
        for (int k = sub; k < K; k += G) sel_merge(bv, bk, ldf(row + k), k);
      }
    }
    for (int o = 1; o < G; o <<= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
      sel_merge(bv, bk, ov, ok);
    }
    if (r < rows && sub == 0) s[r] = bk;
  }
}

cudaError_t launch_select(int logits_t, const void *logits, int64_t rows, int K, int32_t *s,
                          cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const size_t esz = logits_t == PDSSM_BF16 ? 2 : 4;
  const bool vec = (K * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0;
  // lanes per row: one per 16-byte chunk (vector form) or per logit (scalar form), at most 32
  const int per_row = vec ? (int)(K * esz / 16) : K;
  int lg = 0;
  while ((1 << lg) < per_row && lg < 5) ++lg;
  const int threads = 256;
  const int64_t rows_per_block = (threads / 32) * (32 >> lg);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // enough blocks for every row, capped at 16 resident-size waves of the GPU
  const int64_t blocks = std::min<int64_t>((rows + rows_per_block - 1) / rows_per_block, (int64_t)sms * 8 * 16);
  cudaError_t e = trace_before(st, "select");
  if (e != cudaSuccess) return e;
  if (logits_t == PDSSM_BF16) {
    auto p = static_cast<const __nv_bfloat16 *>(logits);
    if (vec) select_kernel<__nv_bfloat16, true><<<(unsigned)blocks, threads, 0, st>>>(p, rows, K, lg, s);
    else select_kernel<__nv_bfloat16, false><<<(unsigned)blocks, threads, 0, st>>>(p, rows, K, lg, s);
  } else {
    auto p = static_cast<const float *>(logits);
    if (vec) select_kernel<float, true><<<(unsigned)blocks, threads, 0, st>>>(p, rows, K, lg, s);
    else select_kernel<float, false><<<(unsigned)blocks, threads, 0, st>>>(p, rows, K, lg, s);
  }
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
