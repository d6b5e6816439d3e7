// Selection inputs that come from dense matrices (Flash PD-SSM page, Technical
// Summary, Methodology 1):
//   - the fused projection and selection: the input u_t gives the K scores of
//     each head by a linear map, logits = u W, and the highest score selects
//     (hard argmax, Methodology 2). The map is a dense contraction, so it runs on
//     the 5th-generation tensor cores (tcgen05.mma, bf16 x bf16 -> fp32 in tensor
//     memory) and the argmax is the epilogue that reads the accumulator;
//   - dictionary construction: each of the K sparse dictionary matrices is the
//     column-wise hardmax of a dense trainable matrix, idx[k][j] = argmax_i M[k][i][j].
#include <algorithm>
#include <type_traits>

#include "launch.h"
#include "sm100.cuh"

namespace pdssm {

using namespace sm100;

namespace {

constexpr int kPM = 128;       // rows per CTA: one tensor-memory lane each
constexpr int kPK = 64;        // reduction depth staged per step
constexpr int kPThreads = 128;
constexpr uint32_t kPCols = 256;  // tensor-memory columns per CTA (the widest N tile)
constexpr uint64_t kPTimeoutNs = 2000000000ull;

struct PParams {
  int64_t rows, D, HK;
  int K;      // columns per head (a power of two)
  int ntile;  // columns per CTA (MMA N): HK when HK <= 256, else 256
  const __nv_bfloat16 *u, *W;
  int32_t *s;
  float *logits;
  uint32_t *err;
};

__device__ __forceinline__ uint64_t gtimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Waits for the mbarrier phase with the given parity for at most kPTimeoutNs;
// on timeout records kErrTimeout and returns false.
__device__ __noinline__ bool pwait(uint64_t *bar, uint32_t parity, uint32_t *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 2000)) {
    if (gtimer_ns() - t0 > kPTimeoutNs) {
      flag_error(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

// The selection's winner (sel_merge's order: the first NaN, else the maximum, +0 == -0,
// the lowest index on ties) among CW consecutive values: a maximum and a search for its
// first occurrence instead of CW sequential merges.
template <int CW>
__device__ __forceinline__ void run_winner(const float *v, float &val, int &idx) {
  float m = v[0];
  bool nan = false;
#pragma unroll
  for (int c = 0; c < CW; ++c) {
    m = fmaxf(m, v[c]);
    nan |= v[c] != v[c];
  }
  idx = 0;
#pragma unroll
  for (int c = CW - 1; c >= 0; --c)
    if (nan ? v[c] != v[c] : v[c] == m) idx = c;
  // the merge looks only at whether a winner is a NaN, so any NaN stands for one (and
  // no run-time index into v, which would move it to local memory)
  val = nan ? __int_as_float(0x7fffffff) : m;
}

// One CTA: rows [row0, row0 + 128) x columns [n0, n0 + ntile) of u W, reduced over
// D in steps of 64 through two cp.async stages. Stage layouts (no swizzle, 8-row
// x 16-byte core matrices):
//   A = u tile, K-major:   (r % 8) * 16 + (r / 8) * 1024 + (k / 8) * 128 + (k % 8) * 2
//   B = W tile, MN-major:  (k % 8) * 16 + (k / 8) * (ntile * 16) + (n / 8) * 128 + (n % 8) * 2
__global__ void __launch_bounds__(kPThreads) proj_select_kernel(PParams a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int aBytes = kPM * kPK * 2, bBytes = kPK * a.ntile * 2, stBytes = aBytes + bBytes;
  uint64_t *done = reinterpret_cast<uint64_t *>(smem + 2 * stBytes);  // MMAs of a stage completed
  uint32_t *tslot = reinterpret_cast<uint32_t *>(done + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = (int64_t)blockIdx.x * kPM, n0 = (int64_t)blockIdx.y * a.ntile;
  const int nch = a.ntile / 8;  // 16-byte chunks of a W row inside the tile

  if (tid == 0) {
    mbar_init(&done[0], 1);
    mbar_init(&done[1], 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, kPCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  auto load = [&](int kt) {
    uint8_t *sA = smem + (kt & 1) * stBytes, *sB = sA + aBytes;
    const int64_t k0 = (int64_t)kt * kPK;
    for (int c = tid; c < kPM * 8; c += kPThreads) {
      const int r = c >> 3, kc = c & 7;
      uint8_t *dst = sA + (r & 7) * 16 + (r >> 3) * 1024 + kc * 128;
      if (row0 + r < a.rows)
        cp_async16(dst, a.u + (row0 + r) * a.D + k0 + kc * 8);
      else
        *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
    for (int c = tid; c < kPK * nch; c += kPThreads) {
      const int k = c / nch, nc = c - k * nch;
      cp_async16(sB + (k & 7) * 16 + (k >> 3) * (nch * 128) + nc * 128, a.W + (k0 + k) * a.HK + n0 + nc * 8);
    }
  };

  const int nk = (int)(a.D / kPK);
  const uint32_t idesc = idesc_bf16_f32(kPM, a.ntile, false, true);
  bool ok = true;
  load(0);
  cp_async_commit();
  for (int kt = 0; kt < nk; ++kt) {
    if (kt + 1 < nk) {
      // the next tile's stage was read by the MMAs of tile kt - 1
      if (kt >= 1 && ok) ok = pwait(&done[(kt - 1) & 1], ((kt - 1) >> 1) & 1, a.err);
      load(kt + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0 && ok) {
      tc_fence_after();
      const uint32_t sA = smem_u32(smem + (kt & 1) * stBytes), sB = sA + aBytes;
#pragma unroll
      for (int ks = 0; ks < kPK / 16; ++ks)
        mma_bf16(tbase, smem_desc(sA + ks * 256, 128, 1024), smem_desc(sB + ks * 2 * nch * 128, nch * 128, 128), idesc,
                 (kt | ks) != 0);
      mma_commit(&done[kt & 1]);
    }
  }
  // the last commit arrives once every MMA issued before it has completed
  const bool fin = pwait(&done[(nk - 1) & 1], ((nk - 1) >> 1) & 1, a.err);
  ok = __syncthreads_and(ok && fin);
  tc_fence_after();

  // epilogue: thread = row; argmax over each head's K columns as they stream out
  const int64_t row = row0 + warp * 32 + lane;
  const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
  const int64_t heads = a.HK / a.K;
  // each head's K scores by runs of CW = min(K, 32) consecutive columns: the run's
  // winner, merged into the head's (one instantiation of the loop per CW, so that the
  // loaded columns stay in registers)
  auto epilogue = [&](auto cw_tag) {
    constexpr int CW = decltype(cw_tag)::value;
    float bv = 0.f;
    int bk = INT_MAX;
    for (int c0 = 0; c0 < a.ntile; c0 += 32) {
      float v[32];
      tmem_ld32(tl + c0, v);
      tmem_wait_ld();
      if (ok && row < a.rows) {
        if (a.logits) {
          float4 *dst = reinterpret_cast<float4 *>(a.logits + row * a.HK + n0 + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
#pragma unroll
        for (int h0 = 0; h0 < 32; h0 += CW) {
          float cv;
          int ci;
          run_winner<CW>(v + h0, cv, ci);
          const int k0 = (c0 + h0) & (a.K - 1);
          if (k0 == 0) {
            bv = cv;
            bk = ci;
          } else {
            sel_merge(bv, bk, cv, k0 + ci);
          }
          if (k0 + CW == a.K) a.s[row * heads + (n0 + c0 + h0) / a.K] = bk;
        }
      }
    }
  };
  switch (a.K) {
    case 1: epilogue(std::integral_constant<int, 1>{}); break;
    case 2: epilogue(std::integral_constant<int, 2>{}); break;
    case 4: epilogue(std::integral_constant<int, 4>{}); break;
    case 8: epilogue(std::integral_constant<int, 8>{}); break;
    case 16: epilogue(std::integral_constant<int, 16>{}); break;
    default: epilogue(std::integral_constant<int, 32>{}); break;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kPCols);
  }
}

// Column-wise hardmax of dense matrices: thread (k, j) scans column j of M_k.
__global__ void __launch_bounds__(256) dict_hardmax_kernel(const float *__restrict__ M, int64_t K, int N,
                                                           int32_t *__restrict__ idx) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= K * N) return;
  const int64_t k = e / N;
  const int j = (int)(e - k * N);
  const float *col = M + k * N * N + j;
  float bv = 0.f;
  int bi = INT_MAX;
  for (int i = 0; i < N; ++i) sel_merge(bv, bi, __ldg(col + (int64_t)i * N), i);
  idx[e] = bi;
}

// ------------------------------------------------------------ soft selection
// The original PD-SSM's transition for one step (Flash PD-SSM page, Methodology 1,
// "Original PD-SSM"): the convex combination sum_k pi_k M_k of the K dense
// dictionary matrices with pi = softmax(logits / tau), made sparse by the
// column-wise hardmax: idx_t[j] = argmax_i sum_k pi_k M_k[i][j]. For 128 tokens of
// one head the mixtures of all (i, j) are one dense product [tokens x K] x [K x N^2]
// on the tensor cores, with pi and M split into bf16 hi + lo (three products,
// about 16 bits); the epilogue takes the argmax over i of each column j.
// The dictionary is prepared once into the workspace as Mt[d][k][j][i] (hi, lo),
// so that 8 consecutive i of one (k, j) are one 16-byte chunk.

constexpr int kSM = 128;  // tokens per CTA

struct SParams {
  int64_t rows, H;  // rows = batch * seqlen
  int K, K16, N;    // dictionary entries, K rounded up to 16, state size
  int logit_bf16;
  float inv_tau;
  int head_dicts;
  const void *logits;            // [rows][H][K]
  const __nv_bfloat16 *mt;       // [dicts][2][K16][N][N] prepared parts (hi, lo)
  uint8_t *steps;                // [rows][H][N]
  uint32_t *err;
};

__global__ void __launch_bounds__(256) soft_prep_kernel(const float *__restrict__ M, int64_t dicts, int K, int K16,
                                                        int N, __nv_bfloat16 *__restrict__ mt) {
  // mt[d][part][k][j][i] = part of M[d][k][i][j] (zero for k >= K)
  const int64_t nn = (int64_t)N * N, total = dicts * K16 * nn;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t d = e / (K16 * nn);
    const int64_t r = e - d * K16 * nn;
    const int k = (int)(r / nn), ji = (int)(r - (int64_t)k * nn), j = ji / N, i = ji - j * N;
    const float v = k < K ? M[((d * K + k) * N + i) * N + j] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    mt[(d * 2 + 0) * K16 * nn + r] = hi;
    mt[(d * 2 + 1) * K16 * nn + r] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

// Stage layouts (no swizzle): A = pi part [128 tokens x K16], K-major:
//   (r % 8) * 16 + (r / 8) * (K16 * 16) + (k / 8) * 128 + (k % 8) * 2
// B = dictionary part [K16 x 256 columns (j, i)], MN-major:
//   (k % 8) * 16 + (k / 8) * 4096 + (n / 8) * 128 + (n % 8) * 2
__global__ void __launch_bounds__(kPThreads) soft_select_kernel(SParams a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int aBytes = kSM * a.K16 * 2;             // one pi part
  const int bBytes = a.K16 * 256 * 2;             // one dictionary part of one N tile
  uint8_t *sA = smem;                             // pi hi, pi lo
  uint8_t *sB = smem + 2 * aBytes;                // two stages x (hi, lo)
  uint64_t *done = reinterpret_cast<uint64_t *>(sB + 4 * bBytes);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(done + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t h = blockIdx.y, row0 = (int64_t)blockIdx.x * kSM;
  const int64_t nn = (int64_t)a.N * a.N;
  const int ntiles = (int)(nn / 256);
  const __nv_bfloat16 *mt = a.mt + (a.head_dicts ? h : 0) * 2 * a.K16 * nn;

  if (tid == 0) {
    mbar_init(done, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, kPCols);
    tmem_relinquish();
  }
  auto load_b = [&](int nt) {
    uint8_t *dst0 = sB + (nt & 1) * 2 * bBytes;
    for (int c = tid; c < 2 * a.K16 * 32; c += kPThreads) {  // (part, k, 32 chunks of 8 columns)
      const int part = c / (a.K16 * 32), rem = c - part * a.K16 * 32, k = rem >> 5, nc = rem & 31;
      cp_async16(dst0 + part * bBytes + (k & 7) * 16 + (k >> 3) * 4096 + nc * 128,
                 mt + ((int64_t)part * a.K16 + k) * nn + (int64_t)nt * 256 + nc * 8);
    }
  };
  load_b(0);
  cp_async_commit();
  // pi = softmax(logits / tau) of this thread's token, split into bf16 hi + lo
  const int r = warp * 32 + lane;
  const int64_t row = row0 + r;
  {
    float lg[64];
    float m = -INFINITY;
    for (int k = 0; k < a.K; ++k) {
      const int64_t o = (row * a.H + h) * a.K + k;
      const float v = row < a.rows ? (a.logit_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.logits)[o])
                                                   : static_cast<const float *>(a.logits)[o]) * a.inv_tau
                                   : 0.f;
      lg[k] = v;
      m = fmaxf(m, v);
    }
    float sum = 0.f;
    for (int k = 0; k < a.K; ++k) {
      lg[k] = expf(lg[k] - m);
      sum += lg[k];
    }
    const float inv = 1.f / sum;
    for (int k = 0; k < a.K16; ++k) {
      const float p = k < a.K ? lg[k] * inv : 0.f;
      const __nv_bfloat16 hi = __float2bfloat16_rn(p);
      const int off = (r & 7) * 16 + (r >> 3) * (a.K16 * 16) + (k >> 3) * 128 + (k & 7) * 2;
      *reinterpret_cast<__nv_bfloat16 *>(sA + off) = hi;
      *reinterpret_cast<__nv_bfloat16 *>(sA + aBytes + off) = __float2bfloat16_rn(p - __bfloat162float(hi));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const uint32_t idesc = idesc_bf16_f32(kSM, 256, false, true);
  const uint32_t aHi = smem_u32(sA), aLo = aHi + aBytes;
  const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
  const int groups = 256 / a.N;  // columns j per tile
  bool ok = true;
  for (int nt = 0; nt < ntiles; ++nt) {
    if (nt + 1 < ntiles) {
      load_b(nt + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    fence_proxy_async_smem();
    __syncthreads();  // tile nt's dictionary parts are in place; the previous epilogue read its accumulator
    if (tid == 0 && ok) {
      tc_fence_after();
      const uint32_t bHi = smem_u32(sB + (nt & 1) * 2 * bBytes), bLo = bHi + bBytes;
      for (int ks = 0; ks < a.K16 / 16; ++ks) {
        const uint64_t dAh = smem_desc(aHi + ks * 256, 128, a.K16 * 16), dAl = smem_desc(aLo + ks * 256, 128, a.K16 * 16);
        const uint64_t dBh = smem_desc(bHi + ks * 2 * 4096, 4096, 128), dBl = smem_desc(bLo + ks * 2 * 4096, 4096, 128);
        mma_bf16(tbase, dAh, dBh, idesc, ks != 0);
        mma_bf16(tbase, dAh, dBl, idesc, 1);
        mma_bf16(tbase, dAl, dBh, idesc, 1);
      }
      mma_commit(done);
    }
    ok = __syncthreads_and(ok && pwait(done, nt & 1, a.err));
    tc_fence_after();
    // columns jj * N + i of this tile: argmax over i for each j, by runs of CW
    // consecutive i (the winner of a run merged into the group's)
    float bv = 0.f;
    int bi = INT_MAX;
    auto runs = [&](auto cw_tag, const float *v, int c0) {
      constexpr int CW = decltype(cw_tag)::value;
#pragma unroll
      for (int h0 = 0; h0 < 32; h0 += CW) {
        float cv;
        int ci;
        run_winner<CW>(v + h0, cv, ci);
        const int col = c0 + h0, i0 = col & (a.N - 1);
        if (i0 == 0) {  // a new group: its first run's winner
          bv = cv;
          bi = ci;
        } else {
          sel_merge(bv, bi, cv, i0 + ci);
        }
        if (i0 + CW == a.N && ok && row < a.rows)
          a.steps[(row * a.H + h) * a.N + nt * groups + col / a.N] = (uint8_t)bi;
      }
    };
    for (int c0 = 0; c0 < 256; c0 += 32) {
      float v[32];
      tmem_ld32(tl + c0, v);
      tmem_wait_ld();
      if (a.N == 16) runs(std::integral_constant<int, 16>{}, v, c0);
      else runs(std::integral_constant<int, 32>{}, v, c0);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kPCols);
  }
}

}  // namespace

bool soft_select_supported(int64_t N, int64_t K) {
  return N >= 16 && N <= 128 && (N & (N - 1)) == 0 && K >= 1 && K <= 64;
}

size_t soft_select_ws_bytes(int64_t dicts, int64_t N, int64_t K) {
  const int64_t K16 = (K + 15) / 16 * 16;
  return (size_t)(dicts * 2 * K16 * N * N * 2);
}

cudaError_t launch_soft_select(int64_t rows, int64_t H, int64_t N, int64_t K, int logits_t, const void *logits,
                               const float *M, bool head_dicts, float tau, void *prep, uint8_t *steps, uint32_t *err,
                               cudaStream_t st) {
  SParams a;
  a.rows = rows;
  a.H = H;
  a.K = (int)K;
  a.K16 = (int)((K + 15) / 16 * 16);
  a.N = (int)N;
  a.logit_bf16 = logits_t == PDSSM_BF16;
  a.inv_tau = 1.f / tau;
  a.head_dicts = head_dicts;
  a.logits = logits;
  a.mt = static_cast<const __nv_bfloat16 *>(prep);
  a.steps = steps;
  a.err = err;
  const int64_t dicts = head_dicts ? H : 1;
  cudaError_t e = trace_before(st, "soft_prep");
  if (e != cudaSuccess) return e;
  soft_prep_kernel<<<1024, 256, 0, st>>>(M, dicts, a.K, a.K16, a.N, static_cast<__nv_bfloat16 *>(prep));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = trace_after(st)) != cudaSuccess) return e;
  const size_t smem = (size_t)2 * kSM * a.K16 * 2 + (size_t)4 * a.K16 * 256 * 2 + 64;
  e = cudaFuncSetAttribute(soft_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if ((e = trace_before(st, "soft_select")) != cudaSuccess) return e;
  soft_select_kernel<<<dim3((unsigned)((rows + kSM - 1) / kSM), (unsigned)H), kPThreads, smem, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

bool proj_select_supported(int64_t D, int64_t H, int64_t K) {
  const int64_t HK = H * K;
  if (D < kPK || D % kPK != 0 || K < 1 || (K & (K - 1)) != 0 || HK % 32 != 0) return false;
  return HK <= 256 || HK % 256 == 0;
}

size_t proj_select_smem_bytes(int64_t H, int64_t K) {
  const int ntile = (int)std::min<int64_t>(H * K, 256);
  return (size_t)2 * (kPM * kPK * 2 + kPK * ntile * 2) + 64;
}

cudaError_t launch_proj_select(int64_t rows, int64_t D, int64_t H, int64_t K, const void *u, const void *W,
                               int32_t *s, float *logits, uint32_t *err, cudaStream_t st) {
  PParams a;
  a.rows = rows;
  a.D = D;
  a.HK = H * K;
  a.K = (int)K;
  a.ntile = (int)std::min<int64_t>(a.HK, 256);
  a.u = static_cast<const __nv_bfloat16 *>(u);
  a.W = static_cast<const __nv_bfloat16 *>(W);
  a.s = s;
  a.logits = logits;
  a.err = err;
  const size_t smem = proj_select_smem_bytes(H, K);
  cudaError_t e = cudaFuncSetAttribute(proj_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((rows + kPM - 1) / kPM), (unsigned)(a.HK / a.ntile));
  if ((e = trace_before(st, "proj_select")) != cudaSuccess) return e;
  proj_select_kernel<<<grid, kPThreads, smem, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

cudaError_t launch_dict_hardmax(int64_t K, int N, const float *M, int32_t *idx, cudaStream_t st) {
  const int64_t n = K * N;
  if (n == 0) return cudaSuccess;
  cudaError_t e = trace_before(st, "dict_hardmax");
  if (e != cudaSuccess) return e;
  dict_hardmax_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(M, K, N, idx);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

}  // namespace pdssm
