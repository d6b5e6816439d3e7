// The plain three-phase chunked PD scan: one launch per phase.
//
// Flash PD-SSM page, Technical Summary, Methodology 3:
//   phase A  independent sequential recurrences inside chunks of length T,
//            each started from a zero state;
//   phase B  a scan over the chunks' dependencies gives the carry states;
//   phase C  the carry corrections are applied.
// Chunks are combined with the composition of (index, value) pairs of the
// one-hot-column transitions (the associative-operator framing of the Prefix
// Scannable Models abstract): (idx, val) o (idx', val') = (idx[idx'], val[idx']*val').
//
// Thread p of a block owns column p of the N x P state, so the row gather
// H'[i][p] = sum_{j in pre(i)} d[j] H[j][p] + B[i] x[p] needs no exchange
// between threads, and y_t[p] = sum_i C[i] H'[i][p] is a per-thread sum.
// The state lives in shared memory because the gather index is dynamic.
// Per-step vectors (d, B, C, x and the selected entry's preimage lists) are
// staged in shared memory by all threads. The chunk's own pair (idx, val) is
// kept by the thread that owns column j of it.
#include <algorithm>

#include "launch.h"

namespace pdssm {

namespace {

constexpr int kMaxPairsPerThread = PDSSM_MAX_N / 32;

struct KParams {
  int64_t L, H, N, P, K, T, nC;
  int64_t PB, nPB;  // columns per block and column blocks (columns are independent)
  const int32_t *s;
  const int32_t *idx;  // sanitised [K][N]
  const int32_t *off;  // [K][N+1]
  const int32_t *src;  // [K][N]
  const void *d, *B, *C, *x, *h0;
  void *y_loc, *chunk_state, *chunk_val, *y, *h_final, *prod_val;
  int32_t *chunk_idx, *prod_idx;
  uint32_t *err;
};

__device__ __forceinline__ int load_s(const KParams &a, int64_t row) {
  int st = a.s[row];
  if (st < 0 || st >= a.K) {
    flag_error(a.err, kErrSRange);
    st = 0;
  }
  return st;
}

// ------------------------------------------------------------------ phase A
template <bool CPLX, typename TD, typename TIn>
__global__ void __launch_bounds__(128) phase_a_kernel(KParams a) {
  using Nm = Num<CPLX>;
  using T = typename Nm::T;
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = (int)a.N, NT = blockDim.x, tid = threadIdx.x;
  const int64_t c = blockIdx.x / a.nPB, pb = blockIdx.x % a.nPB, h = blockIdx.y, b = blockIdx.z;
  const int p0 = (int)(pb * a.PB), P = (int)min(a.PB, a.P - p0), PG = (int)a.P;
  const int64_t t0 = c * a.T, t1 = min(t0 + a.T, a.L);

  T *Hc = reinterpret_cast<T *>(smem);
  T *Hn = Hc + N * P;
  T *dsh = Hn + N * P;
  float *Bsh = reinterpret_cast<float *>(dsh + N);
  float *Csh = Bsh + N;
  float *xsh = Csh + N;
  int *offsh = reinterpret_cast<int *>(xsh + P);
  int *srcsh = offsh + N + 1;

  for (int p = tid; p < P; p += NT)
    for (int i = 0; i < N; ++i) Hc[i * P + p] = Nm::zero();

  int pidx[kMaxPairsPerThread];
  T pval[kMaxPairsPerThread];
#pragma unroll
  for (int m = 0; m < kMaxPairsPerThread; ++m) {
    pidx[m] = tid + m * NT;
    pval[m] = Nm::one();
  }

  const TD *dg = static_cast<const TD *>(a.d);
  const TIn *Bg = static_cast<const TIn *>(a.B);
  const TIn *Cg = static_cast<const TIn *>(a.C);
  const TIn *xg = static_cast<const TIn *>(a.x);
  T *yl = static_cast<T *>(a.y_loc);

  for (int64_t t = t0; t < t1; ++t) {
    const int64_t row = (b * a.L + t) * a.H + h;
    const int st = load_s(a, row);
    __syncthreads();  // the previous step is done with the staged vectors
    for (int j = tid; j < N; j += NT) {
      dsh[j] = LoadD<CPLX, TD>::ld(dg + row * N + j);
      Bsh[j] = ldf(Bg + row * N + j);
      Csh[j] = ldf(Cg + row * N + j);
      srcsh[j] = a.src[(int64_t)st * N + j];
    }
    for (int j = tid; j <= N; j += NT) offsh[j] = a.off[(int64_t)st * (N + 1) + j];
    for (int p = tid; p < P; p += NT) xsh[p] = ldf(xg + row * PG + p0 + p);
    __syncthreads();

    // chunk pair <- (idx_s, d_t) o pair
#pragma unroll
    for (int m = 0; m < kMaxPairsPerThread; ++m) {
      if (tid + m * NT < N) {
        const int r = pidx[m];
        pval[m] = Nm::mul(dsh[r], pval[m]);
        pidx[m] = a.idx[(int64_t)st * N + r];
      }
    }

    for (int p = tid; p < P; p += NT) {
      const float xp = xsh[p];
      T yacc = Nm::zero();
      for (int i = 0; i < N; ++i) {
        T acc = Nm::from_real(Bsh[i] * xp);
        const int r1 = offsh[i + 1];
        for (int r = offsh[i]; r < r1; ++r) {
          const int j = srcsh[r];
          acc = Nm::fma(dsh[j], Hc[j * P + p], acc);
        }
        Hn[i * P + p] = acc;
        yacc = Nm::fma_r(Csh[i], acc, yacc);
      }
      yl[row * PG + p0 + p] = yacc;
    }
    T *tmp = Hc;
    Hc = Hn;
    Hn = tmp;
  }

  // chunk-end local state and chunk pair
  const int64_t slot = (b * a.H + h) * a.nC + c;
  T *cs = static_cast<T *>(a.chunk_state) + slot * N * PG;
  for (int p = tid; p < P; p += NT)
    for (int i = 0; i < N; ++i) cs[i * PG + p0 + p] = Hc[i * P + p];
  if (pb != 0) return;  // every column block computes the pair; one writes it
  T *cv = static_cast<T *>(a.chunk_val) + slot * N;
  int32_t *ci = a.chunk_idx + slot * N;
#pragma unroll
  for (int m = 0; m < kMaxPairsPerThread; ++m) {
    const int j = tid + m * NT;
    if (j < N) {
      ci[j] = pidx[m];
      cv[j] = pval[m];
    }
  }
}

// ------------------------------------------------------------------ phase B
// carry_c = apply(pair_c, carry_{c-1}) + local_c, carry_{-1} = h0 (or 0);
// apply((idx, val), H)[idx[j]] += val[j] * H[j]. The carries overwrite the
// local states in place; h_final is the last carry and (prod_idx, prod_val)
// the composition of all chunk pairs.
template <bool CPLX>
__global__ void __launch_bounds__(128) phase_b_kernel(KParams a) {
  using Nm = Num<CPLX>;
  using T = typename Nm::T;
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = (int)a.N, NT = blockDim.x, tid = threadIdx.x;
  const int64_t h = blockIdx.x / a.nPB, pb = blockIdx.x % a.nPB, b = blockIdx.y;
  const int p0 = (int)(pb * a.PB), P = (int)min(a.PB, a.P - p0), PG = (int)a.P;
  T *Hc = reinterpret_cast<T *>(smem);
  T *Hn = Hc + N * P;
  T *pv = Hn + N * P;
  int *pi = reinterpret_cast<int *>(pv + N);

  const T *h0 = static_cast<const T *>(a.h0);
  for (int p = tid; p < P; p += NT)
    for (int i = 0; i < N; ++i)
      Hc[i * P + p] = h0 ? h0[((b * a.H + h) * N + i) * PG + p0 + p] : Nm::zero();

  int tidx[kMaxPairsPerThread];
  T tval[kMaxPairsPerThread];
#pragma unroll
  for (int m = 0; m < kMaxPairsPerThread; ++m) {
    tidx[m] = tid + m * NT;
    tval[m] = Nm::one();
  }

  for (int64_t c = 0; c < a.nC; ++c) {
    const int64_t slot = (b * a.H + h) * a.nC + c;
    __syncthreads();
    for (int j = tid; j < N; j += NT) {
      pi[j] = a.chunk_idx[slot * N + j];
      pv[j] = static_cast<const T *>(a.chunk_val)[slot * N + j];
    }
    __syncthreads();
    T *cs = static_cast<T *>(a.chunk_state) + slot * N * PG + p0;
    for (int p = tid; p < P; p += NT) {
      for (int i = 0; i < N; ++i) Hn[i * P + p] = cs[i * PG + p];
      for (int j = 0; j < N; ++j) {
        T &dst = Hn[pi[j] * P + p];
        dst = Nm::fma(pv[j], Hc[j * P + p], dst);
      }
      for (int i = 0; i < N; ++i) cs[i * PG + p] = Hn[i * P + p];
    }
#pragma unroll
    for (int m = 0; m < kMaxPairsPerThread; ++m) {
      if (tid + m * NT < N) {
        const int r = tidx[m];
        tval[m] = Nm::mul(pv[r], tval[m]);
        tidx[m] = pi[r];
      }
    }
    T *tmp = Hc;
    Hc = Hn;
    Hn = tmp;
  }

  if (a.h_final) {
    T *hf = static_cast<T *>(a.h_final) + (b * a.H + h) * N * PG + p0;
    for (int p = tid; p < P; p += NT)
      for (int i = 0; i < N; ++i) hf[i * PG + p] = Hc[i * P + p];
  }
  if (pb != 0) return;
#pragma unroll
  for (int m = 0; m < kMaxPairsPerThread; ++m) {
    const int j = tid + m * NT;
    if (j < N) {
      if (a.prod_idx) a.prod_idx[(b * a.H + h) * N + j] = tidx[m];
      if (a.prod_val) static_cast<T *>(a.prod_val)[(b * a.H + h) * N + j] = tval[m];
    }
  }
}

// ------------------------------------------------------------------ phase C
// y_t = y_loc_t + carry_in^T Ctil_t, Ctil_t[j] = val_t[j] * C_t[idx_t[j]], where
// (idx_t, val_t) is the pair of the chunk's prefix up to and including t.
template <bool CPLX, typename TD, typename TIn, typename TOut>
__global__ void __launch_bounds__(128) phase_c_kernel(KParams a) {
  using Nm = Num<CPLX>;
  using T = typename Nm::T;
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = (int)a.N, NT = blockDim.x, tid = threadIdx.x;
  const int64_t c = blockIdx.x / a.nPB, pb = blockIdx.x % a.nPB, h = blockIdx.y, b = blockIdx.z;
  const int p0 = (int)(pb * a.PB), P = (int)min(a.PB, a.P - p0), PG = (int)a.P;
  const int64_t t0 = c * a.T, t1 = min(t0 + a.T, a.L);
  T *Hin = reinterpret_cast<T *>(smem);
  T *ct = Hin + N * P;
  T *dsh = ct + N;
  float *Csh = reinterpret_cast<float *>(dsh + N);

  const bool carry = (c > 0) || (a.h0 != nullptr);
  if (carry) {
    const T *src = c > 0 ? static_cast<const T *>(a.chunk_state) + ((b * a.H + h) * a.nC + c - 1) * N * PG
                         : static_cast<const T *>(a.h0) + (b * a.H + h) * N * PG;
    for (int p = tid; p < P; p += NT)
      for (int i = 0; i < N; ++i) Hin[i * P + p] = src[i * PG + p0 + p];
  }
  int pidx[kMaxPairsPerThread];
  T pval[kMaxPairsPerThread];
#pragma unroll
  for (int m = 0; m < kMaxPairsPerThread; ++m) {
    pidx[m] = tid + m * NT;
    pval[m] = Nm::one();
  }
  const TD *dg = static_cast<const TD *>(a.d);
  const TIn *Cg = static_cast<const TIn *>(a.C);
  const T *yl = static_cast<const T *>(a.y_loc);
  TOut *yo = static_cast<TOut *>(a.y);

  for (int64_t t = t0; t < t1; ++t) {
    const int64_t row = (b * a.L + t) * a.H + h;
    if (carry) {
      const int st = load_s(a, row);
      __syncthreads();
      for (int j = tid; j < N; j += NT) {
        dsh[j] = LoadD<CPLX, TD>::ld(dg + row * N + j);
        Csh[j] = ldf(Cg + row * N + j);
      }
      __syncthreads();
#pragma unroll
      for (int m = 0; m < kMaxPairsPerThread; ++m) {
        const int j = tid + m * NT;
        if (j < N) {
          const int r = pidx[m];
          pval[m] = Nm::mul(dsh[r], pval[m]);
          pidx[m] = a.idx[(int64_t)st * N + r];
          ct[j] = Nm::mul(pval[m], Nm::from_real(Csh[pidx[m]]));
        }
      }
      __syncthreads();
    }
    for (int p = tid; p < P; p += NT) {
      T acc = yl[row * PG + p0 + p];
      if (carry)
        for (int j = 0; j < N; ++j) acc = Nm::fma(ct[j], Hin[j * P + p], acc);
      st_out(yo + row * PG + p0 + p, acc);
    }
  }
}

// ------------------------------------------------------------ empty L == 0
template <bool CPLX>
__global__ void empty_outputs_kernel(KParams a, int64_t slices) {
  using Nm = Num<CPLX>;
  using T = typename Nm::T;
  const int64_t N = a.N, P = a.P;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < slices * N * P && a.h_final)
    static_cast<T *>(a.h_final)[e] = a.h0 ? static_cast<const T *>(a.h0)[e] : Nm::zero();
  if (e < slices * N) {
    if (a.prod_idx) a.prod_idx[e] = (int32_t)(e % N);
    if (a.prod_val) static_cast<T *>(a.prod_val)[e] = Nm::one();
  }
}

KParams make_params(const ScanArgs &s) {
  KParams k;
  k.L = s.L; k.H = s.H; k.N = s.N; k.P = s.P; k.K = s.K; k.T = s.T; k.nC = s.nC;
  k.PB = s.P; k.nPB = 1;
  k.s = s.s; k.idx = s.ws.idx; k.off = s.ws.csr_off; k.src = s.ws.csr_src;
  k.d = s.d; k.B = s.B; k.C = s.C; k.x = s.x; k.h0 = s.h0;
  k.y_loc = s.ws.y_loc; k.chunk_state = s.ws.chunk_state; k.chunk_val = s.ws.chunk_val;
  k.chunk_idx = s.ws.chunk_idx; k.y = s.y; k.h_final = s.h_final;
  k.prod_idx = s.prod_idx; k.prod_val = s.prod_val; k.err = s.ws.err;
  return k;
}

template <typename Kern>
cudaError_t launch_dyn(Kern kern, const char *name, dim3 grid, int threads, size_t smem,
                       cudaStream_t st, const KParams &k) {
  cudaError_t e;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  if ((e = trace_before(st, name)) != cudaSuccess) return e;
  kern<<<grid, threads, smem, st>>>(k);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

template <bool CPLX, typename TD, typename TIn, typename TOut>
cudaError_t run_chunked(const ScanArgs &s, cudaStream_t st) {
  using T = typename Num<CPLX>::T;
  KParams k = make_params(s);
  const size_t ts = sizeof(T);
  auto smem_a = [&](int64_t pb) { return 2 * s.N * pb * ts + s.N * ts + (2 * s.N + pb) * 4 + (2 * s.N + 1) * 4; };
  // columns are independent: split them over blocks until the state fits
  int64_t PB = s.P;
  while (smem_a(PB) > 200 * 1024) PB = (PB + 1) / 2;
  k.PB = PB;
  k.nPB = (s.P + PB - 1) / PB;
  const int threads = (int)std::min<int64_t>(128, std::max<int64_t>(32, (PB + 31) / 32 * 32));
  const size_t smem_b = 2 * s.N * PB * ts + s.N * ts + s.N * 4;
  const size_t smem_c = s.N * PB * ts + 2 * s.N * ts + s.N * 4;
  const dim3 grid_chunks((unsigned)(s.nC * k.nPB), (unsigned)s.H, (unsigned)s.Bt);
  cudaError_t e = launch_dyn(phase_a_kernel<CPLX, TD, TIn>, "chunked_phase_a", grid_chunks, threads, smem_a(PB), st, k);
  if (e != cudaSuccess) return e;
  e = launch_dyn(phase_b_kernel<CPLX>, "chunked_phase_b", dim3((unsigned)(s.H * k.nPB), (unsigned)s.Bt), threads, smem_b,
                 st, k);
  if (e != cudaSuccess) return e;
  return launch_dyn(phase_c_kernel<CPLX, TD, TIn, TOut>, "chunked_phase_c", grid_chunks, threads, smem_c, st, k);
}

}  // namespace

cudaError_t launch_chunked_scan(const ScanArgs &s, cudaStream_t st) {
  if (s.cplx) {
    if (s.in_t == PDSSM_BF16) return run_chunked<true, float2, __nv_bfloat16, float2>(s, st);
    return run_chunked<true, float2, float, float2>(s, st);
  }
#define PDSSM_REAL_CASE(DT, IT, OT, TD, TI, TO) \
  if (s.d_t == DT && s.in_t == IT && s.out_t == OT) return run_chunked<false, TD, TI, TO>(s, st);
  PDSSM_REAL_CASE(PDSSM_F32, PDSSM_F32, PDSSM_F32, float, float, float)
  PDSSM_REAL_CASE(PDSSM_F32, PDSSM_F32, PDSSM_BF16, float, float, __nv_bfloat16)
  PDSSM_REAL_CASE(PDSSM_F32, PDSSM_BF16, PDSSM_F32, float, __nv_bfloat16, float)
  PDSSM_REAL_CASE(PDSSM_F32, PDSSM_BF16, PDSSM_BF16, float, __nv_bfloat16, __nv_bfloat16)
  PDSSM_REAL_CASE(PDSSM_BF16, PDSSM_F32, PDSSM_F32, __nv_bfloat16, float, float)
  PDSSM_REAL_CASE(PDSSM_BF16, PDSSM_F32, PDSSM_BF16, __nv_bfloat16, float, __nv_bfloat16)
  PDSSM_REAL_CASE(PDSSM_BF16, PDSSM_BF16, PDSSM_F32, __nv_bfloat16, __nv_bfloat16, float)
  PDSSM_REAL_CASE(PDSSM_BF16, PDSSM_BF16, PDSSM_BF16, __nv_bfloat16, __nv_bfloat16, __nv_bfloat16)
#undef PDSSM_REAL_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_empty_outputs(const ScanArgs &s, cudaStream_t st) {
  const KParams k = make_params(s);
  const int64_t slices = s.Bt * s.H;
  const int64_t n = slices * std::max<int64_t>(s.N * s.P, s.N);
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  cudaError_t e = trace_before(st, "empty_outputs");
  if (e != cudaSuccess) return e;
  if (s.cplx)
    empty_outputs_kernel<true><<<blocks, threads, 0, st>>>(k, slices);
  else
    empty_outputs_kernel<false><<<blocks, threads, 0, st>>>(k, slices);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

}  // namespace pdssm
