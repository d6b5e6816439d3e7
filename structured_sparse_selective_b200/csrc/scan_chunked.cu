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
// A block owns a range of columns of one (batch, head) state and all N rows, in
// shared memory (the gather index is dynamic). In phases A and C (32 columns a
// block) a thread owns a 16-byte run of columns (4 real or 2 complex) of the rows
// g, g + RG, ... of its row group, so that each row's preimage list is read once
// for the whole run, the state moves in 16-byte loads and eight consecutive
// lanes read 128 contiguous bytes of a row (no bank conflicts). Phase B runs its
// chunks in sequence, so its blocks are narrower (8 columns, one column a thread)
// to spread few sequences over many blocks. New rows are held in registers until
// every thread has read the old state, so one state buffer suffices. Per-step
// vectors (d, B, C, x and the selected entry's preimage lists) are fetched into
// registers one step ahead and staged in shared memory; a column's output is the
// sum of the row groups' parts. (Complex phase A is held to 64 registers a thread
// for occupancy, measured faster despite a few spilled bytes; real phase A has no
// occupancy bound, minBlocks 0, which measured faster for it.)
#include <algorithm>

#include "launch.h"

namespace pdssm {

namespace {

constexpr int kPB = 32;       // columns per block (one warp per row group)

struct KParams {
  int64_t L, H, N, P, K, T, nC;
  int64_t Kh;   // dictionary entries per head with per-head dictionaries (else 0)
  int64_t nPB;   // column blocks of phases A and C (columns are independent)
  int64_t nPBB;  // column blocks of phase B (narrower: its blocks run the chunks in sequence)
  const int32_t *s;
  const int32_t *idx;  // sanitised [K][N]
  const int32_t *off;  // [K][N+1]
  const int32_t *src;  // [K][N]
  const void *d, *B, *C, *x, *h0;
  void *y_loc, *chunk_state, *chunk_val, *y, *h_final, *prod_val;
  int32_t *chunk_idx, *prod_idx;
  uint32_t *err;
};

// Dictionary entry of row `row` (head h): the selection, validated, plus h * Kh.
__device__ __forceinline__ int load_s(const KParams &a, int64_t row, int64_t h) {
  int st = a.s[row];
  if (st < 0 || st >= a.K) {
    flag_error(a.err, kErrSRange);
    st = 0;
  }
  return st + (int)(h * a.Kh);
}

// ------------------------------------------------------------------ phase A
// Within chunk c, from a zero state: H_t[i] = B_t[i] x_t + sum_{j in pre(i)} d_t[j] H_{t-1}[j],
// y_loc_t = H_t^T C_t; the chunk's pair is the composition of its steps' pairs.
template <typename T>
struct StepVec {  // one thread's share of a step's vectors (entry j = tid)
  T d;
  float B, C, x;
  int src, off, st;
};

// Columns a phase-A thread owns: one 16-byte run (4 real or 2 complex values), so
// that the preimage lists of a row are read once for several columns and eight
// consecutive lanes read 128 contiguous bytes of a state row (no bank conflicts).
template <typename T>
struct ColRun {
  static constexpr int VW = 16 / (int)sizeof(T);  // columns per thread
  static constexpr int TPR = kPB / VW;            // threads per row group
  static constexpr int MR = 16 / VW;              // rows per thread at most (RG * MR >= N)
};

__device__ __forceinline__ float shfl_xor(float v, int o) { return __shfl_xor_sync(0xffffffffu, v, o); }
__device__ __forceinline__ float2 shfl_xor(float2 v, int o) {
  return make_float2(__shfl_xor_sync(0xffffffffu, v.x, o), __shfl_xor_sync(0xffffffffu, v.y, o));
}

__device__ __forceinline__ void ld_run(const float *p, float (&v)[4]) {
  const float4 w = *reinterpret_cast<const float4 *>(p);
  v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
}
__device__ __forceinline__ void ld_run(const float2 *p, float2 (&v)[2]) {
  const float4 w = *reinterpret_cast<const float4 *>(p);
  v[0] = make_float2(w.x, w.y); v[1] = make_float2(w.z, w.w);
}
__device__ __forceinline__ void st_run(float *p, const float (&v)[4]) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void st_run(float2 *p, const float2 (&v)[2]) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
}

// Threads: RG row groups of TPR threads; thread (g, cl) updates rows g, g + RG, ...
// of columns [cl * VW, cl * VW + VW) of the block's kPB columns.
// kLocalOut: write y_loc (false when only the carries are wanted).
template <int RG, bool CPLX, typename TD, typename TIn, bool kLocalOut>
__global__ void __launch_bounds__(RG * ColRun<typename Num<CPLX>::T>::TPR,
                                  CPLX ? 1024 / (RG * ColRun<typename Num<CPLX>::T>::TPR) : 0)
    phase_a_kernel(KParams a) {
  using Nm = Num<CPLX>;
  using T = typename Nm::T;
  constexpr int VW = ColRun<T>::VW, TPR = ColRun<T>::TPR, MR = ColRun<T>::MR, NT = RG * TPR, NW = NT / 32;
  static_assert(NT % 32 == 0 && 32 % TPR == 0, "row groups tile whole warps");
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = (int)a.N, tid = threadIdx.x, cl = tid % TPR, g = tid / TPR, pc = cl * VW;
  const int64_t c = blockIdx.x / a.nPB, pb = blockIdx.x % a.nPB, h = blockIdx.y, b = blockIdx.z;
  const int p0 = (int)(pb * kPB), P = (int)min((int64_t)kPB, a.P - p0), PG = (int)a.P;
  const int64_t t0 = c * a.T, t1 = min(t0 + a.T, a.L);

  T *Hs = reinterpret_cast<T *>(smem);  // [N][kPB]
  T *ysh = Hs + N * kPB;                // [NW][kPB] per-warp parts of the output
  T *dsh = ysh + NW * kPB;              // [N]
  float *Bsh = reinterpret_cast<float *>(dsh + N);
  float *Csh = Bsh + N;
  float *xsh = Csh + N;                 // [kPB]
  int *offsh = reinterpret_cast<int *>(xsh + kPB);
  int *srcsh = offsh + N + 1;

  const TD *dg = static_cast<const TD *>(a.d);
  const TIn *Bg = static_cast<const TIn *>(a.B);
  const TIn *Cg = static_cast<const TIn *>(a.C);
  const TIn *xg = static_cast<const TIn *>(a.x);
  T *yl = static_cast<T *>(a.y_loc);

  for (int e = tid; e < N * kPB; e += NT) Hs[e] = Nm::zero();
  int pidx = tid;  // chunk pair entry tid (tid < N)
  T pval = Nm::one();

  // NT > N: thread tid fetches entry tid of each vector (and off[N], x[tid])
  auto fetch = [&](int64_t t) {
    StepVec<T> v;
    const int64_t row = (b * a.L + t) * a.H + h;
    v.st = load_s(a, row, h);
    if (tid < N) {
      v.d = LoadD<CPLX, TD>::ld(dg + row * N + tid);
      v.B = ldf(Bg + row * N + tid);
      v.C = ldf(Cg + row * N + tid);
      v.src = a.src[(int64_t)v.st * N + tid];
    }
    if (tid <= N) v.off = a.off[(int64_t)v.st * (N + 1) + tid];
    if (tid < kPB) v.x = tid < P ? ldf(xg + row * PG + p0 + tid) : 0.f;
    return v;
  };
  auto commit = [&](const StepVec<T> &v) {
    if (tid < N) {
      dsh[tid] = v.d;
      Bsh[tid] = v.B;
      Csh[tid] = v.C;
      srcsh[tid] = v.src;
    }
    if (tid <= N) offsh[tid] = v.off;
    if (tid < kPB) xsh[tid] = v.x;
  };
  // output of step t from the warps' parts (fixed order)
  auto finish_y = [&](int64_t t) {
    if (kLocalOut && tid < P) {
      T acc = ysh[tid];
#pragma unroll
      for (int w = 1; w < NW; ++w) acc = Nm::add(acc, ysh[w * kPB + tid]);
      yl[((b * a.L + t) * a.H + h) * PG + p0 + tid] = acc;
    }
  };

  StepVec<T> cur = fetch(t0);  // t0 < t1: every chunk holds a token
  commit(cur);
  int st = cur.st;
  for (int64_t t = t0; t < t1; ++t) {
    StepVec<T> nxt;
    if (t + 1 < t1) nxt = fetch(t + 1);  // in flight during this step
    __syncthreads();  // step t's vectors, the state and the parts of step t - 1 are visible
    if (t > t0) finish_y(t - 1);
    if (tid < N) {  // chunk pair <- (idx_s, d_t) o pair
      pval = Nm::mul(dsh[pidx], pval);
      pidx = a.idx[(int64_t)st * N + pidx];
    }
    T nv[MR][VW];
    T yp[VW];
    float xv[VW];
#pragma unroll
    for (int e = 0; e < VW; ++e) {
      yp[e] = Nm::zero();
      xv[e] = xsh[pc + e];
    }
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      const int i = g + RG * m;
      if (i < N) {
        const float bi = Bsh[i];
#pragma unroll
        for (int e = 0; e < VW; ++e) nv[m][e] = Nm::from_real(bi * xv[e]);
        // sources in increasing order (fixed summation order); the first two outside
        // the loop so that their loads overlap (most rows have at most two)
        auto add_src = [&](int j) {
          const T dj = dsh[j];
          T hv[VW];
          ld_run(Hs + j * kPB + pc, hv);
#pragma unroll
          for (int e = 0; e < VW; ++e) nv[m][e] = Nm::fma(dj, hv[e], nv[m][e]);
        };
        const int r0 = offsh[i], r1 = offsh[i + 1];
        if (r0 < r1) {
          add_src(srcsh[r0]);
          if (r0 + 1 < r1) {
            add_src(srcsh[r0 + 1]);
            for (int r = r0 + 2; r < r1; ++r) add_src(srcsh[r]);
          }
        }
        const float ci = Csh[i];
#pragma unroll
        for (int e = 0; e < VW; ++e) yp[e] = Nm::fma_r(ci, nv[m][e], yp[e]);
      }
    }
    // the row groups of a warp share columns: sum their parts, one per warp to memory
#pragma unroll
    for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < VW; ++e) yp[e] = Nm::add(yp[e], shfl_xor(yp[e], o));
    __syncthreads();  // every read of the old state and of the staged vectors is done
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      const int i = g + RG * m;
      if (i < N) st_run(Hs + i * kPB + pc, nv[m]);
    }
    if ((tid & 31) < TPR) st_run(ysh + (tid >> 5) * kPB + pc, yp);
    if (t + 1 < t1) {
      commit(nxt);
      st = nxt.st;
    }
  }
  __syncthreads();
  finish_y(t1 - 1);

  // chunk-end local state and chunk pair
  const int64_t slot = (b * a.H + h) * a.nC + c;
  T *cs = static_cast<T *>(a.chunk_state) + slot * N * PG;
  for (int e = tid; e < N * kPB; e += NT) {
    const int i = e / kPB, p = e % kPB;
    if (p < P) cs[i * PG + p0 + p] = Hs[e];
  }
  if (pb != 0 || tid >= N) return;  // every column block computes the pair; one writes it
  a.chunk_idx[slot * N + tid] = pidx;
  static_cast<T *>(a.chunk_val)[slot * N + tid] = pval;
}

// ------------------------------------------------------------------ phase B
// carry_c = apply(pair_c, carry_{c-1}) + local_c, carry_{-1} = h0 (or 0), with
// apply((idx, val), H)[i] = sum_{j: idx[j] = i} val[j] H[j], sources in increasing
// j. The carries overwrite the local states in place; h_final is the last carry
// and (prod_idx, prod_val) the composition of all chunk pairs.
// A block owns PB columns (RG row groups of them, at most MRB rows a thread): 8
// for N <= 32, so that a workload with few sequences still spreads its
// sequential chunk loops over many blocks, else 32 (every block sorts the chunk
// pairs' preimages, O(N) a thread).
template <int RG, int PB, int MRB, bool CPLX>
__global__ void __launch_bounds__(RG * PB) phase_b_kernel(KParams a) {
  using Nm = Num<CPLX>;
  using T = typename Nm::T;
  constexpr int NT = RG * PB;
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = (int)a.N, tid = threadIdx.x, pl = tid % PB, g = tid / PB;
  const int64_t h = blockIdx.x / a.nPBB, pb = blockIdx.x % a.nPBB, b = blockIdx.y;
  const int p0 = (int)(pb * PB), P = (int)min((int64_t)PB, a.P - p0), PG = (int)a.P;
  const bool col = pl < P;
  T *Hs = reinterpret_cast<T *>(smem);  // [N][PB]
  T *pv = Hs + N * PB;                 // [N]
  int *pi = reinterpret_cast<int *>(pv + N);
  int *off = pi + N;                    // [N+1] preimage lists of the chunk pair's index map
  int *src = off + N + 1;               // [N]

  const T *h0 = static_cast<const T *>(a.h0);
  for (int i = g; i < N; i += RG)
    Hs[i * PB + pl] = (h0 && col) ? h0[((b * a.H + h) * N + i) * PG + p0 + pl] : Nm::zero();
  int tidx = tid;  // whole-sequence product entry tid (tid < N)
  T tval = Nm::one();
  const int64_t slot0 = (b * a.H + h) * a.nC;
  int pi_n = 0;  // the next chunk's pair entry tid, fetched one chunk ahead
  T pv_n = Nm::zero();
  if (tid < N && a.nC > 0) {
    pi_n = a.chunk_idx[slot0 * N + tid];
    pv_n = static_cast<const T *>(a.chunk_val)[slot0 * N + tid];
  }

  for (int64_t c = 0; c < a.nC; ++c) {
    T *cs = static_cast<T *>(a.chunk_state) + (slot0 + c) * N * PG + p0;
    T nv[MRB];  // the local state's rows, loaded while the lists are built
#pragma unroll
    for (int m = 0; m < MRB; ++m) {
      const int i = g + RG * m;
      if (i < N) nv[m] = col ? cs[i * PG + pl] : Nm::zero();
    }
    __syncthreads();  // the previous chunk's lists are no longer read
    if (tid < N) {
      pi[tid] = pi_n;
      pv[tid] = pv_n;
      if (c + 1 < a.nC) {
        pi_n = a.chunk_idx[(slot0 + c + 1) * N + tid];
        pv_n = static_cast<const T *>(a.chunk_val)[(slot0 + c + 1) * N + tid];
      }
    }
    __syncthreads();
    // stable counting sort of the sources by target: off[i] = #{j : pi[j] < i},
    // source tid goes to off[pi[tid]] + #{j < tid : pi[j] = pi[tid]}
    int mine = 0, rank = 0;
    if (tid < N) {
      mine = pi[tid];
      int below = 0;
      for (int j = 0; j < N; ++j) {
        const int pj = pi[j];
        below += pj < tid;
        rank += (j < tid) & (pj == mine);
      }
      off[tid] = below;
      if (tid == 0) off[N] = N;
      tval = Nm::mul(pv[tidx], tval);  // product <- pair_c o product
      tidx = pi[tidx];
    }
    __syncthreads();
    if (tid < N) src[off[mine] + rank] = tid;
    __syncthreads();
#pragma unroll
    for (int m = 0; m < MRB; ++m) {
      const int i = g + RG * m;
      if (i < N) {
        T acc = nv[m];
        const int r0 = off[i], r1 = off[i + 1];
        if (r0 < r1) {
          const int ja = src[r0];
          acc = Nm::fma(pv[ja], Hs[ja * PB + pl], acc);
          if (r0 + 1 < r1) {
            const int jb = src[r0 + 1];
            acc = Nm::fma(pv[jb], Hs[jb * PB + pl], acc);
            for (int r = r0 + 2; r < r1; ++r) {
              const int j = src[r];
              acc = Nm::fma(pv[j], Hs[j * PB + pl], acc);
            }
          }
        }
        nv[m] = acc;
      }
    }
    __syncthreads();  // every read of the previous carry is done
#pragma unroll
    for (int m = 0; m < MRB; ++m) {
      const int i = g + RG * m;
      if (i < N) {
        Hs[i * PB + pl] = nv[m];
        if (col) cs[i * PG + pl] = nv[m];
      }
    }
  }
  __syncthreads();

  if (a.h_final && col) {
    T *hf = static_cast<T *>(a.h_final) + (b * a.H + h) * N * PG + p0;
    for (int i = g; i < N; i += RG) hf[i * PG + pl] = Hs[i * PB + pl];
  }
  (void)NT;
  if (pb != 0 || tid >= N) return;
  if (a.prod_idx) a.prod_idx[(b * a.H + h) * N + tid] = tidx;
  if (a.prod_val) static_cast<T *>(a.prod_val)[(b * a.H + h) * N + tid] = tval;
}

// ------------------------------------------------------------------ phase C
// y_t = y_loc_t + carry_in^T Ctil_t, Ctil_t[j] = val_t[j] * C_t[idx_t[j]], where
// (idx_t, val_t) is the pair of the chunk's prefix up to and including t.
// Steps go in groups of kTG: the prefix pairs give Ctil for the group's steps
// (one thread per entry j), then each thread accumulates the group's outputs for
// its column run over its rows, so a carry row is read once per group.
constexpr int kTG = 8;

template <int RG, bool CPLX, typename TD, typename TIn, typename TOut>
__global__ void __launch_bounds__(RG * ColRun<typename Num<CPLX>::T>::TPR) phase_c_kernel(KParams a) {
  using Nm = Num<CPLX>;
  using T = typename Nm::T;
  constexpr int VW = ColRun<T>::VW, TPR = ColRun<T>::TPR, MR = ColRun<T>::MR, NT = RG * TPR, NW = NT / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = (int)a.N, tid = threadIdx.x, cl = tid % TPR, g = tid / TPR, pc = cl * VW;
  const int64_t c = blockIdx.x / a.nPB, pb = blockIdx.x % a.nPB, h = blockIdx.y, b = blockIdx.z;
  const int p0 = (int)(pb * kPB), P = (int)min((int64_t)kPB, a.P - p0), PG = (int)a.P;
  const int64_t t0 = c * a.T, t1 = min(t0 + a.T, a.L);
  T *Hin = reinterpret_cast<T *>(smem);  // [N][kPB] carry into the chunk
  T *ysh = Hin + N * kPB;                // [NW][kTG][kPB] per-warp parts of the outputs
  T *ct = ysh + NW * kTG * kPB;          // [kTG][N] Ctil of the group's steps
  T *dsh = ct + kTG * N;                 // [kTG][N]
  float *Csh = reinterpret_cast<float *>(dsh + kTG * N);  // [kTG][N]
  int *ssh = reinterpret_cast<int *>(Csh + kTG * N);      // [kTG] dictionary entries

  const TD *dg = static_cast<const TD *>(a.d);
  const TIn *Cg = static_cast<const TIn *>(a.C);
  const T *yl = static_cast<const T *>(a.y_loc);
  TOut *yo = static_cast<TOut *>(a.y);
  auto yrow = [&](int64_t t) { return ((b * a.L + t) * a.H + h) * PG + p0; };

  const bool carry = (c > 0) || (a.h0 != nullptr);
  if (!carry) {
    for (int64_t e = tid; e < (t1 - t0) * P; e += NT) {
      const int64_t t = t0 + e / P;
      const int p = (int)(e % P);
      st_out(yo + yrow(t) + p, yl[yrow(t) + p]);
    }
    return;
  }
  const T *hin = c > 0 ? static_cast<const T *>(a.chunk_state) + ((b * a.H + h) * a.nC + c - 1) * N * PG
                       : static_cast<const T *>(a.h0) + (b * a.H + h) * N * PG;
  for (int e = tid; e < N * kPB; e += NT) {
    const int i = e / kPB, p = e % kPB;
    Hin[e] = p < P ? hin[i * PG + p0 + p] : Nm::zero();
  }
  int pidx = tid;  // prefix pair entry tid (tid < N)
  T pval = Nm::one();

  for (int64_t tg = t0; tg < t1; tg += kTG) {
    const int ng = (int)min((int64_t)kTG, t1 - tg);
    // the group's vectors: the prefix pair needs d_t[pidx] and C_t[idx_t[pidx]],
    // entries another thread may own
    for (int e = tid; e < ng * N; e += NT) {
      const int tau = e / N, j = e % N;
      const int64_t row = (b * a.L + tg + tau) * a.H + h;
      dsh[e] = LoadD<CPLX, TD>::ld(dg + row * N + j);
      Csh[e] = ldf(Cg + row * N + j);
    }
    if (tid < ng) ssh[tid] = load_s(a, (b * a.L + tg + tid) * a.H + h, h);
    __syncthreads();  // the group's vectors; the previous group's parts were read
    if (tid < N) {
      for (int tau = 0; tau < ng; ++tau) {
        pval = Nm::mul(dsh[tau * N + pidx], pval);
        pidx = a.idx[(int64_t)ssh[tau] * N + pidx];
        ct[tau * N + tid] = Nm::mul(pval, Nm::from_real(Csh[tau * N + pidx]));
      }
    }
    __syncthreads();  // Ctil of the group
    T acc[kTG][VW];
#pragma unroll
    for (int tau = 0; tau < kTG; ++tau)
#pragma unroll
      for (int e = 0; e < VW; ++e) acc[tau][e] = Nm::zero();
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      const int i = g + RG * m;
      if (i < N) {
        T hv[VW];
        ld_run(Hin + i * kPB + pc, hv);
#pragma unroll
        for (int tau = 0; tau < kTG; ++tau) {
          const T cv = ct[tau * N + i];  // stale entries past ng are never written out
#pragma unroll
          for (int e = 0; e < VW; ++e) acc[tau][e] = Nm::fma(cv, hv[e], acc[tau][e]);
        }
      }
    }
#pragma unroll
    for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
      for (int tau = 0; tau < kTG; ++tau)
#pragma unroll
        for (int e = 0; e < VW; ++e) acc[tau][e] = Nm::add(acc[tau][e], shfl_xor(acc[tau][e], o));
    if ((tid & 31) < TPR)
#pragma unroll
      for (int tau = 0; tau < kTG; ++tau) st_run(ysh + ((tid >> 5) * kTG + tau) * kPB + pc, acc[tau]);
    __syncthreads();  // the warps' parts
    for (int e = tid; e < ng * kPB; e += NT) {
      const int tau = e / kPB, p = e % kPB;
      if (p < P) {
        const int64_t o = yrow(tg + tau) + p;
        T y = yl[o];
#pragma unroll
        for (int w = 0; w < NW; ++w) y = Nm::add(y, ysh[(w * kTG + tau) * kPB + p]);
        st_out(yo + o, y);
      }
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
  k.Kh = s.head_dicts ? s.K : 0;
  k.nPB = (s.P + kPB - 1) / kPB;
  const int64_t pbb = s.N <= 32 ? 8 : kPB;  // phase B's columns a block (as run_chunked_n)
  k.nPBB = (s.P + pbb - 1) / pbb;
  k.s = s.s; k.idx = s.ws.idx; k.off = s.ws.csr_off; k.src = s.ws.csr_src;
  k.d = s.d; k.B = s.B; k.C = s.C; k.x = s.x; k.h0 = s.h0;
  k.y_loc = s.ws.y_loc; k.chunk_state = s.ws.chunk_state; k.chunk_val = s.ws.chunk_val;
  k.chunk_idx = s.ws.chunk_idx; k.y = s.y; k.h_final = s.h_final;
  k.prod_idx = s.prod_idx; k.prod_val = s.prod_val; k.err = s.ws.err;
  return k;
}

template <typename Kern>
cudaError_t launch_dyn(Kern kern, const char *name, dim3 grid, int threads, size_t smem, cudaStream_t st,
                       const KParams &k) {
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

// NMAX bounds N (16, 32, 64 or 128); it sizes every phase's row groups. Without an
// output (s.y null) only phases A and B run: the carries at the chunk ends.
template <int NMAX, bool CPLX, typename TD, typename TIn, typename TOut>
cudaError_t run_chunked_n(const ScanArgs &s, cudaStream_t st) {
  using T = typename Num<CPLX>::T;
  const KParams k = make_params(s);
  const size_t ts = sizeof(T), N = (size_t)s.N;
  // phases A and C: RGA * MR >= N rows, 2 NMAX threads; phase B: RGB * MRB >= N rows
  constexpr int RGA = NMAX / ColRun<T>::MR, NTA = RGA * ColRun<T>::TPR;
  constexpr int PBB = NMAX <= 32 ? 8 : kPB, MRB = NMAX <= 32 ? 4 : 16, RGB = NMAX / MRB, NTB = RGB * PBB;
  static_assert(NTA > NMAX && NTB >= NMAX, "a thread per vector entry");
  const size_t smem_a = N * kPB * ts + (NTA / 32) * kPB * ts + N * ts + 2 * N * 4 + kPB * 4 + (2 * N + 1) * 4;
  const size_t smem_b = N * PBB * ts + N * ts + N * 4 + (2 * N + 1) * 4;
  const size_t smem_c = N * kPB * ts + (NTA / 32) * kTG * kPB * ts + 2 * kTG * N * ts + kTG * N * 4 + kTG * 4;
  const dim3 grid_chunks((unsigned)(s.nC * k.nPB), (unsigned)s.H, (unsigned)s.Bt);
  cudaError_t e = s.y ? launch_dyn(phase_a_kernel<RGA, CPLX, TD, TIn, true>, "chunked_phase_a", grid_chunks, NTA,
                                   smem_a, st, k)
                      : launch_dyn(phase_a_kernel<RGA, CPLX, TD, TIn, false>, "chunked_phase_a", grid_chunks, NTA,
                                   smem_a, st, k);
  if (e != cudaSuccess) return e;
  e = launch_dyn(phase_b_kernel<RGB, PBB, MRB, CPLX>, "chunked_phase_b", dim3((unsigned)(s.H * k.nPBB), (unsigned)s.Bt), NTB,
                 smem_b, st, k);
  if (e != cudaSuccess || !s.y) return e;
  return launch_dyn(phase_c_kernel<RGA, CPLX, TD, TIn, TOut>, "chunked_phase_c", grid_chunks, NTA, smem_c, st, k);
}

template <bool CPLX, typename TD, typename TIn, typename TOut>
cudaError_t run_chunked(const ScanArgs &s, cudaStream_t st) {
  if (s.N <= 16) return run_chunked_n<16, CPLX, TD, TIn, TOut>(s, st);
  if (s.N <= 32) return run_chunked_n<32, CPLX, TD, TIn, TOut>(s, st);
  if (s.N <= 64) return run_chunked_n<64, CPLX, TD, TIn, TOut>(s, st);
  return run_chunked_n<128, CPLX, TD, TIn, TOut>(s, st);
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

cudaError_t launch_chunked_carries(const ScanArgs &s, cudaStream_t st) {
  // phases A and B only: the output type is not used
  ScanArgs c = s;
  c.y = nullptr;
  c.out_t = c.cplx ? PDSSM_C64 : PDSSM_F32;
  return launch_chunked_scan(c, st);
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
