// Backward pass of the PD scan (real or complex state): gradients of the loss
//   Re[ sum_t <dy_t, y_t> + <dh_final, H_{L-1}> ],  <a, b> = sum conj(a) b,
// with respect to d, B, C, x, h0 and, through the straight-through estimator
// with a tempered softmax, the selection logits. For a complex quantity
// z = u + i v the gradient is dLoss/du + i dLoss/dv; for a real state every
// conjugate and real part below is the identity.
//
// Flash PD-SSM page, Technical Summary, Methodology 2 ("Gradient Propagation"):
// the forward pass uses the hard argmax; the backward pass approximates the
// selection by a tempered softmax. The step's transition is read as the mixture
// A_t = sum_k pi_k P_k diag(d_t), one-hot at s_t in the forward pass; the gradient
// in the weights, dpi_t[k] = Re sum_j conj((Lam_t H_{t-1}^H)[idx_k[j]][j]) d_t[j],
// goes through the Jacobian of softmax(logits_t / tau).
//
// The adjoint Lam_t = dLoss/dH_t runs backwards:
//   Lam_t = Lam'_t + C_t dy_t^T,  Lam'_{t-1} = A_t^H Lam_t  ((A^H Lam)[j] = conj(d[j]) Lam[idx[j]]),
// and the step's gradients are
//   dC_t = Re(H_t conj(dy_t)), dB_t = Re(Lam_t) x_t, dx_t = Re(Lam_t)^T B_t,
//   dd_t[j] = sum_p Lam_t[idx_{s_t}[j]][p] conj(H_{t-1}[j][p]).
//
// One block per (batch, head) sequence, or per range of its columns. The
// checkpoints, the state every kTb steps (O(L N P / kTb) memory), are the carries
// of the chunked forward scan at chunk length kTb, computed in parallel over the
// chunks before this kernel; the reverse sweep recomputes each kTb-step stretch
// from its checkpoint into a per-block scratch and walks it backwards. Three N x P
// buffers in shared memory hold the adjoint, H_t and H_{t-1}; threads move their
// rows in 16-byte runs (4 real or 2 complex values), so a row's preimage list or
// dictionary row is read once per run.
#include "launch.h"

namespace pdssm {

namespace {

// Threads per block: 512 when a block owns all P columns of its sequence, 256 when
// the columns are split over several blocks (either way at most 64 registers a
// thread: 2 or 4 blocks an SM).
constexpr int kBTWhole = 512, kBTSplit = 256;
constexpr int kTb = 16;   // steps between checkpoints
static_assert(PDSSM_MAX_N <= 256, "the dictionary is held in shared memory as uint8 row indices");
static_assert(PDSSM_MAX_K <= 64, "warp 0 holds two selection logits a lane");
static_assert(PDSSM_MAX_N + 128 <= kBTSplit && PDSSM_MAX_P + 32 <= kBTSplit,
              "a thread per vector entry; dC uses threads 128.., dx threads 32..");

struct BParams {
  int64_t L, H, N, P, K, nCk;
  int64_t Pg;    // columns of the state; a block owns P of them (P * nPB >= Pg)
  int64_t nPB;   // column blocks per sequence
  int64_t rows;  // batch * seqlen * heads
  float tau;
  int logits_bf16, dy_bf16;
  bool head_dicts;  // idx/off/src hold heads * K entries, head h's from h * K
  const int32_t *s;
  const int32_t *idx;  // sanitised [K][N]
  const int32_t *off;  // [K][N+1]
  const int32_t *src;  // [K][N]
  const void *logits, *d, *B, *C, *x, *dy;
  const void *h0, *dh_final;  // state type
  const void *ckpt;  // [Bt*H][nCk][N][Pg] state type: the state after each 16-step chunk
  void *scratch;  // [Bt*H*nPB][kTb][N][P], state type
  float *dlogits, *dB, *dC, *dx;
  void *dd, *dh0;  // state type
  // with nPB > 1, each column block's share of the sums over columns, [nPB][rows][*]
  // (the reduction kernel adds them and forms the logits' gradient)
  void *pdd;
  float *pdB, *pdC, *pdpi;
  uint32_t *err;
};

__device__ __forceinline__ float ld_flag(const void *p, int64_t i, int bf16) {
  return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]) : static_cast<const float *>(p)[i];
}

// Conjugates and real parts of the state type (identities for a real state).
__device__ __forceinline__ float conj_of(float v) { return v; }
__device__ __forceinline__ float2 conj_of(float2 v) { return make_float2(v.x, -v.y); }
__device__ __forceinline__ float re_of(float v) { return v; }
__device__ __forceinline__ float re_of(float2 v) { return v.x; }
// c + a conj(b)
__device__ __forceinline__ float fma_conj(float a, float b, float c) { return fmaf(a, b, c); }
__device__ __forceinline__ float2 fma_conj(float2 a, float2 b, float2 c) {
  return make_float2(fmaf(a.x, b.x, fmaf(a.y, b.y, c.x)), fmaf(a.y, b.x, fmaf(-a.x, b.y, c.y)));
}
// c + Re(a conj(b))
__device__ __forceinline__ float fma_re_conj(float a, float b, float c) { return fmaf(a, b, c); }
__device__ __forceinline__ float fma_re_conj(float2 a, float2 b, float c) { return fmaf(a.x, b.x, fmaf(a.y, b.y, c)); }

// dy as stored: f32 / bf16 for a real state, complex64 for a complex one.
__device__ __forceinline__ void ld_dy(const void *p, int64_t i, int bf16, float *v) { *v = ld_flag(p, i, bf16); }
__device__ __forceinline__ void ld_dy(const void *p, int64_t i, int, float2 *v) {
  *v = static_cast<const float2 *>(p)[i];
}

// 16 bytes of a state row: 4 real or 2 complex values.
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

template <bool CPLX, typename TD, typename TIn, int kBT>
__global__ void __launch_bounds__(kBT, 1024 / kBT) scan_bwd_kernel(BParams a) {
  using NT = Num<CPLX>;
  using T = typename NT::T;
  constexpr int VW = 16 / (int)sizeof(T);  // values per 16-byte run
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = (int)a.N, K = (int)a.K;
  const int P = (int)min(a.P, a.Pg - (int64_t)(blockIdx.x % a.nPB) * a.P);  // this block's columns
  // Rows hold PV = P rounded up to whole runs (the extra columns stay zero: their
  // x and dy are zero) plus one run of padding, which keeps rows 16-byte aligned
  // and puts consecutive rows 16 bytes apart in the banks.
  const int NR = (P + VW - 1) / VW, PV = NR * VW, PS = PV + VW;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = blockIdx.x / a.nPB, pb = blockIdx.x % a.nPB, b = bh / a.H, h = bh % a.H;
  const int64_t Pg = a.Pg, c0 = pb * a.P;  // this block's first column
  const bool split = a.nPB > 1;

  T *buf0 = reinterpret_cast<T *>(smem);  // three [N][PS] buffers
  T *buf1 = buf0 + N * PS;
  T *buf2 = buf1 + N * PS;
  T *dsh = buf2 + N * PS;  // [N]
  T *dysh = dsh + N;       // [PV]
  float *Bsh = reinterpret_cast<float *>(dysh + PV);  // [N]
  float *Csh = Bsh + N;                               // [N]
  float *xsh = Csh + N;                               // [PV]
  float *dpi = xsh + PV;                              // [K]
  int *offsh = reinterpret_cast<int *>(dpi + K);  // [N+1] preimage lists of the step's entry
  int *srcsh = offsh + N + 1;                     // [N]
  uint8_t *idxsh = reinterpret_cast<uint8_t *>(srcsh + N);  // [K][N] dictionary

  const int64_t kh = a.head_dicts ? h * K : 0;  // this head's first dictionary entry
  for (int e = tid; e < K * N; e += kBT) idxsh[e] = (uint8_t)a.idx[kh * N + e];
  for (int p = P + tid; p < PV; p += kBT) {  // the padding columns' x and dy stay zero
    xsh[p] = 0.f;
    dysh[p] = NT::zero();
  }

  const TD *dg = static_cast<const TD *>(a.d);
  const TIn *Bg = static_cast<const TIn *>(a.B);
  const TIn *Cg = static_cast<const TIn *>(a.C);
  const TIn *xg = static_cast<const TIn *>(a.x);
  const T *h0g = static_cast<const T *>(a.h0);
  const T *dhg = static_cast<const T *>(a.dh_final);
  T *ddg = static_cast<T *>(a.dd);
  const T *ck = static_cast<const T *>(a.ckpt) + bh * a.nCk * N * Pg + c0;  // this block's columns
  T *scr = static_cast<T *>(a.scratch) + (int64_t)blockIdx.x * kTb * N * a.P;

  // loop over the runs of a dense [N][PV] array: thread tid starts at run tid
  const int dr = kBT / NR, dq = kBT - dr * NR;
  const int r_start = tid / NR, q_start = tid - r_start * NR;
#define FOR_RUNS(i, q)                                                         \
  for (int i = r_start, q = q_start; i < N; i += dr, q += dq, (q >= NR ? (q -= NR, ++i) : 0))

  auto row_of = [&](int64_t t) { return (b * a.L + t) * a.H + h; };
  auto load_s = [&](int64_t row) {
    int st = a.s[row];
    if (st < 0 || st >= K) {
      flag_error(a.err, kErrSRange);
      st = 0;
    }
    return st;
  };
  // A step's vectors, fetched into registers a step ahead: thread tid holds entry
  // tid of d, B, C (and of the entry's preimage lists), of x and dy (N, P <= 128 <
  // kBT, so one entry each) and s.
  struct Vec {
    T d, dy;
    float B, C, x;
    int src, off, st;
  };
  auto fetch = [&](int64_t t, bool rev) {
    Vec v;
    const int64_t row = row_of(t);
    v.st = load_s(row);
    if (tid < N) {
      v.d = LoadD<CPLX, TD>::ld(dg + row * N + tid);
      v.B = to_f32(Bg[row * N + tid]);
      if (rev) v.C = to_f32(Cg[row * N + tid]);
      else v.src = a.src[(kh + v.st) * N + tid];
    }
    if (!rev && tid <= N) v.off = a.off[(kh + v.st) * (N + 1) + tid];
    if (tid < P) {
      v.x = to_f32(xg[row * Pg + c0 + tid]);
      if (rev) ld_dy(a.dy, row * Pg + c0 + tid, a.dy_bf16, &v.dy);
    }
    return v;
  };
  auto commit = [&](const Vec &v, bool rev) {
    if (tid < N) {
      dsh[tid] = v.d;
      Bsh[tid] = v.B;
      if (rev) Csh[tid] = v.C;
      else srcsh[tid] = v.src;
    }
    if (!rev && tid <= N) offsh[tid] = v.off;
    if (tid < P) {
      xsh[tid] = v.x;
      if (rev) dysh[tid] = v.dy;
    }
  };
  // Hn = A_t Hc + B_t x_t^T (after commit of step t's vectors and a barrier)
  auto step_fwd = [&](const T *Hc, T *Hn) {
    FOR_RUNS(i, q) {
      const int p0 = q * VW;
      T acc[VW];
      const float bi = Bsh[i];
#pragma unroll
      for (int e = 0; e < VW; ++e) acc[e] = NT::from_real(bi * xsh[p0 + e]);
      const int r1 = offsh[i + 1];
      for (int r = offsh[i]; r < r1; ++r) {
        const int j = srcsh[r];
        const T dj = dsh[j];
        T hv[VW];
        ld_run(Hc + j * PS + p0, hv);
#pragma unroll
        for (int e = 0; e < VW; ++e) acc[e] = NT::fma(dj, hv[e], acc[e]);
      }
      st_run(Hn + i * PS + p0, acc);
    }
  };
  // [N][P] in global memory (rows ld apart) <-> [N][PV] rows in shared memory (the
  // padding columns read as zero)
  auto store_dense = [&](const T *S, T *g, int64_t ld) {
    FOR_RUNS(i, q) {
      const int p0 = q * VW;
      T v[VW];
      ld_run(S + i * PS + p0, v);
#pragma unroll
      for (int e = 0; e < VW; ++e)
        if (p0 + e < P) g[i * ld + p0 + e] = v[e];
    }
  };
  auto load_dense = [&](const T *g, T *S, int64_t ld) {
    FOR_RUNS(i, q) {
      const int p0 = q * VW;
      T v[VW];
#pragma unroll
      for (int e = 0; e < VW; ++e) v[e] = (g && p0 + e < P) ? g[i * ld + p0 + e] : NT::zero();
      st_run(S + i * PS + p0, v);
    }
  };

  // The checkpoints (the state before steps 0, kTb, 2 kTb, ...) are h0 and the
  // carries of the chunked forward scan (phases A and B at chunk length kTb), which
  // the caller computes in parallel over the chunks before this kernel.
  T *Hc = buf0, *Hn = buf1;
  Vec nv;

  // ---- reverse sweep
  T *Lam = buf2;
  __syncthreads();
  load_dense(dhg ? dhg + bh * N * Pg + c0 : nullptr, Lam, Pg);
  for (int64_t c = a.nCk - 1; c >= 0; --c) {
    const int64_t t0 = c * kTb, t1 = t0 + kTb < a.L ? t0 + kTb : a.L;
    // recompute the stretch: scratch[t - t0] = H_{t-1}; Hc ends as H_{t1-1}
    Hc = (Lam == buf0) ? buf1 : buf0;
    Hn = (Lam == buf2) ? buf1 : buf2;
    if (Lam == buf1) Hn = buf2;
    __syncthreads();
    if (c == 0) load_dense(h0g ? h0g + bh * N * Pg + c0 : nullptr, Hc, Pg);
    else load_dense(ck + (c - 1) * N * Pg, Hc, Pg);
    nv = fetch(t0, false);
    for (int64_t t = t0; t < t1; ++t) {
      __syncthreads();
      store_dense(Hc, scr + (t - t0) * N * P, P);
      commit(nv, false);
      if (t + 1 < t1) nv = fetch(t + 1, false);
      __syncthreads();
      step_fwd(Hc, Hn);
      T *tmp = Hc;
      Hc = Hn;
      Hn = tmp;
    }
    T *Hp = Hn;  // receives H_{t-1}
    Vec rv = fetch(t1 - 1, true);
    for (int64_t t = t1 - 1; t >= t0; --t) {
      const int64_t row = row_of(t);
      __syncthreads();  // [A] the previous step is done with every buffer and vector
      const int st = rv.st;
      commit(rv, true);
      if (t > t0) rv = fetch(t - 1, true);
      load_dense(scr + (t - t0) * N * P, Hp, P);
      __syncthreads();
      // [B] Lam_t = Lam'_t + C_t dy_t^T
      FOR_RUNS(i, q) {
        const int p0 = q * VW;
        T v[VW];
        ld_run(Lam + i * PS + p0, v);
        const float ci = Csh[i];
#pragma unroll
        for (int e = 0; e < VW; ++e) v[e] = NT::fma_r(ci, dysh[p0 + e], v[e]);
        st_run(Lam + i * PS + p0, v);
      }
      __syncthreads();
      // [C] dB_t, dC_t (a thread per row), and per entry k, lanes over j:
      // q_kj = sum_p Lam_t[idx_k[j]][p] conj(H_{t-1}[j][p]) (dd_t at k = s_t, dpi_t[k]).
      // These sum over the columns: a column block writes its share (sums over its own
      // columns) to the partial arrays instead.
      const int64_t prow = split ? pb * a.rows + row : row;  // row of the partial arrays
      float *dBo = split ? a.pdB : a.dB, *dCo = split ? a.pdC : a.dC;
      T *ddo = split ? static_cast<T *>(a.pdd) : ddg;
      if (tid < N) {
        float acc = 0.f;
        for (int q = 0; q < NR; ++q) {
          T v[VW];
          ld_run(Lam + tid * PS + q * VW, v);
#pragma unroll
          for (int e = 0; e < VW; ++e) acc = fmaf(re_of(v[e]), xsh[q * VW + e], acc);
        }
        dBo[prow * N + tid] = acc;
      }
      if (tid >= 128 && tid - 128 < N) {
        const int i = tid - 128;
        float acc = 0.f;
        for (int q = 0; q < NR; ++q) {
          T v[VW];
          ld_run(Hc + i * PS + q * VW, v);
#pragma unroll
          for (int e = 0; e < VW; ++e) acc = fma_re_conj(v[e], dysh[q * VW + e], acc);
        }
        dCo[prow * N + i] = acc;
      }
      for (int k = warp; k < K; k += kBT / 32) {
        float part = 0.f;
        for (int j = lane; j < N; j += 32) {
          const T *lr = Lam + idxsh[k * N + j] * PS, *hr = Hp + j * PS;
          T q0 = NT::zero(), q1 = NT::zero();  // two partial sums: a shorter dependent chain
          for (int q = 0; q < NR; ++q) {
            T l[VW], hp[VW];
            ld_run(lr + q * VW, l);
            ld_run(hr + q * VW, hp);
#pragma unroll
            for (int e = 0; e < VW; e += 2) {
              q0 = fma_conj(l[e], hp[e], q0);
              q1 = fma_conj(l[e + 1], hp[e + 1], q1);
            }
          }
          const T qv = NT::add(q0, q1);
          if (k == st) ddo[prow * N + j] = qv;
          part = fma_re_conj(dsh[j], qv, part);  // Re(conj(q) d_j)
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) {
          if (split) a.pdpi[prow * K + k] = part;
          else dpi[k] = part;
        }
      }
      __syncthreads();
      // [D] logits through the tempered softmax (warp 0); Lam'_{t-1} = A_t^H Lam_t into
      // Hc's buffer; dx_t
      if (warp == 0 && a.dlogits && !split) {
        const float v0 = lane < K ? ld_flag(a.logits, row * K + lane, a.logits_bf16) / a.tau : -INFINITY;
        const float v1 = lane + 32 < K ? ld_flag(a.logits, row * K + lane + 32, a.logits_bf16) / a.tau : -INFINITY;
        float m = fmaxf(v0, v1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float e0 = lane < K ? expf(v0 - m) : 0.f, e1 = lane + 32 < K ? expf(v1 - m) : 0.f;
        float sum = e0 + e1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float p0 = e0 / sum, p1 = e1 / sum;
        const float g0 = lane < K ? dpi[lane] : 0.f, g1 = lane + 32 < K ? dpi[lane + 32] : 0.f;
        float dot = p0 * g0 + p1 * g1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (lane < K) a.dlogits[row * K + lane] = p0 * (g0 - dot) / a.tau;
        if (lane + 32 < K) a.dlogits[row * K + lane + 32] = p1 * (g1 - dot) / a.tau;
      }
      FOR_RUNS(j, q) {
        const int p0 = q * VW;
        const T dc = conj_of(dsh[j]);
        T v[VW];
        ld_run(Lam + idxsh[st * N + j] * PS + p0, v);
#pragma unroll
        for (int e = 0; e < VW; ++e) v[e] = NT::mul(dc, v[e]);
        st_run(Hc + j * PS + p0, v);
      }
      if (tid >= 32 && tid - 32 < P) {
        const int p = tid - 32;
        float acc = 0.f;
        for (int i = 0; i < N; ++i) acc = fmaf(re_of(Lam[i * PS + p]), Bsh[i], acc);
        a.dx[row * Pg + c0 + p] = acc;
      }
      // rotate: the new adjoint is in Hc's buffer, H_{t-1} becomes the next step's H_t
      T *old = Lam;
      Lam = Hc;
      Hc = Hp;
      Hp = old;
    }
  }
  __syncthreads();
  if (a.dh0) store_dense(Lam, static_cast<T *>(a.dh0) + bh * N * Pg + c0, Pg);
#undef FOR_RUNS
}

// Column blocks' shares summed in a fixed order (block 0 first): dd, dB, dC, and dpi,
// which then goes through the tempered softmax's Jacobian into dlogits. One warp a row.
template <bool CPLX>
__global__ void __launch_bounds__(256) scan_bwd_reduce_kernel(BParams a) {
  using NT = Num<CPLX>;
  using T = typename NT::T;
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= a.rows) return;  // whole warps leave together
  const int N = (int)a.N, K = (int)a.K;
  const T *pdd = static_cast<const T *>(a.pdd);
  for (int i = lane; i < N; i += 32) {
    T dd = NT::zero();
    float dB = 0.f, dC = 0.f;
    for (int64_t pb = 0; pb < a.nPB; ++pb) {
      const int64_t o = (pb * a.rows + row) * N + i;
      dd = NT::add(dd, pdd[o]);
      dB += a.pdB[o];
      dC += a.pdC[o];
    }
    static_cast<T *>(a.dd)[row * N + i] = dd;
    a.dB[row * N + i] = dB;
    a.dC[row * N + i] = dC;
  }
  if (!a.dlogits) return;
  float g0 = 0.f, g1 = 0.f;
  for (int64_t pb = 0; pb < a.nPB; ++pb) {
    const float *pp = a.pdpi + (pb * a.rows + row) * K;
    if (lane < K) g0 += pp[lane];
    if (lane + 32 < K) g1 += pp[lane + 32];
  }
  const float v0 = lane < K ? ld_flag(a.logits, row * K + lane, a.logits_bf16) / a.tau : -INFINITY;
  const float v1 = lane + 32 < K ? ld_flag(a.logits, row * K + lane + 32, a.logits_bf16) / a.tau : -INFINITY;
  float m = fmaxf(v0, v1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float e0 = lane < K ? expf(v0 - m) : 0.f, e1 = lane + 32 < K ? expf(v1 - m) : 0.f;
  float sum = e0 + e1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float p0 = e0 / sum, p1 = e1 / sum;
  float dot = p0 * g0 + p1 * g1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  if (lane < K) a.dlogits[row * K + lane] = p0 * (g0 - dot) / a.tau;
  if (lane + 32 < K) a.dlogits[row * K + lane + 32] = p1 * (g1 - dot) / a.tau;
}

}  // namespace

size_t scan_bwd_smem_bytes(int64_t N, int64_t P, int64_t K, bool cplx) {
  const int64_t es = cplx ? 8 : 4, vw = 16 / es, pv = (P + vw - 1) / vw * vw;
  return (size_t)((3 * N * (pv + vw) + N + pv) * es + (2 * N + pv + K) * 4 + (2 * N + 1) * 4 + K * N);
}

int64_t scan_bwd_checkpoints(int64_t L) { return (L + kTb - 1) / kTb; }
int64_t scan_bwd_scratch_steps() { return kTb; }

// Column blocks per sequence: doubled while the sequences alone give fewer than two
// blocks an SM and the halves keep at least one 16-byte run of columns.
int64_t scan_bwd_column_blocks(int64_t slices, int64_t P, bool cplx) {
  const int64_t vw = cplx ? 2 : 4;
  int64_t n = 1;
  while (slices * n < 2 * 148 && P % (2 * n) == 0 && P / (2 * n) >= vw) n *= 2;
  return n;
}

cudaError_t launch_scan_bwd(const ScanBwdArgs &s, cudaStream_t st) {
  BParams a;
  a.L = s.L; a.H = s.H; a.N = s.N; a.K = s.K;
  a.Pg = s.P; a.nPB = s.nPB; a.P = s.P / s.nPB; a.rows = s.Bt * s.L * s.H;
  a.pdd = s.pdd; a.pdB = s.pdB; a.pdC = s.pdC; a.pdpi = s.pdpi;
  a.nCk = scan_bwd_checkpoints(s.L);
  a.tau = s.tau;
  a.logits_bf16 = s.logits_t == PDSSM_BF16;
  a.dy_bf16 = s.out_t == PDSSM_BF16;
  a.s = s.s; a.idx = s.ws.idx; a.off = s.ws.csr_off; a.src = s.ws.csr_src;
  a.logits = s.logits; a.d = s.d; a.B = s.B; a.C = s.C; a.x = s.x; a.dy = s.dy;
  a.h0 = s.h0; a.dh_final = s.dh_final;
  a.ckpt = s.ckpt; a.scratch = s.scratch;
  a.dlogits = s.dlogits; a.dd = s.dd; a.dB = s.dB; a.dC = s.dC; a.dx = s.dx; a.dh0 = s.dh0;
  a.err = s.ws.err;
  a.head_dicts = s.head_dicts;
  const bool cplx = s.d_t == PDSSM_C64;
  const size_t smem = scan_bwd_smem_bytes(s.N, a.P, s.K, cplx);
  const bool split = s.nPB > 1;
  void (*kern)(BParams);
#define PDSSM_BWD_KERNEL(BT)                                                                              \
  if (cplx)                                                                                               \
    kern = s.in_t == PDSSM_BF16 ? scan_bwd_kernel<true, float2, __nv_bfloat16, BT>                        \
                                : scan_bwd_kernel<true, float2, float, BT>;                               \
  else if (s.d_t == PDSSM_BF16)                                                                           \
    kern = s.in_t == PDSSM_BF16 ? scan_bwd_kernel<false, __nv_bfloat16, __nv_bfloat16, BT>                \
                                : scan_bwd_kernel<false, __nv_bfloat16, float, BT>;                       \
  else                                                                                                    \
    kern = s.in_t == PDSSM_BF16 ? scan_bwd_kernel<false, float, __nv_bfloat16, BT>                        \
                                : scan_bwd_kernel<false, float, float, BT>;
  if (split) {
    PDSSM_BWD_KERNEL(kBTSplit)
  } else {
    PDSSM_BWD_KERNEL(kBTWhole)
  }
#undef PDSSM_BWD_KERNEL
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if ((e = trace_before(st, "scan_bwd")) != cudaSuccess) return e;
  kern<<<(unsigned)(s.Bt * s.H * s.nPB), split ? kBTSplit : kBTWhole, smem, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = trace_after(st)) != cudaSuccess) return e;
  if (!split) return cudaSuccess;
  if ((e = trace_before(st, "scan_bwd_reduce")) != cudaSuccess) return e;
  const int64_t warps = a.rows, blocks = (warps * 32 + 255) / 256;
  if (cplx) scan_bwd_reduce_kernel<true><<<(unsigned)blocks, 256, 0, st>>>(a);
  else scan_bwd_reduce_kernel<false><<<(unsigned)blocks, 256, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

}  // namespace pdssm
