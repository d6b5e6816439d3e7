// Fused forward pass on sm_100a: selection, the three phases of the chunked
// scan and the output, in one kernel per (batch, head) sequence.
//
// Flash PD-SSM page, Technical Summary: Methodology 1 (hard selection of one
// one-hot-column dictionary matrix per step), Methodology 3 (phase A:
// recurrences inside chunks; phase B: prefix over chunk dependencies gives the
// carry states; phase C: carry corrections). This kernel runs the three
// phases as a software pipeline over 16-token sub-chunks of one sequence, with
// the dense contractions of the chunked form on the 5th-generation tensor
// cores and the carry state resident in tensor memory.
//
// Notation for one sub-chunk a of T = 16 steps (tau, sigma in [0, T)):
//   A_t = P_{s_t} diag(d_t)                   one-hot-column transition
//   Phi_tau = A_tau ... A_0                   prefix from the sub-chunk start
//   Psi_sigma = A_{T-1} ... A_{sigma+1}       suffix to the sub-chunk end
//   Ct_tau = Phi_tau^T C_tau      (gather)    readout seen from the start
//   Bh_sigma = Psi_sigma B_sigma  (scatter)   input seen at the end
//   G[tau][sigma] = C_tau^T A_tau...A_{sigma+1} B_sigma  (sigma <= tau)
// With S_a the state entering the sub-chunk (N x P):
//   y_tau   = S_a^T Ct_tau + sum_sigma G[tau][sigma] x_sigma        (phase A + C)
//   S_{a+1} = Phi_{T-1} S_a + sum_sigma Bh_sigma x_sigma^T          (phase B)
// Only S_{a+1} depends on S_a through a sparse map; everything else is dense:
//   U^T   = X^T Bh        (64 x 64, K = 16)  bf16 x bf16 (X exact, Bh = hi + lo)
//   Y^T   = X^T G^T       (64 x 16, K = 16)  bf16 x bf16 (G = hi + lo)
//   Y^T  += S^T Ct^T      (64 x 16, K = 64)  tf32 (S read from tensor memory)
// The tensor core reads S as tf32 (it drops the low 13 mantissa bits). The
// readout precision follows the output type:
//   bf16 y: Ct rounded to tf32, one product, relative error below 2^-10 per
//           term (the rounding of y to bf16 is 2^-9);
//   fp32 y: S_lo = S - tf32(S) kept in tensor memory and Ct split hi + lo, three
//           products hi*hi + hi*lo + lo*hi, about 21 bits.
// The state itself is accumulated in fp32. No N x N matrix is formed.
//
// State order. S_a lives in tensor memory with its rows in the source order of
// Phi_{T-1} of sub-chunk a: sources grouped by target row, increasing source
// row inside a group. A carry step then needs one 64-column load of S_a, a
// segmented sum in registers and one read-modify-write per target row. The
// prep warp of sub-chunk a composes sub-chunk a+1's indices as well, so it
// writes Bh (hence U and S_{a+1}) in sub-chunk a+1's order and Ct in its own.
// The state after the last sub-chunk is in natural order.
//
// Tensor memory holds a ring of 64-column state regions (S_a in region a mod R;
// U_a, the input term of S_{a+1}, is accumulated into region (a+1) mod R ahead
// of time) and four 16-column output slots. R = 3 for bf16 output; for fp32
// output R = 2 and the third region holds S_lo.
//
// Roles (256 threads): warps 0-3 each prepare every fourth sub-chunk's
// operands; warps 4-7 (one per tensor-memory quarter) advance the carry state
// and write y, and one thread of warp 4 issues the MMAs. Every wait is
// bounded; a timeout sets an error bit, makes every role leave its loop,
// drains outstanding MMAs and copies, and frees tensor memory.
#include <algorithm>
#include <type_traits>

#include "launch.h"
#include "sm100.cuh"

namespace pdssm {

using namespace sm100;

namespace {

constexpr int kN = 64;   // state rows
constexpr int kP = 64;   // state columns
constexpr int kT = 16;   // sub-chunk length
constexpr int kNW = 4;   // prep warp pairs; pair w prepares sub-chunks w, w + 4, ...
constexpr int kPrepWarps = 2 * kNW;
constexpr int kCarryWarp0 = kPrepWarps;  // warps 8-11 carry the state (one per tensor-memory quarter)
constexpr int kIssuerWarp = kCarryWarp0 + 4;  // warp 12: one thread issues the MMAs
constexpr int kMaxStages = 6;  // operand stages (sub-chunk a uses stage a mod nst, nst >= kNW)
constexpr int kNY = 4;   // output accumulator slots
constexpr int kThreads = 32 * (kPrepWarps + 5);  // 8 prep warps, 4 carry warps, 1 MMA-issuing warp
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s

// tensor-memory columns: 64-column state regions (a ring of 3, or 2 plus S_lo
// at column 128), then the output slots
constexpr uint32_t kColSlo = 128;
constexpr uint32_t kColY = 192;
constexpr uint32_t kTmemCols = 256;
__device__ __forceinline__ uint32_t col_state(int region) { return 64u * (uint32_t)region; }

// Operand stage layout (bytes). Strides are padded so that the prep warp's
// stores of one column spread over all shared-memory banks.
constexpr int kCtLbo = 144;                   // Ct, tf32 K-major (n = tau, k = position)
constexpr int kCtSbo = 16 * kCtLbo;           //   2 row groups of 2304 B
constexpr int kBhSbo = 144;                   // Bh, bf16 MN-major (n = position, k = sigma)
constexpr int kBhLbo = 8 * kBhSbo;            //   2 k groups of 1152 B
constexpr int kOffCt = 0;
constexpr int kOffBhHi = kOffCt + 2 * kCtSbo;
constexpr int kOffBhLo = kOffBhHi + 2 * kBhLbo;
constexpr int kOffGtHi = kOffBhLo + 2 * kBhLbo;  // G^T, bf16 K-major (n = tau, k = sigma): 512 B
constexpr int kOffGtLo = kOffGtHi + 512;
constexpr int kOffX = kOffGtLo + 512;            // x, bf16 MN-major (mn = p, k = tau): 2 KB
constexpr int kOffMeta = kOffX + 2048;           // int [N] by position: carry-step record (below)
constexpr int kOffNu = kOffMeta + 256;           // float [N] by position: Phi_{T-1} value of the source
constexpr int kOffPhiIdx = kOffNu + 256;         // int [N] by source row: Phi_{T-1} index
constexpr int kOffPhiVal = kOffPhiIdx + 256;     // float [N] by source row: Phi_{T-1} value
constexpr int kOffSrc = kOffPhiVal + 256;        // int [N] by position: source row
constexpr int kOffGDst = kOffSrc + 256;          // uint8 [N] by group ordinal: target's column in the next order
constexpr int kOffHdr = kOffGDst + 64;           // int [4]: number of groups, the group crossing position 32 (or -1)
constexpr int kOffCtLo = kOffHdr + 16;           // low part of Ct (fp32 output only), as kOffCt
__host__ __device__ constexpr int op_stage_bytes(bool precise) { return kOffCtLo + (precise ? 2 * kCtSbo : 0); }

// carry-step record of a position: whether it continues a target group (else
// it starts one), whether it ends it, and the group's ordinal
constexpr int kMetaKeep = 1 << 8;
constexpr int kMetaEnd = 1 << 9;
constexpr int kMetaOrdShift = 10;

// per-prep-warp scratch (bytes)
constexpr int kScrBins = 0;                   // int [2][N] fixed-point accumulators (by sigma parity)
constexpr int kScrCnt = 512;                  // int [N] sources per target
constexpr int kScrCntLo = 768;                // int [N] sources j < 32 per target
constexpr int kScrOffs = 1024;                // int [N] first position of each target's group
constexpr int kScrBytes = 1280;

// input stage layout: logits [T][K] raw, d/B/C [T][N] bf16, x canonical
struct InLayout {
  int logits, nlogits, d, B, C, x, bytes;  // nlogits: the next sub-chunk's logits
};

struct FParams {
  int64_t L, H;
  int K, logit_size;
  int nsub;
  const void *logits;   // null when the selections are given
  const int32_t *s_in;  // selections [Bt][L][H] (when logits is null)
  const int32_t *idx;
  const __nv_bfloat16 *d, *B, *C, *x;
  const float *h0;
  void *y;
  float *h_final;
  int32_t *prod_idx;
  float *prod_val;
  int32_t *s_out;
  uint32_t *err;
  InLayout in;
  int nst;  // operand stages
  int off_in, off_op, off_dict, off_scr, off_bar;
};

struct Bars {
  uint64_t full[kMaxStages], opfree[kMaxStages], yfull[kNY], yfree[kNY];
  // sready[k % 4]: S_k complete (all four carry warps). A ring: the carry warps
  // can complete the next state before the issuing thread has observed this one,
  // and two completions of one barrier ahead of its waiter alias in the parity test.
  uint64_t ufull[3], sready[4], slofree, drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait shared by every role: false (and the abort flag set) on timeout.
__device__ __noinline__ bool wait_bar(Bars *bars, uint64_t *bar, uint32_t parity, uint32_t *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000)) return true;
    if (*(volatile int *)&bars->abort) return false;
    if (now_ns() - t0 > kTimeoutNs) {
      *(volatile int *)&bars->abort = 1;
      flag_error(err, kErrTimeout);
      return false;
    }
  }
}

// The same bounded wait, with one decision for the whole warp.
__device__ __forceinline__ bool wait_bar_warp(Bars *bars, uint64_t *bar, uint32_t parity, uint32_t *err) {
  const bool ok = wait_bar(bars, bar, parity, err);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float tf32_trunc(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

// fp32 -> tf32, round to nearest (ties away from zero), as a 32-bit pattern
__device__ __forceinline__ float tf32_rn(float v) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(v));
  return __uint_as_float(r);
}

__device__ __forceinline__ float ld_bf16(const uint8_t *base, int idx) {
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[idx]);
}

// 2^e as a float, e clamped to the normal range
__device__ __forceinline__ float exp2i(int e) {
  e = max(-126, min(127, e));
  return __int_as_float((127 + e) << 23);
}

// operand element offsets
__device__ __forceinline__ int off_ct_pos(int pos) { return (pos >> 2) * kCtLbo + (pos & 3) * 4; }
__device__ __forceinline__ int off_ct_tau(int tau) { return (tau & 7) * 16 + (tau >> 3) * kCtSbo; }
__device__ __forceinline__ int off_bh(int pos, int sigma) {
  return (sigma & 7) * 16 + (sigma >> 3) * kBhLbo + (pos >> 3) * kBhSbo + (pos & 7) * 2;
}
__device__ __forceinline__ int off_gt(int tau, int sigma) {  // SBO = 256, LBO = 128
  return (tau & 7) * 16 + (tau >> 3) * 256 + (sigma >> 3) * 128 + (sigma & 7) * 2;
}

__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ void st_bf16_split(uint8_t *hi, uint8_t *lo, int off, float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  *reinterpret_cast<__nv_bfloat16 *>(hi + off) = h;
  *reinterpret_cast<__nv_bfloat16 *>(lo + off) = __float2bfloat16_rn(v - __bfloat162float(h));
}

// ---------------------------------------------------------------- loads

// cp.async of one sub-chunk's inputs (and the next sub-chunk's logits) into an
// input stage by one warp; rows past the end of the sequence are zero-filled.
template <typename TL>
__device__ __forceinline__ void load_inputs(const FParams &a, uint8_t *st, int64_t b, int64_t h, int sub,
                                            int lane) {
  const int t0 = sub * kT;
  const int nvalid = (int)(a.L - t0 < kT ? a.L - t0 : kT);
  const int nnext = (int)(a.L - t0 - kT < kT ? (a.L - t0 - kT > 0 ? a.L - t0 - kT : 0) : kT);
  const int64_t row0 = (b * a.L + t0) * a.H + h;  // row of token t0 in [Bt][L][H]
  // d, B, C, x: 16 rows of 128 B (8 chunks of 16 B); lane takes chunk lane % 8 of
  // rows lane / 8 + 4c, c = 0..3
  const int ch = lane & 7, tau0 = lane >> 3;
  const int64_t e0 = (row0 + (int64_t)tau0 * a.H) * kN + ch * 8;  // element offset of (tau0, ch)
  const int64_t estep = (int64_t)4 * a.H * kN;                    // 4 rows further
  const int so = tau0 * 128 + ch * 16;                            // row-major stage offset
  const int sx = (tau0 & 7) * 16 + ch * 128;                      // x: (tau%8)*16 + (tau/8)*1024 + (p/8)*128
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int tau = tau0 + 4 * c;
    const int64_t ge = e0 + c * estep;
    uint8_t *dd = st + a.in.d + so + c * 512;
    uint8_t *db = st + a.in.B + so + c * 512;
    uint8_t *dc = st + a.in.C + so + c * 512;
    uint8_t *dx = st + a.in.x + sx + ((tau0 + 4 * c) >> 3) * 1024 + ((4 * c) & 7) * 16;
    if (tau < nvalid) {
      cp_async16(dd, a.d + ge);
      cp_async16(db, a.B + ge);
      cp_async16(dc, a.C + ge);
      cp_async16(dx, a.x + ge);  // P == N
    } else {
      const uint4 z = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(dd) = z;
      *reinterpret_cast<uint4 *>(db) = z;
      *reinterpret_cast<uint4 *>(dc) = z;
      *reinterpret_cast<uint4 *>(dx) = z;
    }
  }
  if (a.logits) {
    const int lchunks = a.K * a.logit_size / 16;  // 16-byte chunks per logits row
    const uint8_t *lg = static_cast<const uint8_t *>(a.logits);
#pragma unroll 1
    for (int e = lane; e < 2 * kT * lchunks; e += 32) {
      const int nx = e >= kT * lchunks;
      const int f = e - nx * kT * lchunks;
      const int tau = f / lchunks, c = f - tau * lchunks;
      uint8_t *dst = st + (nx ? a.in.nlogits : a.in.logits) + f * 16;
      if (tau < (nx ? nnext : nvalid))
        cp_async16(dst, lg + ((row0 + (int64_t)(tau + nx * kT) * a.H) * lchunks + c) * 16);
      else
        *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
}

// Hard selection of one token from its logits row: the largest value, the lowest
// k among ties, and the first NaN if there is one. Reads 16-byte chunks.
template <typename TL>
__device__ __forceinline__ int argmax_row(const uint8_t *row, int K) {
  constexpr int kPer = 16 / (int)sizeof(TL);
  float best = 0.f;
  int bi = 0, nan_at = -1;
  for (int c = 0; c < K; c += kPer) {
    const uint4 q = *reinterpret_cast<const uint4 *>(row + c * sizeof(TL));
    const TL *e = reinterpret_cast<const TL *>(&q);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const float v = to_f32(e[u]);
      const int k = c + u;
      if (v != v && nan_at < 0) nan_at = k;
      if (k == 0 || v > best) {
        best = v;
        bi = k;
      }
    }
  }
  return nan_at >= 0 ? nan_at : bi;
}

// Positions of the 64 sources j0 = lane, j1 = lane + 32 of an index map when the
// sources are grouped by target row (targets ascending, sources ascending in a
// group). Leaves per-target counts and first positions in the warp's scratch.
__device__ __noinline__ int2 group_positions(int t0, int t1, uint8_t *ws, int lane) {
  int *cnt = reinterpret_cast<int *>(ws + kScrCnt);
  int *cntlo = reinterpret_cast<int *>(ws + kScrCntLo);
  int *offs = reinterpret_cast<int *>(ws + kScrOffs);
  cnt[lane] = 0;
  cnt[lane + 32] = 0;
  cntlo[lane] = 0;
  cntlo[lane + 32] = 0;
  __syncwarp();
  atomicAdd(&cnt[t0], 1);
  atomicAdd(&cntlo[t0], 1);
  atomicAdd(&cnt[t1], 1);
  __syncwarp();
  const int ca = cnt[2 * lane], cb = cnt[2 * lane + 1];
  int incl = ca + cb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  const int excl = incl - ca - cb;
  offs[2 * lane] = excl;
  offs[2 * lane + 1] = excl + ca;
  __syncwarp();
  const unsigned lt = (1u << lane) - 1u;
  const unsigned m0 = __match_any_sync(0xffffffffu, t0);
  const unsigned m1 = __match_any_sync(0xffffffffu, t1);
  return make_int2(offs[t0] + __popc(m0 & lt), offs[t1] + cntlo[t1] + __popc(m1 & lt));
}

// Named barrier over the two warps of a prep pair; the _and form also returns
// whether the predicate held in every thread of both warps.
__device__ __forceinline__ void pair_sync(uint32_t id) {
  asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}
__device__ __forceinline__ bool pair_and(uint32_t id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.b32 p, %1, 0;\n bar.red.and.pred q, %2, 64, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}

// ------------------------------------------------------------- MMA issue

// U_u into state region (u + 1) mod R and the intra-sub-chunk part of Y_u
// (written, not accumulated). The region held S_{u+1-R}: this is issued only
// after the carry step of sub-chunk u+1-R is complete and its readout has been
// issued (tensor-core operations of one thread execute in issue order).
template <bool kPrecise>
__device__ __noinline__ void mma_issue_input(Bars *bars, uint32_t ob, int nst, uint32_t tbase, int u) {
  constexpr int kRing = kPrecise ? 2 : 3;
  constexpr uint32_t kIdU = idesc_bf16_f32(64, kN, true, true);
  constexpr uint32_t kIdG = idesc_bf16_f32(64, kT, true, false);
  const uint32_t o = ob + (u % nst) * op_stage_bytes(kPrecise);
  const uint32_t dU = tbase + col_state((u + 1) % kRing), dY = tbase + kColY + (u % kNY) * kT;
  const uint64_t dX = smem_desc(o + kOffX, (kP / 8) * 128, 128);
  mma_bf16(dU, dX, smem_desc(o + kOffBhHi, kBhLbo, kBhSbo), kIdU, 0);
  mma_bf16(dU, dX, smem_desc(o + kOffBhLo, kBhLbo, kBhSbo), kIdU, 1);
  mma_bf16(dY, dX, smem_desc(o + kOffGtHi, 128, 256), kIdG, 0);
  mma_bf16(dY, dX, smem_desc(o + kOffGtLo, 128, 256), kIdG, 1);
  mma_commit(&bars->ufull[(u + 1) % kRing]);
}

// Readout of the entering state S_s into Y_s: A operand from tensor memory (tf32).
// Releases the operand stage (and the S_lo plane) once done.
template <bool kPrecise>
__device__ __noinline__ void mma_issue_readout(Bars *bars, uint32_t ob, int nst, uint32_t tbase, int s) {
  constexpr int kRing = kPrecise ? 2 : 3;
  constexpr uint32_t kIdC = idesc_tf32_f32(64, kT);
  const int st = s % nst;
  const uint32_t o = ob + st * op_stage_bytes(kPrecise);
  const uint32_t dY = tbase + kColY + (s % kNY) * kT, aS = tbase + col_state(s % kRing);
  const uint64_t dCt = smem_desc(o + kOffCt, kCtLbo, kCtSbo), dCl = smem_desc(o + kOffCtLo, kCtLbo, kCtSbo);
#pragma unroll
  for (int ks = 0; ks < kN / 8; ++ks) {
    const uint64_t kso = (uint64_t)((ks * 2 * kCtLbo) >> 4);  // start-address field step (no carry out)
    mma_tf32_ts(dY, aS + ks * 8, dCt + kso, kIdC, 1);
    if constexpr (kPrecise) {
      mma_tf32_ts(dY, aS + ks * 8, dCl + kso, kIdC, 1);
      mma_tf32_ts(dY, tbase + kColSlo + ks * 8, dCt + kso, kIdC, 1);
    }
  }
  mma_commit(&bars->yfull[s % kNY]);
  mma_commit(&bars->opfree[st]);
  if constexpr (kPrecise) mma_commit(&bars->slofree);
}

// ------------------------------------------------------------- the kernel

template <typename TL, typename TO, bool kPrecise>
__global__ void __launch_bounds__(kThreads, 2) fused_scan_kernel(FParams a) {
  constexpr int kRing = kPrecise ? 2 : 3;
  constexpr int kOpStage = op_stage_bytes(kPrecise);
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *in_base = smem + a.off_in;
  uint8_t *op_base = smem + a.off_op;
  uint8_t *dict = smem + a.off_dict;     // uint8 [K][N]
  uint8_t *scr = smem + a.off_scr;       // prep scratch
  Bars *bars = reinterpret_cast<Bars *>(smem + a.off_bar);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int nsub = a.nsub;

  // ---- setup
  if (tid == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&bars->full[i], 2);  // both warps of the prep pair
      mbar_init(&bars->opfree[i], 1 + 4);  // MMA commit + one arrival per carry warp
    }
    for (int i = 0; i < kNY; ++i) {
      mbar_init(&bars->yfull[i], 1);
      mbar_init(&bars->yfree[i], 4);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&bars->ufull[i], 1);
    for (int i = 0; i < 4; ++i) mbar_init(&bars->sready[i], 4);
    mbar_init(&bars->slofree, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    mbar_fence_init();
  }
  for (int e = tid; e < a.K * kN; e += kThreads) {
    int v = a.idx[e];
    if (v < 0 || v >= kN) {
      flag_error(a.err, kErrIdxRange);
      v = 0;
    }
    dict[e] = (uint8_t)v;
  }
  if (warp == kCarryWarp0) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;

  if (warp < kPrepWarps) {
    // ================================================================ prep
    // Warp pair w prepares sub-chunks w, w + kNW, ... (sub-chunk a into operand
    // stage a mod nst). Role 0 loads the inputs and builds the composites, the
    // forward chain (Ct), the carry records and the suffix scatter (Bh); role 1
    // the backward readouts and G. Lanes own rows j0 = lane and j1 = lane + 32.
    const int pair = warp >> 1, role = warp & 1;
    const uint32_t pbar = 1 + pair;
    uint8_t *in = in_base + pair * a.in.bytes;
    uint8_t *ws = scr + pair * kScrBytes;
    int *bins = reinterpret_cast<int *>(ws + kScrBins);
    if (role == 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c) bins[lane + 32 * c] = 0;
    }
    const int j0 = lane, j1 = lane + 32;
    for (int sub = pair; sub < nsub; sub += kNW) {
      const int stg = sub % a.nst;
      uint8_t *op = op_base + stg * kOpStage;
      const int t0 = sub * kT;
      const int nvalid = (int)(a.L - t0 < kT ? a.L - t0 : kT);
      const int nnext = (int)(a.L - t0 - kT < kT ? (a.L - t0 - kT > 0 ? a.L - t0 - kT : 0) : kT);
      // the inputs load while the stage is being released
      if (role == 0) {
        load_inputs<TL>(a, in, b, h, sub, lane);
        cp_async_commit();
      }
      bool ok = wait_bar_warp(bars, &bars->opfree[stg], ((sub / a.nst) & 1) ^ 1, a.err);
      if (role == 0) cp_async_wait<0>();
      // one decision for the pair; the barrier also publishes the loaded inputs
      if (!pair_and(pbar, ok)) break;

      // selections: lanes 0-15 take this sub-chunk's tokens, lanes 16-31 the next one's
      int s_lane = 0;
      {
        const int tok = lane & 15;
        const bool nx = lane >= 16;
        if (tok < (nx ? nnext : nvalid)) {
          if (a.logits) {
            s_lane = argmax_row<TL>(in + (nx ? a.in.nlogits : a.in.logits) + tok * a.K * a.logit_size, a.K);
          } else {
            s_lane = a.s_in[(b * a.L + t0 + (nx ? kT : 0) + tok) * a.H + h];
            if (s_lane < 0 || s_lane >= a.K) {
              flag_error(a.err, kErrSRange);
              s_lane = 0;
            }
          }
          if (role == 0 && !nx && a.s_out) a.s_out[(b * a.L + t0 + tok) * a.H + h] = s_lane;
        }
      }


      const uint8_t *din = in + a.in.d, *Bin = in + a.in.B, *Cin = in + a.in.C;
      if (role == 0) {
        // x into the operand stage (2 KB)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          reinterpret_cast<uint4 *>(op + kOffX)[lane + 32 * c] = reinterpret_cast<const uint4 *>(in + a.in.x)[lane + 32 * c];

        // ---- the next sub-chunk's composite (indices only) -> the order of S_{a+1}
        int posB0, posB1;
        {
          int n0 = j0, n1 = j1;
          for (int tau = 0; tau < nnext; ++tau) {
            const uint8_t *dk = dict + __shfl_sync(0xffffffffu, s_lane, 16 + tau) * kN;
            n0 = dk[n0];
            n1 = dk[n1];
          }
          { const int2 pp = group_positions(n0, n1, ws, lane); posB0 = pp.x; posB1 = pp.y; }
        }
        __syncwarp();

        // ---- Phi_{T-1} (indices): the positions of S_a's order
        int posA0, posA1, i0 = j0, i1 = j1;
        for (int tau = 0; tau < nvalid; ++tau) {
          const uint8_t *dk = dict + __shfl_sync(0xffffffffu, s_lane, tau) * kN;
          i0 = dk[i0];
          i1 = dk[i1];
        }
        { const int2 pp = group_positions(i0, i1, ws, lane); posA0 = pp.x; posA1 = pp.y; }
        // ---- forward chain: Phi_tau and Ct_tau = Phi_tau^T C_tau at the positions of S_a's order
        float v0 = 1.f, v1 = 1.f;
        {
          const int o0 = kOffCt + off_ct_pos(posA0), o1 = kOffCt + off_ct_pos(posA1);
          int f0 = j0, f1 = j1;
#pragma unroll 1
          for (int tau = 0; tau < kT; ++tau) {
            const uint8_t *dk = dict + __shfl_sync(0xffffffffu, s_lane, tau) * kN;
            float c0 = 0.f, c1 = 0.f;
            if (tau < nvalid) {
              v0 *= ld_bf16(din, tau * kN + f0);
              v1 *= ld_bf16(din, tau * kN + f1);
              f0 = dk[f0];
              f1 = dk[f1];
              c0 = v0 * ld_bf16(Cin, tau * kN + f0);
              c1 = v1 * ld_bf16(Cin, tau * kN + f1);
            }
            float *c0p = reinterpret_cast<float *>(op + o0 + off_ct_tau(tau));
            float *c1p = reinterpret_cast<float *>(op + o1 + off_ct_tau(tau));
            if constexpr (kPrecise) {  // hi as fp32 (read as tf32), lo = the rest
              c0p[0] = c0;
              c1p[0] = c1;
              c0p[(kOffCtLo - kOffCt) / 4] = c0 - tf32_trunc(c0);
              c1p[(kOffCtLo - kOffCt) / 4] = c1 - tf32_trunc(c1);
            } else {
              c0p[0] = tf32_rn(c0);
              c1p[0] = tf32_rn(c1);
            }
          }
        }
        // ---- Phi_{T-1} = (i, v): carry-step records
        {
          const int *cnt = reinterpret_cast<const int *>(ws + kScrCnt);
          const int *offs = reinterpret_cast<const int *>(ws + kScrOffs);
          // ordinal of each nonempty target group (targets ascending): target t's is
          // the exclusive count of nonempty targets below t
          const int na = cnt[2 * lane] > 0, nb = cnt[2 * lane + 1] > 0;
          int incl = na + nb;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
          }
          const int gex = incl - na - nb;
          const int n_img = __shfl_sync(0xffffffffu, incl, 31);
          const int g0 = __shfl_sync(0xffffffffu, gex, i0 >> 1), h0 = __shfl_sync(0xffffffffu, na, i0 >> 1);
          const int g1 = __shfl_sync(0xffffffffu, gex, i1 >> 1), h1 = __shfl_sync(0xffffffffu, na, i1 >> 1);
          const int e0 = g0 + ((i0 & 1) ? h0 : 0), e1 = g1 + ((i1 & 1) ? h1 : 0);
          // the target's column in the next order: posB of row i (held by lane i & 31)
          const int pb0a = __shfl_sync(0xffffffffu, posB0, i0 & 31), pb0b = __shfl_sync(0xffffffffu, posB1, i0 & 31);
          const int pb1a = __shfl_sync(0xffffffffu, posB0, i1 & 31), pb1b = __shfl_sync(0xffffffffu, posB1, i1 & 31);
          const int f0 = offs[i0], f1 = offs[i1];
          const bool keep0 = posA0 != f0, keep1 = posA1 != f1;
          const bool end0 = posA0 == f0 + cnt[i0] - 1, end1 = posA1 == f1 + cnt[i1] - 1;
          int *meta = reinterpret_cast<int *>(op + kOffMeta);
          meta[posA0] = (keep0 ? kMetaKeep : 0) | (end0 ? kMetaEnd : 0) | (e0 << kMetaOrdShift);
          meta[posA1] = (keep1 ? kMetaKeep : 0) | (end1 ? kMetaEnd : 0) | (e1 << kMetaOrdShift);
          if (end0) op[kOffGDst + e0] = (uint8_t)(i0 < 32 ? pb0a : pb0b);
          if (end1) op[kOffGDst + e1] = (uint8_t)(i1 < 32 ? pb1a : pb1b);
          int *hdr = reinterpret_cast<int *>(op + kOffHdr);
          if (lane == 0) hdr[0] = n_img;
          if (posA0 == 32) hdr[1] = keep0 ? e0 : -1;
          if (posA1 == 32) hdr[1] = keep1 ? e1 : -1;
          reinterpret_cast<float *>(op + kOffNu)[posA0] = v0;
          reinterpret_cast<float *>(op + kOffNu)[posA1] = v1;
          reinterpret_cast<int *>(op + kOffSrc)[posA0] = j0;
          reinterpret_cast<int *>(op + kOffSrc)[posA1] = j1;
          reinterpret_cast<int *>(op + kOffPhiIdx)[j0] = i0;
          reinterpret_cast<int *>(op + kOffPhiIdx)[j1] = i1;
          reinterpret_cast<float *>(op + kOffPhiVal)[j0] = v0;
          reinterpret_cast<float *>(op + kOffPhiVal)[j1] = v1;
        }


        // ---- backward: the suffix Psi_sigma and Bh_sigma = Psi_sigma B_sigma as an
        //      exact fixed-point sum (integer adds are order-independent), written at
        //      the target's position in S_{a+1}'s order. Steps past the end of the
        //      sequence are the identity; their B rows were zero-filled.
        int k0 = j0, k1 = j1;          // Psi_sigma
        float m0 = 1.f, m1 = 1.f;
#pragma unroll 1
        for (int sg = kT - 1; sg >= 0; --sg) {
          const bool sv = sg < nvalid;
          const float bs0 = ld_bf16(Bin, sg * kN + j0), bs1 = ld_bf16(Bin, sg * kN + j1);
          int *bn = bins + (sg & 1) * kN;  // the other parity's accumulators serve the next step
          const float w0 = m0 * bs0, w1 = m1 * bs1;
          const unsigned mb = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fabsf(w0), fabsf(w1))));
          // |w| < 2^ex; 64 terms of magnitude < 2^24 stay below 2^30
          const int ex = (int)((mb >> 23) & 0xff) - 126;
          const int e = mb ? 24 - ex : 0;
          const float up = exp2i(e), dn = exp2i(-e);
          atomicAdd(&bn[k0], __float2int_rn(w0 * up));
          atomicAdd(&bn[k1], __float2int_rn(w1 * up));
          // Psi_{sg-1} = Psi_sg A_sg: column j <- d[j] * column idx[j]
          {
            const uint8_t *dk = dict + __shfl_sync(0xffffffffu, s_lane, sg) * kN;
            const int r0 = sv ? dk[j0] : j0, r1 = sv ? dk[j1] : j1;
            const float d0 = sv ? ld_bf16(din, sg * kN + j0) : 1.f, d1 = sv ? ld_bf16(din, sg * kN + j1) : 1.f;
            const int ka = __shfl_sync(0xffffffffu, k0, r0 & 31), kb = __shfl_sync(0xffffffffu, k1, r0 & 31);
            const float ma = __shfl_sync(0xffffffffu, m0, r0 & 31), mb2 = __shfl_sync(0xffffffffu, m1, r0 & 31);
            const int kc = __shfl_sync(0xffffffffu, k0, r1 & 31), kd = __shfl_sync(0xffffffffu, k1, r1 & 31);
            const float mc = __shfl_sync(0xffffffffu, m0, r1 & 31), md = __shfl_sync(0xffffffffu, m1, r1 & 31);
            k0 = r0 < 32 ? ka : kb;
            m0 = (r0 < 32 ? ma : mb2) * d0;
            k1 = r1 < 32 ? kc : kd;
            m1 = (r1 < 32 ? mc : md) * d1;
          }
          __syncwarp();
          const float bh0 = (float)bn[j0] * dn, bh1 = (float)bn[j1] * dn;
          bn[j0] = 0;
          bn[j1] = 0;
          st_bf16_split(op + kOffBhHi, op + kOffBhLo, off_bh(posB0, sg), bh0);
          st_bf16_split(op + kOffBhHi, op + kOffBhLo, off_bh(posB1, sg), bh1);
        }
      } else {
        // ---- backward readouts R_sigma[j][tau] = (A_tau...A_{sigma+1})^T C_tau and
        //      G[tau][sigma] = B_sigma . R_sigma[:, tau]. Columns tau < sigma are zero
        //      and stay zero under the gathers; rows past the end of the sequence
        //      were zero-filled, so their columns stay zero too.
        reinterpret_cast<uint4 *>(op + kOffGtHi)[lane] = make_uint4(0, 0, 0, 0);  // G^T above the diagonal
        reinterpret_cast<uint4 *>(op + kOffGtHi)[lane + 32] = make_uint4(0, 0, 0, 0);
        float R0[kT], R1[kT];
#pragma unroll
        for (int c = 0; c < kT; ++c) R0[c] = R1[c] = 0.f;
        // lo_c: readout columns [lo, T) can be nonzero (sigma >= lo)
        auto readout_step = [&](auto lo_c, int sg) {
          constexpr int lo = decltype(lo_c)::value;
          const float bs0 = ld_bf16(Bin, sg * kN + j0), bs1 = ld_bf16(Bin, sg * kN + j1);
          // R_sg = A_{sg+1}^T R_{sg+1} on the columns tau > sg
          {
            const int sn = sg + 1 < kT ? sg + 1 : sg;
            const uint8_t *dk = dict + __shfl_sync(0xffffffffu, s_lane, sn) * kN;
            const int r0 = dk[j0], r1 = dk[j1];
            const float d0 = ld_bf16(din, sn * kN + j0), d1 = ld_bf16(din, sn * kN + j1);
#pragma unroll
            for (int tau = lo + 1; tau < kT; ++tau) {
              const float a0 = __shfl_sync(0xffffffffu, R0[tau], r0 & 31);
              const float a1 = __shfl_sync(0xffffffffu, R1[tau], r0 & 31);
              const float c0 = __shfl_sync(0xffffffffu, R0[tau], r1 & 31);
              const float c1 = __shfl_sync(0xffffffffu, R1[tau], r1 & 31);
              R0[tau] = d0 * (r0 < 32 ? a0 : a1);
              R1[tau] = d1 * (r1 < 32 ? c0 : c1);
            }
          }
          // R_sg[:, sg] = C_sg (sg is in [lo, lo + 8))
          {
            const float c0 = ld_bf16(Cin, sg * kN + j0), c1 = ld_bf16(Cin, sg * kN + j1);
#pragma unroll
            for (int tau = lo; tau < lo + 8; ++tau) {
              R0[tau] = tau == sg ? c0 : R0[tau];
              R1[tau] = tau == sg ? c1 : R1[tau];
            }
          }
          // G[tau][sg] for tau in [8 * rnd, 8 * rnd + 8): partials, then a
          // reduce-scatter of 8 values over 32 lanes
#pragma unroll
          for (int rnd = lo / 8; rnd < 2; ++rnd) {
            float g[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) g[c] = bs0 * R0[8 * rnd + c] + bs1 * R1[8 * rnd + c];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const bool upr = lane & 16;
              const float send = upr ? g[c] : g[c + 4];
              const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
              g[c] = (upr ? g[c + 4] : g[c]) + recv;
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const bool upr = lane & 8;
              const float send = upr ? g[c] : g[c + 2];
              const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
              g[c] = (upr ? g[c + 2] : g[c]) + recv;
            }
            {
              const bool upr = lane & 4;
              const float send = upr ? g[0] : g[1];
              const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
              g[0] = (upr ? g[1] : g[0]) + recv;
            }
            g[0] += __shfl_xor_sync(0xffffffffu, g[0], 2);
            g[0] += __shfl_xor_sync(0xffffffffu, g[0], 1);
            if ((lane & 3) == 0) {
              const int tau = 8 * rnd + ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
              st_bf16_split(op + kOffGtHi, op + kOffGtLo, off_gt(tau, sg), g[0]);
            }
          }
        };
#pragma unroll 1
        for (int sg = kT - 1; sg >= 8; --sg) readout_step(std::integral_constant<int, 8>(), sg);
#pragma unroll 1
        for (int sg = 7; sg >= 0; --sg) readout_step(std::integral_constant<int, 0>(), sg);
      }

      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->full[stg]);
      // both warps are done with the input stage before the next load overwrites it
      pair_sync(pbar);
    }
  } else if (warp < kIssuerWarp) {
    // ============================================ carry state and output (warps 8-11)
    const int q = warp & 3;                 // tensor-memory quarter
    const bool act = lane < 16;
    const int p = 16 * q + lane;            // state column owned by this lane
    const uint32_t lanebase = (uint32_t)(32 * q) << 16;
    bool ok = true;
    // S_0 = h0 (or 0) in the source order of sub-chunk 0's composite
    if (nsub > 0 && !wait_bar_warp(bars, &bars->full[0], 0, a.err)) ok = false;
    if (__all_sync(0xffffffffu, ok)) {
      const int *src0 = reinterpret_cast<const int *>(op_base + kOffSrc);
      float v[16];
      for (int c0 = 0; c0 < kN; c0 += 16) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int row = nsub > 0 ? src0[c0 + i] : c0 + i;
          v[i] = (act && a.h0) ? a.h0[((b * a.H + h) * kN + row) * kP + p] : 0.f;
        }
        tmem_st16(tbase + lanebase + col_state(0) + c0, v);
        if constexpr (kPrecise) {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] -= tf32_trunc(v[i]);
          tmem_st16(tbase + lanebase + kColSlo + c0, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->sready[0]);
    }
    TO *yout = static_cast<TO *>(a.y);
    // output rows of sub-chunk sub from its accumulator slot (already loaded)
    auto store_y = [&](int sub, const float *v) {
      const int t0 = sub * kT;
      const int nvalid = (int)(a.L - t0 < kT ? a.L - t0 : kT);
      if (act) {
#pragma unroll
        for (int tau = 0; tau < kT; ++tau)
          if (tau < nvalid) store_out(yout + ((b * a.L + t0 + tau) * a.H + h) * kP + p, v[tau]);
      }
    };
    int pidx0 = lane, pidx1 = lane + 32;
    float pval0 = 1.f, pval1 = 1.f;
    int done = 0;  // sub-chunks whose carry step completed
    for (int sub = 0; sub < nsub; ++sub) {
      if (!__all_sync(0xffffffffu, ok)) break;
      const int st = sub % a.nst;
      const uint8_t *op = op_base + st * kOpStage;
      if (!wait_bar_warp(bars, &bars->ufull[(sub + 1) % kRing], (sub / kRing) & 1, a.err)) break;
      if (!wait_bar_warp(bars, &bars->full[st], (sub / a.nst) & 1, a.err)) break;
      if (sub > 0 && !wait_bar_warp(bars, &bars->yfull[(sub - 1) % kNY], ((sub - 1) / kNY) & 1, a.err)) break;
      tc_fence_after();
      const uint32_t RS = tbase + lanebase + col_state(sub % kRing);
      const uint32_t RU = tbase + lanebase + col_state((sub + 1) % kRing);
      const int4 *meta4 = reinterpret_cast<const int4 *>(op + kOffMeta);
      const float4 *nu4 = reinterpret_cast<const float4 *>(op + kOffNu);
      // running whole-sequence product (warp 4 keeps it; sub-chunks arrive in order)
      if (q == 0) {
        const int *pi = reinterpret_cast<const int *>(op + kOffPhiIdx);
        const float *pv = reinterpret_cast<const float *>(op + kOffPhiVal);
        pval0 *= pv[pidx0];
        pval1 *= pv[pidx1];
        pidx0 = pi[pidx0];
        pidx1 = pi[pidx1];
      }
      // S_{a+1}[i] = U[i] + sum_{j: Phi[j] = i} nu_j S_a[j], in place over U. The
      // sources of a target are adjacent in S_a, so a segmented sum over the
      // positions yields each target's total at its group's last position. All 32
      // threads work: thread (hh, pl) holds state column 16 q + pl at positions
      // [32 hh, 32 hh + 32). The previous sub-chunk's output rides on the same
      // tensor-memory round trip.
      {
        const int hh = lane >> 4, pl = lane & 15;
        float v[32];
        tmem_ld_x2_32<32>(RS, v);
        float yv[8];
        if (sub > 0) tmem_ld_x2_8<8>(tbase + lanebase + kColY + ((sub - 1) % kNY) * kT, yv);
        tmem_wait_ld();
        if (sub > 0) {
          const int tp = (sub - 1) * kT;
          const int nv = (int)(a.L - tp < kT ? a.L - tp : kT);
          TO *yrow = yout + ((b * a.L + tp + 8 * hh) * a.H + h) * kP + 16 * q + pl;
          const int64_t ystep = a.H * kP;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (8 * hh + i < nv) store_out(yrow + i * ystep, yv[i]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->yfree[(sub - 1) % kNY]);
        }
        const int *hdr = reinterpret_cast<const int *>(op + kOffHdr);
        const int n_img = hdr[0], ecross = hdr[1];
        // group totals go through this warp's 1 KB of the stage's Bh area (its MMA
        // completed before ufull was signalled)
        float *cs = reinterpret_cast<float *>(const_cast<uint8_t *>(op) + kOffBhHi) + q * 256;
        for (int base = 0; base < n_img; base += 16) {
          float run = 0.f;
#pragma unroll
          for (int r4 = 0; r4 < 8; ++r4) {
            const int4 m4 = meta4[8 * hh + r4];
            const float4 n4 = nu4[8 * hh + r4];
            const int mt[4] = {m4.x, m4.y, m4.z, m4.w};
            const float nu[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              run = (mt[c] & kMetaKeep) ? run : 0.f;
              run = fmaf(nu[c], v[4 * r4 + c], run);
              const unsigned e = (unsigned)((mt[c] >> kMetaOrdShift) - base);
              if ((mt[c] & kMetaEnd) && e < 16u) cs[e * 16 + pl] = run;
            }
          }
          // the group that crosses positions 31 | 32 gets the lower half's part
          const float tail = __shfl_sync(0xffffffffu, run, pl);
          const unsigned ec = (unsigned)(ecross - base);
          if (hh == 1 && ecross >= 0 && ec < 16u) cs[ec * 16 + pl] += tail;
          __syncwarp();
          // U at the group ends += group totals, eight at a time
#pragma unroll 1
          for (int e8 = base; e8 < base + 16 && e8 < n_img; e8 += 8) {
            float u[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) tmem_ld1_if(RU + op[kOffGDst + e8 + e], u[e], e8 + e < n_img);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e)
              tmem_st1_if(RU + op[kOffGDst + e8 + e], u[e] + cs[(e8 - base + e) * 16 + pl], e8 + e < n_img);
          }
          __syncwarp();
        }
      }
      tmem_wait_st();
      if constexpr (kPrecise) {
        // tf32 low part of S_{a+1}, once the readout of S_a is done with the plane
        if (!wait_bar_warp(bars, &bars->slofree, sub & 1, a.err)) break;
        tc_fence_after();
        float v[32];
        tmem_ld_x2_32<32>(RU, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] -= tf32_trunc(v[i]);
        tmem_st_x2_32<32>(tbase + lanebase + kColSlo, v);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->sready[(sub + 1) & 3]);
        mbar_arrive(&bars->opfree[st]);
      }
      done = sub + 1;
    }
    // output of the last sub-chunk
    if (__all_sync(0xffffffffu, ok) && done == nsub && nsub > 0 &&
        wait_bar_warp(bars, &bars->yfull[(nsub - 1) % kNY], ((nsub - 1) / kNY) & 1, a.err)) {
      tc_fence_after();
      float v[16];
      tmem_ld16(tbase + lanebase + kColY + ((nsub - 1) % kNY) * kT, v);
      tmem_wait_ld();
      store_y(nsub - 1, v);
    }
    const bool clean = !*(volatile int *)&bars->abort;
    if (q == 0 && clean) {
      const int64_t o = (b * a.H + h) * kN;
      if (a.prod_idx) {
        a.prod_idx[o + lane] = pidx0;
        a.prod_idx[o + lane + 32] = pidx1;
      }
      if (a.prod_val) {
        a.prod_val[o + lane] = pval0;
        a.prod_val[o + lane + 32] = pval1;
      }
    }
    if (clean && a.h_final) {
      const uint32_t RF = tbase + lanebase + col_state(nsub % kRing);
      for (int c0 = 0; c0 < kN; c0 += 16) {
        float v[16];
        tmem_ld16(RF + c0, v);
        tmem_wait_ld();
        if (act)
          for (int i = 0; i < 16; ++i) a.h_final[((b * a.H + h) * kN + c0 + i) * kP + p] = v[i];
      }
    }
    __syncwarp();

  } else if (lane == 0) {
    // ============================================ MMA issue (warp 12, one thread)
    const uint32_t ob = smem_u32(op_base);
    auto issue_u_now = [&](int u) { mma_issue_input<kPrecise>(bars, ob, a.nst, tbase, u); };
    auto issue_y_now = [&](int s_) { mma_issue_readout<kPrecise>(bars, ob, a.nst, tbase, s_); };
    // issue U groups up to `upto`: waiting for their operands and output slot when
    // `block`, else only those already ready
    int next_u = 0;
    auto issue_us = [&](int upto, bool block) -> bool {
      for (; next_u <= upto && next_u < nsub; ++next_u) {
        const int st = next_u % a.nst;
        uint64_t *fb = &bars->full[st];
        const uint32_t fp = (next_u / a.nst) & 1;
        const bool needy = next_u >= kNY;
        uint64_t *yb = &bars->yfree[next_u % kNY];
        const uint32_t yp = ((next_u / kNY) - 1) & 1;
        if (!block) {
          if (!mbar_test_wait(fb, fp) || (needy && !mbar_test_wait(yb, yp))) return true;
        } else {
          if (!mbar_test_wait(fb, fp) && !wait_bar(bars, fb, fp, a.err)) return false;
          if (needy && !mbar_test_wait(yb, yp) && !wait_bar(bars, yb, yp, a.err)) return false;
        }
        tc_fence_after();
        issue_u_now(next_u);
      }
      return true;
    };
    auto issue_y = [&](int s) -> bool {
      uint64_t *sb = &bars->sready[s & 3];
      if (!mbar_test_wait(sb, (s >> 2) & 1) && !wait_bar(bars, sb, (s >> 2) & 1, a.err)) return false;
      tc_fence_after();
      issue_y_now(s);
      return true;
    };
    // U_0 (and U_1 when ready), the readout of S_0 once the carry warps wrote it,
    // then per sub-chunk s, once S_{s+1} is complete: U_{s+1} (its output part
    // must precede the readout of S_{s+1}: it is written, not accumulated), the
    // input term furthest ahead that the ring allows if its operands are ready
    // (the next carry steps wait for it), the readout of S_{s+1}, and that input
    // term after all.
    bool ok = issue_us(0, true) && issue_us(kRing - 2, false) && (nsub == 0 || issue_y(0));
    for (int s = 0; ok && s + 1 < nsub; ++s) {
      uint64_t *sb = &bars->sready[(s + 1) & 3];
      ok = mbar_test_wait(sb, ((s + 1) >> 2) & 1) || wait_bar(bars, sb, ((s + 1) >> 2) & 1, a.err);
      ok = ok && issue_us(s + 1, true) && issue_us(s + kRing - 1, false) && issue_y(s + 1) &&
           issue_us(s + kRing - 1, true);
    }
    // every MMA issued so far has completed once this arrives
    mma_commit(&bars->drain);
    const uint64_t t0 = now_ns();
    while (!mbar_try_wait(&bars->drain, 0) && now_ns() - t0 < kTimeoutNs) {
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kCarryWarp0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace

bool fused_scan_applies(const pdssm_problem *pb) {
  if (pb->flags & PDSSM_FLAG_REFERENCE_PATH) return false;
  if (pb->chunk != 0 && pb->chunk != kT) return false;
  if (pb->state_t != PDSSM_F32 || pb->N != kN || pb->P != kP) return false;
  if (pb->d_t != PDSSM_BF16 || pb->in_t != PDSSM_BF16) return false;
  const int lsz = pb->logits_t == PDSSM_BF16 ? 2 : 4;
  return (pb->K * lsz) % 16 == 0;
}

bool fused_scan_pointers_ok(const ScanArgs &s) {
  if (!s.logits && !s.s) return false;
  auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return (!s.logits || al16(s.logits)) && al16(s.d) && al16(s.B) && al16(s.C) && al16(s.x);
}

cudaError_t launch_fused_scan(const ScanArgs &s, cudaStream_t st) {
  FParams a;
  a.L = s.L;
  a.H = s.H;
  a.K = (int)s.K;
  a.logit_size = s.logits_t == PDSSM_BF16 ? 2 : 4;
  a.nsub = (int)((s.L + kT - 1) / kT);
  a.logits = s.logits;
  a.s_in = s.logits ? nullptr : s.s;
  a.idx = s.idx;
  a.d = static_cast<const __nv_bfloat16 *>(s.d);
  a.B = static_cast<const __nv_bfloat16 *>(s.B);
  a.C = static_cast<const __nv_bfloat16 *>(s.C);
  a.x = static_cast<const __nv_bfloat16 *>(s.x);
  a.h0 = static_cast<const float *>(s.h0);
  a.y = s.y;
  a.h_final = static_cast<float *>(s.h_final);
  a.prod_idx = s.prod_idx;
  a.prod_val = static_cast<float *>(s.prod_val);
  a.s_out = s.s_out;
  a.err = s.ws.err;
  // input stage
  int o = 0;
  a.in.logits = o; o += s.logits ? kT * a.K * a.logit_size : 0; o = (o + 127) & ~127;
  a.in.nlogits = o; o += s.logits ? kT * a.K * a.logit_size : 0; o = (o + 127) & ~127;
  a.in.d = o; o += kT * kN * 2;
  a.in.B = o; o += kT * kN * 2;
  a.in.C = o; o += kT * kN * 2;
  a.in.x = o; o += kT * kP * 2;
  a.in.bytes = (o + 127) & ~127;
  // smem
  // As many operand stages as fit two CTAs per SM (at least one per prep warp).
  const bool precise = s.out_t != PDSSM_BF16;
  constexpr int kTwoCtaBytes = 228 * 1024 / 2 - 1024;  // per-CTA share of an SM, less the reserved 1 KB
  int off = 0;
  for (a.nst = kMaxStages; a.nst >= kNW; --a.nst) {
    off = 0;
    a.off_op = off; off += a.nst * op_stage_bytes(precise); off = (off + 1023) & ~1023;
    a.off_in = off; off += kNW * a.in.bytes;
    a.off_dict = off; off += (int)((s.K * kN + 127) & ~127);
    a.off_scr = off; off += kNW * kScrBytes;
    off = (off + 127) & ~127;
    a.off_bar = off; off += (int)sizeof(Bars);
    if (off <= kTwoCtaBytes) break;
  }
  if (a.nst < kNW) a.nst = kNW;  // the last layout computed (nst = kNW) is kept

  cudaError_t e;
  auto kern = (s.logits_t == PDSSM_BF16)
                  ? (precise ? fused_scan_kernel<__nv_bfloat16, float, true>
                             : fused_scan_kernel<__nv_bfloat16, __nv_bfloat16, false>)
                  : (precise ? fused_scan_kernel<float, float, true>
                             : fused_scan_kernel<float, __nv_bfloat16, false>);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, off);
  if (e != cudaSuccess) return e;
  if ((e = trace_before(st, "fused_scan")) != cudaSuccess) return e;
  kern<<<(unsigned)(s.Bt * s.H), kThreads, off, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return trace_after(st);
}

}  // namespace pdssm
