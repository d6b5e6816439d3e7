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
// Roles (352 threads, 11 warps):
//   warps 0-5   three prep pairs; pair w prepares sub-chunks w, w + 3, ... into
//               operand stage (sub-chunk mod nst). Both warps of a pair run
//               "walkers": walker (sigma, j) starts at row j after step sigma and
//               follows it through the later steps' maps, carrying B_sigma[j] times
//               the d it passes; it meets C_tau on its way (its part of
//               G[tau][sigma]) and ends at Psi_sigma(j) (its part of Bh_sigma).
//               The walkers of sigma = -1 give Ct and Phi_{T-1} (the carry records
//               and S_a's order). Warp X (even) also orders S_{a+1}; warp Y (odd)
//               orders S_a and runs the sigma = -1 walk.
//   warps 6-9   carry the state (one per tensor-memory lane quarter) and write y
//               two sub-chunks behind the carry.
//   warp 10     one thread issues the MMAs.
// Every wait is bounded; a timeout sets an error bit, makes every role leave its
// loop, drains outstanding MMAs and copies, and frees tensor memory.
#include <algorithm>
#include <climits>
#include <type_traits>

#include "launch.h"
#include "sm100.cuh"

namespace pdssm {

using namespace sm100;

namespace {

constexpr int kN = 64;   // state rows
constexpr int kP = 64;   // state columns
constexpr int kT = 16;   // sub-chunk length
constexpr int kNW = 3;   // prep warp pairs; pair w prepares sub-chunks w, w + kNW, ...
constexpr int kPrepWarps = 2 * kNW;
constexpr int kCarryWarp0 = kPrepWarps;  // warps 6-9 carry the state (one per tensor-memory quarter)
constexpr int kIssuerWarp = kCarryWarp0 + 4;  // warp 10: one thread issues the MMAs
constexpr int kMaxStages = 6;  // operand stages (sub-chunk a uses stage a mod nst, nst >= kNW)
constexpr int kNY = 4;   // output accumulator slots
constexpr int kYLag = 2;  // the carry step of sub-chunk a writes the output of sub-chunk a - kYLag
constexpr int kThreads = 32 * (kPrepWarps + 5);  // 6 prep warps, 4 carry warps, 1 MMA-issuing warp
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s
constexpr uint64_t kShortTimeoutNs = 1000ull;     // 1 us (failure-detection testing)

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

// carry-step record of a position: bit 0 = it continues a target group (else it
// starts one); bits 8-14 = the group's ordinal (kOrdNone: another thread writes the
// group's total); bits 16-31 = the byte offset, in a carry warp's group-total
// rows, where the first pass (groups 0-15) stores the position's running sum
// (row 16 absorbs the positions of other groups)
constexpr int kMetaKeep = 1;
constexpr int kMetaOrdShift = 8;
constexpr int kMetaOffShift = 16;
constexpr int kOrdNone = 127;
__host__ __device__ constexpr int meta_word(bool keep, int ord) {
  return (keep ? kMetaKeep : 0) | (ord << kMetaOrdShift) | ((ord < 16 ? ord : 16) * 64 << kMetaOffShift);
}

// per-pair scratch (bytes); warp X = the pair's even warp, warp Y the odd one
constexpr int kQBytes = 2 * kT * 32 * 4;      // float [2 slots][16 tau][32 lanes] partial G
constexpr int kScrQX = 0;                     // partial G of warp X's walks
constexpr int kScrQY = kScrQX + kQBytes;      // partial G of warp Y's walks
constexpr int kScrBinsX = kScrQY + kQBytes;   // int [2][N] fixed-point accumulators of warp X
constexpr int kScrBinsY = kScrBinsX + 512;    // int [2][N] of warp Y
constexpr int kScrGrpX = kScrBinsY + 512;     // warp X's grouping scratch (counts, offsets: 768 B)
constexpr int kScrGrpY = kScrGrpX + 768;      // warp Y's grouping scratch
constexpr int kScrPosB = kScrGrpY + 768;      // uint8 [N] position of row i in S_{a+1}'s order
constexpr int kScrPosA = kScrPosB + 64;       // uint8 [N] position of row j in S_a's order
constexpr int kScrSel = kScrPosA + 64;        // int [2T] selections of this and the next sub-chunk
constexpr int kScrBytes = ((kScrSel + 4 * 2 * kT) + 127) & ~127;
// offsets inside a grouping scratch (group_positions)
constexpr int kScrCnt = 0;                    // int [N] sources per target
constexpr int kScrCntLo = 256;                // int [N] sources j < 32 per target
constexpr int kScrOffs = 512;                 // int [N] first position of each target's group

// input stage layout: logits [T][K] raw (this and the next sub-chunk), d/B/C [T][N] bf16
struct InLayout {
  int logits, nlogits, d, B, C, bytes;
};

struct FParams {
  int64_t L, H;
  int K, logit_size;
  int nsub;
  const void *logits;   // null when the selections (or the steps' transitions) are given
  const int32_t *s_in;  // selections [Bt][L][H] (when logits is null)
  const uint8_t *steps; // per-step transitions [Bt][L][H][N] (the original PD-SSM), or null
  int row_bytes;        // bytes of one staged logits / transition row (0: selections given)
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
  bool short_waits;
  bool head_dicts;  // idx is [H][K][N]
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
  uint64_t wait_ns;  // limit of the roles' waits (the final drain always uses kTimeoutNs)
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
    if (mbar_try_wait_sleep(bar, parity, bars->wait_ns < 20000 ? (uint32_t)bars->wait_ns : 20000u)) return true;
    if (*(volatile int *)&bars->abort) return false;
    if (now_ns() - t0 > bars->wait_ns) {
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

// two adjacent values as bf16 hi + lo pairs (one 4-byte store per part)
__device__ __forceinline__ void st_bf16x2_split(uint8_t *hi, uint8_t *lo, int off, float v0, float v1) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
  const float2 hf = __bfloat1622float2(h);
  *reinterpret_cast<__nv_bfloat162 *>(hi + off) = h;
  *reinterpret_cast<__nv_bfloat162 *>(lo + off) = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
}

// ---------------------------------------------------------------- loads

// cp.async of one sub-chunk's d, B, C and logits (and the next sub-chunk's
// logits) into an input stage by one warp; rows past the end of the sequence
// are zero-filled.
__device__ __forceinline__ void load_inputs(const FParams &a, uint8_t *st, int64_t b, int64_t h, int sub,
                                            int lane) {
  const int t0 = sub * kT;
  const int nvalid = (int)(a.L - t0 < kT ? a.L - t0 : kT);
  const int nnext = (int)(a.L - t0 - kT < kT ? (a.L - t0 - kT > 0 ? a.L - t0 - kT : 0) : kT);
  const int64_t row0 = (b * a.L + t0) * a.H + h;  // row of token t0 in [Bt][L][H]
  // 16 rows of 128 B (8 chunks of 16 B); lane takes chunk lane % 8 of rows lane / 8 + 4c
  const int ch = lane & 7, tau0 = lane >> 3;
  const int64_t e0 = (row0 + (int64_t)tau0 * a.H) * kN + ch * 8;  // element offset of (tau0, ch)
  const int64_t estep = (int64_t)4 * a.H * kN;                    // 4 rows further
  const int so = tau0 * 128 + ch * 16;                            // row-major stage offset
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int tau = tau0 + 4 * c;
    const int64_t ge = e0 + c * estep;
    uint8_t *dd = st + a.in.d + so + c * 512;
    uint8_t *db = st + a.in.B + so + c * 512;
    uint8_t *dc = st + a.in.C + so + c * 512;
    if (tau < nvalid) {
      cp_async16(dd, a.d + ge);
      cp_async16(db, a.B + ge);
      cp_async16(dc, a.C + ge);
    } else {
      const uint4 z = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(dd) = z;
      *reinterpret_cast<uint4 *>(db) = z;
      *reinterpret_cast<uint4 *>(dc) = z;
    }
  }
  if (a.row_bytes) {
    // logits rows, or the steps' transition rows (one byte per column j)
    const int lchunks = a.row_bytes / 16;  // 16-byte chunks per row
    const uint8_t *lg = a.steps ? a.steps : static_cast<const uint8_t *>(a.logits);
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

// cp.async of one sub-chunk's x straight into its operand stage (bf16 MN-major,
// mn = p, k = tau: (tau % 8) * 16 + (tau / 8) * 1024 + (p / 8) * 128 + (p % 8) * 2).
__device__ __forceinline__ void load_x(const FParams &a, uint8_t *opx, int64_t b, int64_t h, int sub, int lane) {
  const int t0 = sub * kT;
  const int nvalid = (int)(a.L - t0 < kT ? a.L - t0 : kT);
  const int64_t row0 = (b * a.L + t0) * a.H + h;
  const int ch = lane & 7, tau0 = lane >> 3;
  const int64_t e0 = (row0 + (int64_t)tau0 * a.H) * kP + ch * 8;
  const int64_t estep = (int64_t)4 * a.H * kP;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int tau = tau0 + 4 * c;
    uint8_t *dx = opx + (tau & 7) * 16 + (tau >> 3) * 1024 + ch * 128;
    if (tau < nvalid)
      cp_async16(dx, a.x + e0 + c * estep);
    else
      *reinterpret_cast<uint4 *>(dx) = make_uint4(0, 0, 0, 0);
  }
}


// Hard selection of token lane / 2 of a stage's logits block: the two lanes of
// a token each scan every other 16-byte chunk of its row, then merge.
template <typename TL>
__device__ __forceinline__ int argmax_pair(const uint8_t *rows, int K, int lane) {
  constexpr int kPer = 16 / (int)sizeof(TL);
  const uint8_t *row = rows + (lane >> 1) * K * (int)sizeof(TL);
  float bv = 0.f;
  int bk = INT_MAX;
  for (int c = lane & 1; c * kPer < K; c += 2) {
    const uint4 q = *reinterpret_cast<const uint4 *>(row + c * 16);
    const TL *e = reinterpret_cast<const TL *>(&q);
#pragma unroll
    for (int u = 0; u < kPer; ++u) sel_merge(bv, bk, to_f32(e[u]), c * kPer + u);
  }
  sel_merge(bv, bk, __shfl_xor_sync(0xffffffffu, bv, 1), __shfl_xor_sync(0xffffffffu, bk, 1));
  return bk;
}

// packed fp32 pair arithmetic (one instruction for two lanes of data)
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<uint64_t *>(&a)),
      "l"(*reinterpret_cast<uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&r);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(*reinterpret_cast<uint64_t *>(&a)),
      "l"(*reinterpret_cast<uint64_t *>(&b)), "l"(*reinterpret_cast<uint64_t *>(&c)));
  return *reinterpret_cast<float2 *>(&r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(*reinterpret_cast<uint64_t *>(&a)),
      "l"(*reinterpret_cast<uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&r);
}
// float4 = two float2 halves
__device__ __forceinline__ float4 scale4(float4 v, float s) {
  const float2 ss = make_float2(s, s);
  const float2 lo = mul2(make_float2(v.x, v.y), ss), hi = mul2(make_float2(v.z, v.w), ss);
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ float4 dot2_4(float b0, float4 g0, float b1, float4 g1) {  // b0 g0 + b1 g1
  const float2 s0 = make_float2(b0, b0), s1 = make_float2(b1, b1);
  const float2 lo = fma2(make_float2(g1.x, g1.y), s1, mul2(make_float2(g0.x, g0.y), s0));
  const float2 hi = fma2(make_float2(g1.z, g1.w), s1, mul2(make_float2(g0.z, g0.w), s0));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  const float2 lo = add2(make_float2(a.x, a.y), make_float2(b.x, b.y));
  const float2 hi = add2(make_float2(a.z, a.w), make_float2(b.z, b.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// bf16 pair (as loaded, element 0 in the low half) -> floats
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

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
// (written, not accumulated). G is bf16 for bf16 output and hi + lo otherwise. The region held S_{u+1-R}: this is issued only
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
  if constexpr (kPrecise) mma_bf16(dY, dX, smem_desc(o + kOffGtLo, 128, 256), kIdG, 1);
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
    bars->wait_ns = a.short_waits ? kShortTimeoutNs : kTimeoutNs;
    mbar_fence_init();
  }
  const int32_t *idx_h = a.idx + (a.head_dicts ? h * a.K * kN : 0);
  for (int e = tid; e < (a.steps ? 0 : a.K * kN); e += kThreads) {
    int v = idx_h[e];
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
    // Pair w prepares sub-chunks w, w + kNW, ... (sub-chunk a into operand stage
    // a mod nst). Both of its warps run "walkers": a walker (sigma, j) starts at
    // row j just after step sigma and follows the row through the maps of the
    // steps sigma + 1 ... (the last valid step), carrying the product of the d it
    // passes times B_sigma[j]. On its way it meets C_tau at its current row, which
    // is its part of G[tau][sigma] = C_tau^T A_tau...A_{sigma+1} B_sigma; at the end
    // its row is Psi_sigma(j) and its value the part of Bh_sigma = Psi_sigma B_sigma
    // that lands there. Walkers of sigma = -1 (no B) give Ct_tau = Phi_tau^T C_tau
    // and, at the end, Phi_{T-1}: the carry records. Lanes own rows j and j + 32
    // and walk two sigma at once (four independent walkers per lane).
    //   warp X: S_{a+1}'s order, walks sigma = 0,1 | 4,5 | 8,9 | 12,13
    //   warp Y: S_a's order, the sigma = -1 walk and the records, walks 2,3 | ... | 14,15
    const int pair = warp >> 1, role = warp & 1;
    const uint32_t pbar = 1 + pair;
    uint8_t *in = in_base + pair * a.in.bytes;
    uint8_t *ws = scr + pair * kScrBytes;
    int *sel = reinterpret_cast<int *>(ws + kScrSel);
    uint8_t *posBt = ws + kScrPosB;
    uint8_t *posAt = ws + kScrPosA;
    float *Qt = reinterpret_cast<float *>(ws + (role ? kScrQY : kScrQX));
    int *bins = reinterpret_cast<int *>(ws + (role ? kScrBinsY : kScrBinsX));
    uint8_t *grp = ws + (role ? kScrGrpY : kScrGrpX);
    const int j0 = lane, j1 = lane + 32;
#pragma unroll
    for (int c = 0; c < 4; ++c) bins[lane + 32 * c] = 0;
    for (int sub = pair; sub < nsub; sub += kNW) {
      const int stg = sub % a.nst;
      uint8_t *op = op_base + stg * kOpStage;
      const int t0 = sub * kT;
      const int nvalid = (int)(a.L - t0 < kT ? a.L - t0 : kT);
      const int nnext = (int)(a.L - t0 - kT < kT ? (a.L - t0 - kT > 0 ? a.L - t0 - kT : 0) : kT);
      const int tend = nvalid - 1;  // last valid step of the sub-chunk
      // the inputs load while the operand stage is being released
      if (role == 0) {
        load_inputs(a, in, b, h, sub, lane);
        cp_async_commit();
      }
      const bool ok = wait_bar_warp(bars, &bars->opfree[stg], ((sub / a.nst) & 1) ^ 1, a.err);
      if (role == 0) {
        cp_async_wait<0>();
      } else if (ok) {
        load_x(a, op + kOffX, b, h, sub, lane);
        cp_async_commit();
      }
      // one decision for the pair; the barrier also publishes the loaded inputs. A
      // pair that stops waits for its own copies still in flight first.
      if (!pair_and(pbar, ok)) {
        cp_async_wait<0>();
        break;
      }

      // selections, two lanes per token: warp Y this sub-chunk's, warp X the next one's.
      // With per-step transitions the "dictionary" is the stage's table of the 2T
      // steps' rows and step tau selects row tau (values >= N are replaced by 0).
      if (a.steps) {
        uint4 *rows = reinterpret_cast<uint4 *>(in + a.in.logits + (role == 0 ? kT * kN : 0));
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint4 v = rows[lane + 32 * c];
          if (((v.x | v.y | v.z | v.w) & 0xC0C0C0C0u) != 0) {  // a byte >= 64 = N
            uint8_t *bv = reinterpret_cast<uint8_t *>(&v);
            for (int q = 0; q < 16; ++q)
              if (bv[q] >= kN) bv[q] = 0;
            rows[lane + 32 * c] = v;
            flag_error(a.err, kErrIdxRange);
          }
        }
        if (lane < kT) sel[(role == 0 ? kT : 0) + lane] = (role == 0 ? kT : 0) + lane;
      } else {
        const bool nx = role == 0;
        const int tok = lane >> 1;
        int s_tok = 0;
        if (a.logits) {
          s_tok = argmax_pair<TL>(in + (nx ? a.in.nlogits : a.in.logits), a.K, lane);
        } else if (tok < (nx ? nnext : nvalid)) {
          s_tok = a.s_in[(b * a.L + t0 + (nx ? kT : 0) + tok) * a.H + h];
          if (s_tok < 0 || s_tok >= a.K) {
            flag_error(a.err, kErrSRange);
            s_tok = 0;
          }
        }
        if (tok >= (nx ? nnext : nvalid)) s_tok = 0;
        if ((lane & 1) == 0) {
          sel[(nx ? kT : 0) + tok] = s_tok;
          if (!nx && a.s_out && tok < nvalid) a.s_out[(b * a.L + t0 + tok) * a.H + h] = s_tok;
        }
      }
      pair_sync(pbar);
      const uint8_t *dict_p = a.steps ? in + a.in.logits : dict;  // rows indexed by sel

      const uint8_t *din = in + a.in.d, *Bin = in + a.in.B, *Cin = in + a.in.C;
      // ---- orders of the states: X the next sub-chunk's (S_{a+1}), Y this one's (S_a)
      int phi0 = j0, phi1 = j1;  // warp Y: Phi_{T-1} indices
      {
        int n0 = j0, n1 = j1;
        const int nsteps = role == 0 ? nnext : nvalid;
        const int *ss = sel + (role == 0 ? kT : 0);
        for (int tau = 0; tau < nsteps; ++tau) {
          const uint8_t *dk = dict_p + ss[tau] * kN;
          n0 = dk[n0];
          n1 = dk[n1];
        }
        const int2 pp = group_positions(n0, n1, grp, lane);
        uint8_t *pt = role == 0 ? posBt : posAt;
        pt[j0] = (uint8_t)pp.x;
        pt[j1] = (uint8_t)pp.y;
        phi0 = n0;
        phi1 = n1;
        if (role == 0) {  // G^T above the diagonal stays zero
          reinterpret_cast<uint4 *>(op + kOffGtHi)[lane] = make_uint4(0, 0, 0, 0);
          if constexpr (kPrecise) reinterpret_cast<uint4 *>(op + kOffGtLo)[lane] = make_uint4(0, 0, 0, 0);
        }
      }
      pair_sync(pbar);  // both orders are published

      if (role == 1) {
        // ---- the sigma = -1 walk: Ct_tau at the source's position in S_a's order,
        //      then Phi_{T-1} = (row, value) and the carry records
        const int posA0 = posAt[j0], posA1 = posAt[j1];
        const int o0 = kOffCt + off_ct_pos(posA0), o1 = kOffCt + off_ct_pos(posA1);
        int r0 = j0, r1 = j1;
        float v0 = 1.f, v1 = 1.f;
#pragma unroll 1
        for (int tau = 0; tau <= tend; ++tau) {
          const uint8_t *dk = dict_p + sel[tau] * kN;
          v0 *= ld_bf16(din, tau * kN + r0);
          v1 *= ld_bf16(din, tau * kN + r1);
          r0 = dk[r0];
          r1 = dk[r1];
          const float c0 = v0 * ld_bf16(Cin, tau * kN + r0), c1 = v1 * ld_bf16(Cin, tau * kN + r1);
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
        // records of Phi_{T-1} = (i, v) for the carry step
        const int i0 = phi0, i1 = phi1;
        {
          const int *cnt = reinterpret_cast<const int *>(grp + kScrCnt);
          const int *offs = reinterpret_cast<const int *>(grp + kScrOffs);
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
          const int f0 = offs[i0], f1 = offs[i1];
          const bool keep0 = posA0 != f0, keep1 = posA1 != f1;
          const bool end0 = posA0 == f0 + cnt[i0] - 1, end1 = posA1 == f1 + cnt[i1] - 1;
          // the group that continues across positions 31 | 32 (or -1): its positions
          // below 32 carry ordinal kOrdNone, so that only the upper half's thread
          // writes the group's total (the lower half's part is added by shuffle)
          const int c32 = posA0 == 32 ? (keep0 ? e0 : -1) : (posA1 == 32 ? (keep1 ? e1 : -1) : -2);
          const int ecross = __reduce_max_sync(0xffffffffu, c32);
          const int q0 = (posA0 < 32 && e0 == ecross) ? kOrdNone : e0;
          const int q1 = (posA1 < 32 && e1 == ecross) ? kOrdNone : e1;
          int *meta = reinterpret_cast<int *>(op + kOffMeta);
          meta[posA0] = meta_word(keep0, q0);
          meta[posA1] = meta_word(keep1, q1);
          // the target's column in the next order
          if (end0) op[kOffGDst + e0] = posBt[i0];
          if (end1) op[kOffGDst + e1] = posBt[i1];
          int *hdr = reinterpret_cast<int *>(op + kOffHdr);
          if (lane == 0) {
            hdr[0] = n_img;
            hdr[1] = ecross;
          }
          reinterpret_cast<float *>(op + kOffNu)[posA0] = v0;
          reinterpret_cast<float *>(op + kOffNu)[posA1] = v1;
          reinterpret_cast<int *>(op + kOffSrc)[posA0] = j0;
          reinterpret_cast<int *>(op + kOffSrc)[posA1] = j1;
          reinterpret_cast<int *>(op + kOffPhiIdx)[j0] = i0;
          reinterpret_cast<int *>(op + kOffPhiIdx)[j1] = i1;
          reinterpret_cast<float *>(op + kOffPhiVal)[j0] = v0;
          reinterpret_cast<float *>(op + kOffPhiVal)[j1] = v1;
        }
      }

      // ---- walks of the sigma pairs (sa, sa + 1): warp X takes sa = 0, 4, 6, 8 and
      //      warp Y (which also ran the sigma = -1 walk) sa = 2, 10, 12, 14; a pair
      //      (sa, sa + 1) takes 14 - sa joint steps
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int sa = role ? (m == 0 ? 2 : 8 + 2 * m) : (m == 0 ? 0 : 2 + 2 * m), sb = sa + 1;
        float *q = Qt + lane;  // element (slot, tau) of this lane at q[(slot * kT + tau) * 32]
        // B of both starts at the lane's rows, and G's diagonal terms
        const float ba0 = ld_bf16(Bin, sa * kN + j0), ba1 = ld_bf16(Bin, sa * kN + j1);
        const float bb0 = ld_bf16(Bin, sb * kN + j0), bb1 = ld_bf16(Bin, sb * kN + j1);
        q[sa * 32] = fmaf(ba1, ld_bf16(Cin, sa * kN + j1), ba0 * ld_bf16(Cin, sa * kN + j0));
        q[(kT + sb) * 32] = fmaf(bb1, ld_bf16(Cin, sb * kN + j1), bb0 * ld_bf16(Cin, sb * kN + j0));
        int ra0 = j0, ra1 = j1, rb0 = j0, rb1 = j1;
        float wa0 = ba0, wa1 = ba1, wb0 = bb0, wb1 = bb1;
        if (sb <= tend) {  // walker a's first step (sb): b starts after it
          const uint8_t *dk = dict_p + sel[sb] * kN;
          wa0 *= ld_bf16(din, sb * kN + ra0);
          wa1 *= ld_bf16(din, sb * kN + ra1);
          ra0 = dk[ra0];
          ra1 = dk[ra1];
          q[sb * 32] = fmaf(wa1, ld_bf16(Cin, sb * kN + ra1), wa0 * ld_bf16(Cin, sb * kN + ra0));
        }
#pragma unroll 1
        for (int tau = sb + 1; tau <= tend; ++tau) {
          const uint8_t *dk = dict_p + sel[tau] * kN;
          const uint8_t *dr = din + tau * kN * 2, *cr = Cin + tau * kN * 2;
          wa0 *= ld_bf16(dr, ra0);
          wa1 *= ld_bf16(dr, ra1);
          wb0 *= ld_bf16(dr, rb0);
          wb1 *= ld_bf16(dr, rb1);
          ra0 = dk[ra0];
          ra1 = dk[ra1];
          rb0 = dk[rb0];
          rb1 = dk[rb1];
          q[tau * 32] = fmaf(wa1, ld_bf16(cr, ra1), wa0 * ld_bf16(cr, ra0));
          q[(kT + tau) * 32] = fmaf(wb1, ld_bf16(cr, rb1), wb0 * ld_bf16(cr, rb0));
        }
        // Bh_sa and Bh_sb: the walkers' values summed as exact fixed-point integers
        // (order-independent) at their rows' positions in S_{a+1}'s order
        int *bna = bins, *bnb = bins + kN;
        const unsigned mxa = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fabsf(wa0), fabsf(wa1))));
        const unsigned mxb = __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fabsf(wb0), fabsf(wb1))));
        // |w| < 2^ex; 64 terms of magnitude < 2^24 stay below 2^30
        const int ea = mxa ? 24 - ((int)((mxa >> 23) & 0xff) - 126) : 0;
        const int eb = mxb ? 24 - ((int)((mxb >> 23) & 0xff) - 126) : 0;
        const float upa = exp2i(ea), upb = exp2i(eb);
        atomicAdd(&bna[posBt[ra0]], __float2int_rn(wa0 * upa));
        atomicAdd(&bna[posBt[ra1]], __float2int_rn(wa1 * upa));
        atomicAdd(&bnb[posBt[rb0]], __float2int_rn(wb0 * upb));
        atomicAdd(&bnb[posBt[rb1]], __float2int_rn(wb1 * upb));
        __syncwarp();  // the walks' partial G and the scatter are complete
        {
          // Bh at positions 2 lane and 2 lane + 1 (adjacent in the operand: one
          // packed store per part)
          const float dna = exp2i(-ea), dnb = exp2i(-eb);
          const int2 ia = reinterpret_cast<const int2 *>(bna)[lane], ib = reinterpret_cast<const int2 *>(bnb)[lane];
          reinterpret_cast<int2 *>(bna)[lane] = make_int2(0, 0);
          reinterpret_cast<int2 *>(bnb)[lane] = make_int2(0, 0);
          st_bf16x2_split(op + kOffBhHi, op + kOffBhLo, off_bh(2 * lane, sa), (float)ia.x * dna, (float)ia.y * dna);
          st_bf16x2_split(op + kOffBhHi, op + kOffBhLo, off_bh(2 * lane, sb), (float)ib.x * dnb, (float)ib.y * dnb);
        }
        // G[tau][sigma]: lane (slot, tau) sums its row of the partial tile, reading the
        // eight 16-byte chunks in a lane-rotated order (no bank conflicts)
        {
          const int slot = lane >> 4, tau = lane & 15, sig = sa + slot;
          const float4 *row = reinterpret_cast<const float4 *>(Qt + lane * 32);
          float4 acc = row[lane & 7];
#pragma unroll
          for (int c = 1; c < 8; ++c) acc = add4(acc, row[(lane + c) & 7]);
          const float g = (acc.x + acc.y) + (acc.z + acc.w);
          if (tau >= sig && tau <= tend) {
            if constexpr (kPrecise) {
              st_bf16_split(op + kOffGtHi, op + kOffGtLo, off_gt(tau, sig), g);
            } else {
              *reinterpret_cast<__nv_bfloat16 *>(op + kOffGtHi + off_gt(tau, sig)) = __float2bfloat16_rn(g);
            }
          }
        }
        __syncwarp();  // the tile and the accumulators are free for the next pair
      }
      if (role == 1) cp_async_wait<0>();  // x has landed in the operand stage

      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->full[stg]);
      // both warps are done with the input stage before the next load overwrites it
      pair_sync(pbar);
    }
  } else if (warp < kIssuerWarp) {
    // ============================================ carry state and output (warps 6-9)
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
    // this thread's output column and rows (8 hh + i) of sub-chunk 0; rows are ystep apart
    const int64_t ystep = a.H * kP;
    TO *const ybase = yout + ((b * a.L + 8 * (lane >> 4)) * a.H + h) * kP + 16 * q + (lane & 15);
    int pidx0 = lane, pidx1 = lane + 32;
    float pval0 = 1.f, pval1 = 1.f;
    int done = 0;  // sub-chunks whose carry step completed
    for (int sub = 0; sub < nsub; ++sub) {
      if (!__all_sync(0xffffffffu, ok)) break;
      const int st = sub % a.nst;
      const uint8_t *op = op_base + st * kOpStage;
      const int ys = sub - kYLag;  // the sub-chunk whose output rides on this step
      if (!wait_bar_warp(bars, &bars->ufull[(sub + 1) % kRing], (sub / kRing) & 1, a.err)) break;
      if (!wait_bar_warp(bars, &bars->full[st], (sub / a.nst) & 1, a.err)) break;
      if (ys >= 0 && !wait_bar_warp(bars, &bars->yfull[ys % kNY], (ys / kNY) & 1, a.err)) break;
      tc_fence_after();
      const uint32_t RS = tbase + lanebase + col_state(sub % kRing);
      const uint32_t RU = tbase + lanebase + col_state((sub + 1) % kRing);
      const int4 *meta4 = reinterpret_cast<const int4 *>(op + kOffMeta);
      const float4 *nu4 = reinterpret_cast<const float4 *>(op + kOffNu);
      // running whole-sequence product (the quarter-0 carry warp keeps it; sub-chunks arrive in order)
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
        if (ys >= 0) {
          float yv[8];
          tmem_ld_x2_8<8>(tbase + lanebase + kColY + (ys % kNY) * kT, yv);
          tmem_wait_ld();
          const int tp = ys * kT;
          const int nv = (int)(a.L - tp < kT ? a.L - tp : kT);
          TO *yrow = ybase + (int64_t)tp * ystep;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (8 * hh + i < nv) store_out(yrow + i * ystep, yv[i]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->yfree[ys % kNY]);
        }
        const int *hdr = reinterpret_cast<const int *>(op + kOffHdr);
        const int n_img = hdr[0], ecross = hdr[1];
        // group totals go through this warp's 17 x 16 floats of the stage's Bh area
        // (its MMA completed before ufull was signalled): rows 0-15 for the groups
        // of this pass, row 16 absorbs the stores of every other position
        float *cs = reinterpret_cast<float *>(const_cast<uint8_t *>(op) + kOffBhHi) + q * 17 * 16 + pl;
#pragma unroll 1
        for (int base = 0; base < n_img; base += 16) {
          // running sum over the group's positions, stored at every position into the
          // group's row: the last store of a group, at its end, leaves its total
          float run = 0.f;
#pragma unroll 1
          for (int r = 0; r < 4; ++r) {
            float v[8];
            tmem_ld_x2_8<32>(RS + 8 * r, v);
            const int4 ma = meta4[8 * hh + 2 * r], mb = meta4[8 * hh + 2 * r + 1];
            const float4 na = nu4[8 * hh + 2 * r], nb = nu4[8 * hh + 2 * r + 1];
            const int mt[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
            const float nu[8] = {na.x, na.y, na.z, na.w, nb.x, nb.y, nb.z, nb.w};
            tmem_wait_ld();
            if (base == 0) {  // the store offsets of the first pass are precomputed
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                run = (mt[c] & kMetaKeep) ? run : 0.f;
                run = fmaf(nu[c], v[c], run);
                *reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(cs) + (mt[c] >> kMetaOffShift)) = run;
              }
            } else {
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                run = (mt[c] & kMetaKeep) ? run : 0.f;
                run = fmaf(nu[c], v[c], run);
                const unsigned e = (unsigned)(((mt[c] >> kMetaOrdShift) & 127) - base);
                cs[(e < 16u ? e : 16u) * 16] = run;
              }
            }
          }
          // the group that crosses positions 31 | 32 gets the lower half's part
          const float tail = __shfl_sync(0xffffffffu, run, pl);
          const unsigned ec = (unsigned)(ecross - base);
          __syncwarp();
          if (hh == 1 && ecross >= 0 && ec < 16u) cs[ec * 16] += tail;
          __syncwarp();
          // U at the group ends += group totals
          const int ne = n_img - base < 16 ? n_img - base : 16;
#pragma unroll 1
          for (int e = 0; e < ne; ++e) {
            const uint32_t col = RU + op[kOffGDst + base + e];
            float u;
            tmem_ld1(col, u);
            tmem_wait_ld();
            tmem_st1(col, u + cs[e * 16]);
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
    // outputs of the last kYLag sub-chunks
    for (int ys = nsub - kYLag > 0 ? nsub - kYLag : 0; ys < nsub; ++ys) {
      if (!(__all_sync(0xffffffffu, ok) && done == nsub &&
            wait_bar_warp(bars, &bars->yfull[ys % kNY], (ys / kNY) & 1, a.err)))
        break;
      tc_fence_after();
      float v[16];
      tmem_ld16(tbase + lanebase + kColY + (ys % kNY) * kT, v);
      tmem_wait_ld();
      store_y(ys, v);
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
    // ============================================ MMA issue (warp 10, one thread)
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

namespace {

// Shared-memory plan of one CTA: as many operand stages as fit two CTAs per SM
// (at least one per prep pair). Returns false when even that does not fit.
constexpr int kTwoCtaBytes = 228 * 1024 / 2 - 1024;  // per-CTA share of an SM, less the reserved 1 KB
bool plan_smem(int K, int row_bytes, bool precise, FParams *a, int *bytes) {
  int o = 0;
  a->in.logits = o; o += kT * row_bytes; o = (o + 127) & ~127;
  a->in.nlogits = o; o += kT * row_bytes; o = (o + 127) & ~127;
  a->in.d = o; o += kT * kN * 2;
  a->in.B = o; o += kT * kN * 2;
  a->in.C = o; o += kT * kN * 2;
  a->in.bytes = (o + 127) & ~127;
  for (a->nst = kMaxStages; a->nst >= kNW; --a->nst) {
    int off = 0;
    a->off_op = off; off += a->nst * op_stage_bytes(precise); off = (off + 1023) & ~1023;
    a->off_in = off; off += kNW * a->in.bytes;
    a->off_dict = off; off += (K * kN + 127) & ~127;
    a->off_scr = off; off += kNW * kScrBytes;
    off = (off + 127) & ~127;
    a->off_bar = off; off += (int)sizeof(Bars);
    if (off <= kTwoCtaBytes) {
      *bytes = off;
      return true;
    }
  }
  return false;
}

}  // namespace

bool fused_scan_applies(const pdssm_problem *pb) {
  if (pb->flags & PDSSM_FLAG_REFERENCE_PATH) return false;
  if (pb->chunk != 0 && pb->chunk != kT) return false;
  if (pb->state_t != PDSSM_F32 || pb->N != kN || pb->P != kP) return false;
  if (pb->d_t != PDSSM_BF16 || pb->in_t != PDSSM_BF16) return false;
  const int lsz = pb->logits_t == PDSSM_BF16 ? 2 : 4;
  if ((pb->K * lsz) % 16 != 0) return false;
  FParams a;
  int bytes = 0;
  return plan_smem((int)pb->K, (int)pb->K * lsz, pb->out_t != PDSSM_BF16, &a, &bytes) &&
         plan_smem((int)pb->K, kN, pb->out_t != PDSSM_BF16, &a, &bytes);
}

bool fused_scan_pointers_ok(const ScanArgs &s) {
  if (!s.logits && !s.s && !s.steps) return false;
  if (s.steps && (reinterpret_cast<uintptr_t>(s.steps) & 15) != 0) return false;
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
  a.steps = s.steps;
  a.s_in = (s.logits || s.steps) ? nullptr : s.s;
  a.row_bytes = s.steps ? kN : (s.logits ? a.K * a.logit_size : 0);
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
  a.short_waits = s.short_waits;
  a.head_dicts = s.head_dicts;
  const bool precise = s.out_t != PDSSM_BF16;
  int off = 0;
  if (!plan_smem(a.K, a.row_bytes, precise, &a, &off)) return cudaErrorInvalidConfiguration;

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
