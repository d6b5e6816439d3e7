// Device-side helpers shared by the libpdssm kernels (sm_100a).
#pragma once

#include <climits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pdssm.h"

namespace pdssm {

// Bits of the workspace error word (see pdssm_read_device_check).
enum : uint32_t {
  kErrIdxRange = 1u,  // an idx entry outside [0, N)
  kErrSRange = 2u,    // an s entry outside [0, K)
  kErrTimeout = 4u,   // a bounded wait gave up
};

__device__ __forceinline__ void flag_error(uint32_t *err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

// ---------------------------------------------------------------- loads

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ float ldf(const T *p) {
  return to_f32(*p);
}

// (value, k) candidates of one argmax, merged so that the result is the lowest k
// holding the maximum: a NaN beats every number and the lowest NaN wins; +0 and
// -0 tie. k == INT_MAX marks "no candidate yet" (it loses to anything). The merge
// is associative and commutative, so partial winners may be combined in any tree.
__device__ __forceinline__ void sel_merge(float &v, int &k, float ov, int ok) {
  const bool n = v != v, on = ov != ov;
  bool take;
  if (ok == INT_MAX)
    take = false;
  else if (k == INT_MAX)
    take = true;
  else if (n || on)
    take = on && (!n || ok < k);
  else
    take = ov > v || (ov == v && ok < k);
  if (take) {
    v = ov;
    k = ok;
  }
}

// ---------------------------------------------------- real / complex state

// Arithmetic of the state type: float for real state, float2 (re, im) for
// complex state. B, C and x are always real.
template <bool CPLX>
struct Num;

template <>
struct Num<false> {
  using T = float;
  static __device__ __forceinline__ T zero() { return 0.f; }
  static __device__ __forceinline__ T one() { return 1.f; }
  static __device__ __forceinline__ T mul(T a, T b) { return a * b; }
  static __device__ __forceinline__ T fma(T a, T b, T c) { return fmaf(a, b, c); }
  static __device__ __forceinline__ T fma_r(float a, T b, T c) { return fmaf(a, b, c); }  // a real
  static __device__ __forceinline__ T from_real(float a) { return a; }
  static __device__ __forceinline__ T add(T a, T b) { return a + b; }
};

template <>
struct Num<true> {
  using T = float2;
  static __device__ __forceinline__ T zero() { return make_float2(0.f, 0.f); }
  static __device__ __forceinline__ T one() { return make_float2(1.f, 0.f); }
  static __device__ __forceinline__ T mul(T a, T b) {
    return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
  }
  static __device__ __forceinline__ T fma(T a, T b, T c) {
    return make_float2(fmaf(a.x, b.x, fmaf(-a.y, b.y, c.x)), fmaf(a.x, b.y, fmaf(a.y, b.x, c.y)));
  }
  static __device__ __forceinline__ T fma_r(float a, T b, T c) {
    return make_float2(fmaf(a, b.x, c.x), fmaf(a, b.y, c.y));
  }
  static __device__ __forceinline__ T from_real(float a) { return make_float2(a, 0.f); }
  static __device__ __forceinline__ T add(T a, T b) { return make_float2(a.x + b.x, a.y + b.y); }
};

// d as stored (f32, bf16 or complex64) -> state arithmetic type.
template <bool CPLX, typename TD>
struct LoadD;
template <typename TD>
struct LoadD<false, TD> {
  static __device__ __forceinline__ float ld(const TD *p) { return to_f32(*p); }
};
template <>
struct LoadD<true, float2> {
  static __device__ __forceinline__ float2 ld(const float2 *p) { return *p; }
};

// y as stored (f32, bf16 or complex64) from the state arithmetic type.
__device__ __forceinline__ void st_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void st_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void st_out(float2 *p, float2 v) { *p = v; }

// ------------------------------------------------------------- workspace

// Byte layout of the caller's workspace; built on the host, passed by value.
struct Workspace {
  uint32_t *err;        // error word
  int32_t *idx;         // sanitised copy of idx [K][N]
  int32_t *csr_off;     // preimage CSR offsets [K][N+1]
  int32_t *csr_src;     // preimage CSR sources [K][N] (increasing j per row)
  int32_t *s;           // selections when the caller gives no s_out [Bt*L*H]
  void *chunk_state;    // [Bt][H][nC][N][P] state: local end states, then carries
  int32_t *chunk_idx;   // [Bt][H][nC][N] chunk pair indices
  void *chunk_val;      // [Bt][H][nC][N] chunk pair values (state type)
  void *y_loc;          // [Bt][L][H][P] state type: chunk-local outputs
};

}  // namespace pdssm
