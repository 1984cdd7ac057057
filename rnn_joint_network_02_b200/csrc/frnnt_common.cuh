// Shared device helpers of the frnnt library (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "frnnt.h"

namespace frnnt {

__host__ __device__ inline int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Lengths as every kernel sees them: clamped into range so that invalid
// inputs (already flagged in the status word by the validation kernel) can
// never turn into out-of-bounds accesses.
struct Lengths {
  int Tb, Ub;
};
__device__ inline Lengths lengths_of(const int32_t* T_len, const int32_t* U_len, int b, int T, int U) {
  Lengths l;
  l.Tb = clampi(T_len[b], 1, T);
  l.Ub = clampi(U_len[b], 0, U);
  return l;
}
// Status bits found by one thread of a block that checks the lengths and
// labels (strided by nthreads): FRNNT_STATUS_LENGTH for T_len outside [1,T] or
// U_len outside [0,U], FRNNT_STATUS_LABEL for a label (u < U_len) outside
// [0,V) or equal to blank.
__device__ inline int validate_bits(int B, int T, int U, int V, int blank, const int32_t* labels,
                                    const int32_t* T_len, const int32_t* U_len, int tid, int nthreads) {
  int bits = 0;
  for (int b = tid; b < B; b += nthreads) {
    const int tl = T_len[b], ul = U_len[b];
    if (tl < 1 || tl > T || ul < 0 || ul > U) bits |= FRNNT_STATUS_LENGTH;
  }
  const long long n = (long long)B * U;
  for (long long i = tid; i < n; i += nthreads) {
    const int b = (int)(i / U), u = (int)(i % U);
    const int tl = T_len[b], ul = U_len[b];
    if (tl < 1 || tl > T || ul < 0 || ul > U) continue;   // length already flagged
    if (u >= ul) continue;                                // padding label
    const int y = labels[i];
    if (y < 0 || y >= V || y == blank) bits |= FRNNT_STATUS_LABEL;
  }
  return bits;
}
__device__ inline int label_of(const int32_t* labels, int b, int u, int U, int V) {
  return clampi(labels[(size_t)b * U + u], 0, V - 1);
}

// log(exp(a) + exp(b)) in fp32, exact for -inf operands: max + ln(1 + e^-|a-b|),
// with the 1 + e^-d in [1, 2] taken by the hardware exp2 / log2 (absolute error
// of the correction term ~1e-7, far below fp32 rounding of the running sums).
// Both -inf: the correction is NaN and the select returns -inf.  A select, not
// a branch, so that independent calls interleave (a branch per call serialises them).
__device__ __forceinline__ float log_add_exp(float a, float b) {
  const float m = fmaxf(a, b);
  const float r = m + __logf(1.f + __expf(-fabsf(a - b)));
  return m == -INFINITY ? m : r;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

}  // namespace frnnt
