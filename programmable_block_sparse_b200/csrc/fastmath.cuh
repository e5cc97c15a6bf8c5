// Arithmetic helpers for the softmax of the sm_100a kernels: packed f32x2
// operations (two fp32 lanes per instruction), three-input maximum, tree
// reductions, and tanh on the FMA pipe for small arguments.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// ---------------------------------------------------------------------------
// f32x2: IEEE fp32 arithmetic on a register pair per instruction
// (add / mul / fma .f32x2, sm_100a).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t pk2(float2 a) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
  return r;
}
__device__ __forceinline__ float2 up2(uint64_t r) {
  float2 a;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a.x), "=f"(a.y) : "l"(r));
  return a;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(pk2(a)), "l"(pk2(b)), "l"(pk2(c)));
  return up2(r);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk2(a)), "l"(pk2(b)));
  return up2(r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk2(a)), "l"(pk2(b)));
  return up2(r);
}
__device__ __forceinline__ float2 splat2(float x) { return make_float2(x, x); }

// max(a, b, c) in one instruction.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of 64 values as a tree of three-input maxima (depth 4, 32
// instructions) rather than a 64-long dependent chain.
__device__ __forceinline__ float max64(const float (&t)[64]) {
  float a[22];
#pragma unroll
  for (int i = 0; i < 21; ++i) a[i] = max3f(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
  a[21] = t[63];
  float b[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) b[i] = max3f(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
  b[7] = a[21];
  return max3f(max3f(b[0], b[1], b[2]), max3f(b[3], b[4], b[5]), fmaxf(b[6], b[7]));
}

// Sum of 64 values as a tree of paired adds (31 f32x2 adds and one add).
__device__ __forceinline__ float sum64(const float (&t)[64]) {
  float2 s[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) s[i] = add2(make_float2(t[4 * i], t[4 * i + 1]), make_float2(t[4 * i + 2], t[4 * i + 3]));
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) s[i] = add2(s[i], s[i + w]);
  return s[0].x + s[0].y;
}

// ---------------------------------------------------------------------------
// tanh(y) for |y| <= kTanhPolyMax on the FMA pipe: the odd Maclaurin series
// tanh y = y - y^3/3 + 2 y^5/15 - 17 y^7/315 + 62 y^9/2835 - ...
// (coefficients from the Bernoulli numbers, 2^2n (2^2n - 1) B_2n / (2n)!)
// truncated after y^7.  The series alternates with shrinking terms for
// |y| < pi/2, so the error is below the first omitted term,
// 62/2835 |y|^9 <= 4.3e-7 at |y| = 0.3 (a relative error below 1.5e-6);
// callers fall back to the hardware tanh for larger arguments.
// ---------------------------------------------------------------------------
constexpr float kTanhPolyMax = 0.3f;
constexpr float kTanhC3 = -1.0f / 3.0f;
constexpr float kTanhC5 = 2.0f / 15.0f;
constexpr float kTanhC7 = -17.0f / 315.0f;

// tanh of a pair; also returns y^2 of the pair so the caller can check the
// range: the result holds where y^2 <= kTanhPolyMax^2.
__device__ __forceinline__ float2 tanh_poly2(float2 y, float2& u) {
  u = mul2(y, y);
  float2 p = fma2(u, splat2(kTanhC7), splat2(kTanhC5));
  p = fma2(u, p, splat2(kTanhC3));
  const float2 w = mul2(y, u);
  return fma2(w, p, y);
}

}  // namespace fa
