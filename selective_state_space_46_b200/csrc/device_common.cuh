// Device-side helpers shared by the scan and decode kernels (sm_100a).
//
// Transcendentals use the SFU instructions directly (ex2.approx, lg2.approx,
// rcp.approx); softplus and the logistic gate are assembled from them below
// with the error analysis stated next to each.  Packed fp32 pairs use the
// sm_100 f32x2 instructions (one instruction, two fp32 results, round to
// nearest), which halve the issue slots of the state update.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace mssm {

constexpr int kN = 16;                       // state size this library is built for
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;

// ---------------------------------------------------------------- SFU wrappers
__device__ __forceinline__ float ex2f(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float lg2f(float x) {
  float r;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float rcpf(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// softplus(v) = log(1 + e^v).
//  * v > 20: v (the remainder e^-v < 2.1e-9, the threshold PyTorch's softplus uses).
//  * e = e^v < 2^-6: the series e - e^2/2 + e^3/3, whose truncation error is below
//    e^4/4, i.e. relative error < 2^-20; this avoids the cancellation of forming 1 + e.
//  * otherwise log2(1 + e) * ln 2, where 1 + e >= 1 + 2^-6 keeps the relative error
//    of the result near the SFU's 2^-22 absolute log2 error (< 2e-5 relative).
__device__ __forceinline__ float softplus_f(float v) {
  const float e = ex2f(v * kLog2e);
  const float big = lg2f(1.0f + e) * kLn2;
  const float small = e * fmaf(e, fmaf(e, 0.33333333f, -0.5f), 1.0f);
  const float r = (e < 0.015625f) ? small : big;
  return (v > 20.0f) ? v : r;
}

// Zero-order hold ("Linear Attention vs Softmax Attention ...", Core Concepts, item 3;
// "State Space Models in Large Language Models ...", Discretization): the input gain of state n is
// (exp(delta A_n) - 1) / A_n = delta * phi(delta A_n), phi(x) = expm1(x) / x.
// For |x| < 1/16, phi is its Taylor polynomial through x^4/120 (truncation below
// x^5/720 < 1.4e-9 relative), which avoids the cancellation of exp(x) - 1; for
// larger |x|, |exp(x) - 1| >= 0.06, so (e - 1) from the SFU exponential keeps a
// relative error below 4e-6.
__device__ __forceinline__ float expm1_over_x_small(float x) {
  return fmaf(x, fmaf(x, fmaf(x, fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f), 1.0f / 6.0f), 0.5f), 1.0f);
}
// gain = (e - 1) / a with e = exp(dt a) already computed; inv_a = 1 / a (unused when |dt a| < 1/16,
// which covers a = 0, where the gain is dt)
__device__ __forceinline__ float zoh_gain_f(float e, float dt, float a, float inv_a) {
  const float x = dt * a;
  return (fabsf(x) < 0.0625f) ? dt * expm1_over_x_small(x) : (e - 1.0f) * inv_a;
}

// silu(z) = z / (1 + e^-z); e^-z overflowing to +inf gives 0, as it should.
__device__ __forceinline__ float silu_f(float z) {
  return z * rcpf(1.0f + ex2f(-z * kLog2e));
}

// silu(z) = (z/2)(1 + tanh(z/2)) with the SFU tanh (relative error about 2^-11).
// The result's error is at most |z| 2^-12 relative to |silu(z)|'s scale, below
// the rounding of a bf16 output for |z| < 8; used only where the output is bf16.
__device__ __forceinline__ float silu_tanh(float z) {
  const float hz = 0.5f * z;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hz));
  return fmaf(hz, t, hz);
}

// the gate used for an output stored as T: exact for fp32, SFU tanh for bf16
template <typename T>
__device__ __forceinline__ float gate_f(float z) {
  if constexpr (sizeof(T) == 2) {
    return silu_tanh(z);
  } else {
    return silu_f(z);
  }
}

// ---------------------------------------------------------------- bf16 storage
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// round-to-nearest-even conversion of two floats into one bf16x2 word (lo in bits 0..15)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint16_t f_to_bf16(float x) {
  return uint16_t(pack_bf16x2(x, 0.0f) & 0xffffu);
}

// ---------------------------------------------------------------- packed fp32 pairs
typedef unsigned long long f2_t;

__device__ __forceinline__ f2_t f2(float lo, float hi) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2split(f2_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ float f2lo(f2_t v) { float lo, hi; f2split(v, lo, hi); return lo; }
__device__ __forceinline__ float f2hi(f2_t v) { float lo, hi; f2split(v, lo, hi); return hi; }
__device__ __forceinline__ f2_t fma2(f2_t a, f2_t b, f2_t c) {
  f2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2_t add2(f2_t a, f2_t b) {
  f2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t mul2(f2_t a, f2_t b) {
  f2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Storage element traits: bf16 is kept as raw 16-bit patterns.
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPerVec = 4;   // elements per 16-byte vector
  __device__ __forceinline__ static float load(const float* p) { return *p; }
};
template <> struct Elem<uint16_t> {
  static constexpr int kPerVec = 8;
  __device__ __forceinline__ static float load(const uint16_t* p) { return bf16_to_f(*p); }
};

}  // namespace mssm
