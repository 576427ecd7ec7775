// Device helpers shared by the kernels: element conversion, 16-byte vector
// loads/stores and the RoPE angle (double-precision angle, fp32 rotation).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tpa {

constexpr float kLog2e = 1.4426950408889634f;

template <typename T>
struct Vec16;  // 16 bytes of T
template <>
struct Vec16<float> {
  static constexpr int N = 4;
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load 16 bytes (N elements of T) and widen to fp32.
template <typename T>
__device__ __forceinline__ void load16_f32(const T* __restrict__ p, float* out) {
  uint4 raw = *reinterpret_cast<const uint4*>(p);
  const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
  for (int k = 0; k < Vec16<T>::N; ++k) out[k] = to_f32(e[k]);
}

// Narrow N fp32 values to T and store 16 bytes.
template <typename T>
__device__ __forceinline__ void store16_from_f32(T* __restrict__ p, const float* in) {
  uint4 raw;
  T* e = reinterpret_cast<T*>(&raw);
#pragma unroll
  for (int k = 0; k < Vec16<T>::N; ++k) e[k] = from_f32<T>(in[k]);
  *reinterpret_cast<uint4*>(p) = raw;
}

// cos/sin of pos * theta.  The angle is formed and reduced by 2*pi in double
// precision (positions reach 2^19, where an fp32 angle would be off by
// ~0.03 rad): Cody-Waite with 2*pi split into a 32-bit head, so k * head is
// exact for k < 2^21, and a double tail.  The reduced |r| <= pi is then
// rounded to fp32 (error <= 2^-24 pi ~ 1.9e-7 rad) and evaluated with fp32
// sincosf (within 2 ulp), so the rotation is accurate to ~3e-7 relative: far
// below one bf16 rounding (2^-9) and the fp32 workload's 1e-5 budget, at a
// small fraction of a double-precision sincos.  The reduction is exact up
// to |pos * theta| < 2^21 * 2*pi (1.3e7 rad) and off by less than 1e-15 rad there.
__device__ __forceinline__ void rope_cos_sin(int pos, double theta, float* c, float* s) {
  const double kTwoPiHi = 0x1.921fb544p+2;             // 2*pi rounded to 32 significant bits
  const double kTwoPiLo = 0x1.0b4611a626331p-32;       // 2*pi - kTwoPiHi
  const double kInvTwoPi = 0.15915494309189535;        // 1 / (2*pi)
  const double x = static_cast<double>(pos) * theta;
  const double k = rint(x * kInvTwoPi);
  double r = fma(-k, kTwoPiHi, x);
  r = fma(-k, kTwoPiLo, r);
  sincosf(static_cast<float>(r), s, c);
}

// Rotate the pair (x, y): (x c - y s, x s + y c), in fp32, with the roundings
// spelled out so that every kernel that rotates the same pair gets the same bits.
__device__ __forceinline__ void rope_pair(float& x, float& y, float c, float s) {
  const float xr = __fmaf_rn(x, c, -__fmul_rn(y, s));
  const float yr = __fmaf_rn(x, s, __fmul_rn(y, c));
  x = xr;
  y = yr;
}

}  // namespace tpa
