// 16-bit storage formats of the CUDA path: bf16 or fp16 values held in
// uint16_t buffers, converted to/from fp32 in registers.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace nc {

template <bool F16>
struct Half;

template <>
struct Half<false> {  // bfloat16
  __device__ __forceinline__ static uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static float2 unpack2(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(h);
  }
};

template <>
struct Half<true> {  // IEEE binary16; out-of-range values saturate to +-65504
  __device__ __forceinline__ static uint32_t pack2(float a, float b) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(a), "f"(b));
    return r;
  }
  __device__ __forceinline__ static float2 unpack2(uint32_t u) {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  }
};

// e4m3 (OCP E4M3FN: 4 exponent bits, bias 7, 3 mantissa bits, no infinities)
// for the dynamic tensorwise FP8 path.
constexpr float kE4M3Max = 448.0f;   // largest finite e4m3 value
constexpr float kAmaxFloor = 1e-12f;  // keeps the scale of an all-zero tensor finite

// Tensorwise scale 448 / max(amax, 1e-12), one IEEE fp32 division (a NaN amax
// gives a NaN scale).
__device__ __forceinline__ float e4m3_scale(float amax) {
  return kE4M3Max / (amax < kAmaxFloor ? kAmaxFloor : amax);
}

// Two fp32 values -> two e4m3 codes, round to nearest even, saturating at
// +-448 (NaN -> NaN); a in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(a), "f"(b));
  return r;
}

// Fold a non-negative value's bit pattern into an amax slot (non-negative
// floats order like their bits; NaN orders above every number).  The plain
// read skips the atomic when the slot already holds as much, which is safe
// because the slot only grows.
__device__ __forceinline__ void fold_amax(float* slot, uint32_t bits) {
  if (bits > *reinterpret_cast<volatile uint32_t*>(slot))
    atomicMax(reinterpret_cast<unsigned int*>(slot), bits);
}

// |v| (fp32 bits) of a value about to be stored in a 16-bit format, as the
// bits of its stored value: rounding is monotonic and symmetric, so the
// rounded maximum of |v| is the maximum of the stored |v|.
template <bool F16>
__device__ __forceinline__ uint32_t stored_abs_bits(uint32_t abs_bits) {
  const float v = __uint_as_float(abs_bits);
  return __float_as_uint(Half<F16>::unpack2(Half<F16>::pack2(v, v)).x);
}

}  // namespace nc
