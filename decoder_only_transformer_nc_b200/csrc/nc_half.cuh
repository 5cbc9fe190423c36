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

}  // namespace nc
