// Device helpers shared by the libgdr kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr.h"

namespace gdr {

// ---- element access -----------------------------------------------------------------

template <typename T> struct Elem;

template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
  // four consecutive elements (the address is 4-element aligned)
  static __device__ __forceinline__ float4 load4(const float* p) {
    return *reinterpret_cast<const float4*>(p);
  }
};

template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
  }
  static __device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    uint2 raw = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
    float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
  }
};

// log of a gate in [0, 1], floored so that a zero gate stays finite: the state
// carried across such a token is scaled by e^-30 instead of 0.
__device__ __forceinline__ float log_gate(float a) {
  return fmaxf(__logf(fmaxf(a, 1e-38f)), -GDR_LOG_GATE_FLOOR);
}

// accurate variant for the fp32 kernels
__device__ __forceinline__ float log_gate_accurate(float a) {
  return fmaxf(logf(fmaxf(a, 1e-38f)), -GDR_LOG_GATE_FLOOR);
}

// ---- fused prologue (GDR_PROLOGUE_* flags) --------------------------------------------

// softplus(x) = log(1 + e^x), written so that neither branch overflows
__device__ __forceinline__ float softplus(float x) {
  return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}
// the gate alpha = exp(-softplus(x)) from its pre-activation x
__device__ __forceinline__ float gate_from_logit(float x) { return expf(-softplus(x)); }
// log alpha = -softplus(x), floored like log_gate
__device__ __forceinline__ float log_gate_from_logit(float x) {
  return fmaxf(-softplus(x), -GDR_LOG_GATE_FLOOR);
}
// factor that L2-normalises a vector with this sum of squares
__device__ __forceinline__ float l2_scale(float sumsq) {
  return 1.f / sqrtf(sumsq + GDR_L2NORM_EPS);
}
// a normalised value as the kernel's input type holds it (bf16 inputs: rounded to bf16)
template <typename Tin> __device__ __forceinline__ float as_input(float x);
template <> __device__ __forceinline__ float as_input<float>(float x) { return x; }
template <> __device__ __forceinline__ float as_input<__nv_bfloat16>(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

}  // namespace gdr
