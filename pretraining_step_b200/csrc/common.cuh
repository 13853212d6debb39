// common.cuh -- shared device/host helpers of the sm_100a step library.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nc.h"

namespace nc {

// Device status word values (written by kernels, read by the host).
enum : int {
  kDevOk = 0,
  kDevTimeout = 1,    // a bounded mbarrier wait expired
  kDevTokenRange = 2  // a token / target id outside [0, vocab)
};

// RMSNorm epsilon of every norm in the model (pre-norms and QK-norm).
constexpr float kNormEps = 1e-6f;

// Wall-clock limit of one mbarrier wait (ns).  A correct kernel never waits
// more than microseconds on one barrier.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ __nv_bfloat16 f2bf(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}

// Square root by the PTX approximate instruction (relative error about
// 2^-23, sqrt(0) = 0): one instruction where sqrtf's IEEE rounding takes a
// branchy sequence.  Used where the result is rounded to bf16 anyway.
__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace nc
