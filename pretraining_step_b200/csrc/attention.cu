// attention.cu -- causal attention backward driver (head_dim 128): the
// D = rowsum(dO * O) pass, then the tcgen05 backward kernel of
// attention_tc.cu, plus the allocation-free entry point.

#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace nc {
namespace {

constexpr int HD = 128;

// D[b, h, t] = sum_i dO[b, t, h, i] * O[b, t, h, i]; one warp per (token, head).
__global__ void attn_bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                      const __nv_bfloat16* __restrict__ dout, int64_t ldo,
                                      float* __restrict__ delta, int B, int T, int H) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (int64_t)B * T * H) return;
  const int h = (int)(w % H);
  const int64_t tok = w / H;
  const int64_t off = tok * ldo + (int64_t)h * HD + lane * 4;
  const uint2 x = *reinterpret_cast<const uint2*>(o + off);
  const uint2 y = *reinterpret_cast<const uint2*>(dout + off);
  const float2 x0 = unpack_bf16x2(x.x), x1 = unpack_bf16x2(x.y);
  const float2 y0 = unpack_bf16x2(y.x), y1 = unpack_bf16x2(y.y);
  float s = x0.x * y0.x + x0.y * y0.y + x1.x * y1.x + x1.y * y1.y;
  s = warp_sum(s);
  if (lane == 0) {
    const int64_t bb = tok / T, t = tok % T;
    delta[(bb * H + h) * T + t] = s;
  }
}

}  // namespace

nc_status attention_bwd(const void* q, const void* k, const void* v, int64_t ld, const void* o,
                        const void* dout, int64_t ldo, const float* lse, float* dq, void* dk,
                        void* dv, int64_t ldg, float* delta, int B, int T, int H, int* status,
                        cudaStream_t s, Profiler* prof) {
  if (B < 1 || T < 1 || H < 1 || !q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv ||
      !delta)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: bad arguments");
  if (ld % 8 || ldo % 8 || ldg % 8)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: strides must be multiples of 8");
  const int64_t rows = (int64_t)B * T * H;
  {
    Probe probe(prof, s, "attn_bwd_delta", 0.0, rows * HD * 2.0 * 2 + rows * 4.0);
    attn_bwd_delta_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, ldo, delta, B, T, H);
    NC_CUDA_TRY(cudaGetLastError());
  }
  NC_CUDA_TRY(cudaMemsetAsync(dq, 0, sizeof(float) * rows * HD, s));
  return attention_bwd_tc(q, k, v, ld, dout, ldo, lse, delta, dq, dk, dv, ldg, B, T, H, status, s,
                          prof);
}

// ------------------------------------------------------------------ allocation-free backward
// Scratch for the row sums D = rowsum(dO * O) of nc_op_attention_bwd_noalloc:
// a fixed array in the library's device image, so that entry point needs no
// allocation.  Every device that loads the library holds these 4 MiB until
// the process exits.
namespace {
constexpr int64_t kNoAllocDeltaMax = int64_t(1) << 20;  // floats: B * H * T limit
static __device__ __align__(256) float g_attn_delta_scratch[kNoAllocDeltaMax];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  In host code the array's name only stands in for the symbol;
// cudaGetSymbolAddress turns it into the address kernels may use.
nc_status noalloc_scratch(float** out) {
  int dev = 0;
  NC_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(NC_ERR_UNSUPPORTED, "device index too large");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_attn_delta_scratch);
    if (e != cudaSuccess || !ptr) return cuda_fail(e, "cudaGetSymbolAddress(attention scratch)");
    g_scratch_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return NC_OK;
}
}  // namespace

}  // namespace nc

extern "C" nc_status nc_op_attention_bwd_noalloc(const void* q, const void* k, const void* v,
                                                 int64_t ld, const void* o, const void* dout,
                                                 int64_t ldo, const float* lse, float* dq,
                                                 void* dk, void* dv, int64_t ldg, int B, int T,
                                                 int H, void* stream) {
  using namespace nc;
  if (B < 1 || T < 1 || H < 1)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd_noalloc: B, T and H must be positive");
  if ((int64_t)B * H * T > kNoAllocDeltaMax)
    return fail(NC_ERR_INVALID_ARG,
                "attention_bwd_noalloc: B*H*T = " + std::to_string((int64_t)B * H * T) +
                    " exceeds the built-in scratch of " + std::to_string(kNoAllocDeltaMax) +
                    " rows; use nc_op_attention_bwd with a caller-provided buffer");
  float* delta = nullptr;
  NC_TRY(noalloc_scratch(&delta));
  // The row-sum pass rewrites every entry it reads, so nothing from an
  // earlier call leaks into this one and no clearing is needed.
  return attention_bwd(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, delta, B, T, H, nullptr,
                       static_cast<cudaStream_t>(stream), nullptr);
}
