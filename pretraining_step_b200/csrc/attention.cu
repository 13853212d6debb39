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
// D[b, h, t] = sum_d dO[t, h, d] O[t, h, d].  A warp takes one token (all
// heads): every lane's 16-byte loads of both rows are issued before any
// arithmetic, so a warp keeps 2 * H * 256 bytes in flight; half-warps hold
// one head per step.  The block's 32 tokens go through shared memory so the
// [B, H, T] writes are 128-byte runs along t.
constexpr int kDeltaTok = 32;     // tokens per block (8 warps x 4)
constexpr int kDeltaMaxH = 16;    // heads per token handled here
__global__ void __launch_bounds__(256) attn_bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                           const __nv_bfloat16* __restrict__ dout,
                                                           int64_t ldo, float* __restrict__ delta,
                                                           int B, int T, int H) {
  __shared__ float red[kDeltaMaxH][kDeltaTok];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntok = (int64_t)B * T;
  const int64_t tok0 = (int64_t)blockIdx.x * kDeltaTok;
  const int units = H * (HD / 8);  // 16-byte units per row
  for (int k = 0; k < kDeltaTok / 8; ++k) {
    const int lt = warp * (kDeltaTok / 8) + k;
    const int64_t tok = tok0 + lt;
    if (tok >= ntok) break;
    const __nv_bfloat16* orow = o + tok * ldo;
    const __nv_bfloat16* drow = dout + tok * ldo;
    uint4 xs[kDeltaMaxH / 2], ys[kDeltaMaxH / 2];
#pragma unroll
    for (int i = 0; i < kDeltaMaxH / 2; ++i) {
      const int u = lane + 32 * i;
      if (u < units) {
        xs[i] = reinterpret_cast<const uint4*>(orow)[u];
        ys[i] = reinterpret_cast<const uint4*>(drow)[u];
      }
    }
#pragma unroll
    for (int i = 0; i < kDeltaMaxH / 2; ++i) {
      const int u = lane + 32 * i;
      float sum = 0.f;
      if (u < units) {
        const uint32_t* xa = reinterpret_cast<const uint32_t*>(&xs[i]);
        const uint32_t* ya = reinterpret_cast<const uint32_t*>(&ys[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 xv = unpack_bf16x2(xa[e]), yv = unpack_bf16x2(ya[e]);
          sum = fmaf(xv.x, yv.x, fmaf(xv.y, yv.y, sum));
        }
      }
      // lanes [0, 16) hold head 2 i, lanes [16, 32) head 2 i + 1
#pragma unroll
      for (int sh = 8; sh > 0; sh >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, sh);
      const int hh = 2 * i + (lane >> 4);
      if ((lane & 15) == 0 && hh < H) red[hh][lt] = sum;
    }
  }
  __syncthreads();
  // Write [B, H, T]: thread (h, t) for the block's tokens.
  for (int idx = threadIdx.x; idx < H * kDeltaTok; idx += blockDim.x) {
    const int hh = idx / kDeltaTok, lt = idx % kDeltaTok;
    const int64_t tok = tok0 + lt;
    if (tok < ntok) {
      const int64_t bb = tok / T, t = tok % T;
      delta[(bb * H + hh) * T + t] = red[hh][lt];
    }
  }
}

}  // namespace

nc_status attention_bwd_ex(const void* q, int64_t ldq, const void* k, const void* v, int64_t ldkv,
                           const void* o, const void* dout, int64_t ldo, const float* lse,
                           float* dq, void* dk, void* dv, int64_t ldg, float* delta, int B, int T,
                           int H, int Hkv, int window, int* status, cudaStream_t s, Profiler* prof) {
  if (B < 1 || T < 1 || H < 1 || Hkv < 1 || H % Hkv || !q || !k || !v || !o || !dout || !lse ||
      !dq || !dk || !dv || !delta)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: bad arguments (H must be a multiple of Hkv)");
  if (ldq % 8 || ldkv % 8 || ldo % 8 || ldg % 8)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: strides must be multiples of 8");
  if (H > kDeltaMaxH) return fail(NC_ERR_UNSUPPORTED, "attention_bwd: at most 16 heads");
  if ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(dout)) & 15)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: O and dO rows must be 16-byte aligned");
  const int64_t rows = (int64_t)B * T * H;
  {
    Probe probe(prof, s, "attn_bwd_delta", 0.0, rows * HD * 2.0 * 2 + rows * 4.0);
    attn_bwd_delta_kernel<<<(unsigned)(((int64_t)B * T + kDeltaTok - 1) / kDeltaTok), 256, 0, s>>>(
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, ldo, delta, B, T, H);
    NC_CUDA_TRY(cudaGetLastError());
  }
  NC_CUDA_TRY(cudaMemsetAsync(dq, 0, sizeof(float) * rows * HD, s));
  return attention_bwd_tc_ex(q, ldq, k, v, ldkv, dout, ldo, lse, delta, dq, dk, dv, ldg, B, T, H,
                             Hkv, window, nullptr, 0, nullptr, nullptr, 0, status, s, prof);
}

nc_status attention_bwd_model(const void* q, int64_t ldq, const void* k, const void* v,
                              int64_t ldkv, const void* o, const void* dout, int64_t ldo,
                              const float* lse, float* delta, void* ds, int64_t ld_ds,
                              void* dq_out, void* dk, void* dv, int64_t ldg, int B, int T, int H,
                              int Hkv, int window, const float2* rope_tab, int rope_T,
                              const float* rstd_q, const float* rstd_k, int* status, cudaStream_t s,
                              Profiler* prof) {
  if (B < 1 || T < 1 || H < 1 || Hkv < 1 || H % Hkv || H > kDeltaMaxH || !o || !dout || !delta ||
      !ds || !rope_tab || rope_T < T || !rstd_q || !rstd_k)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd_model: bad arguments");
  if (ldo % 8 || ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(dout)) & 15))
    return fail(NC_ERR_INVALID_ARG, "attention_bwd_model: O and dO rows must be 16-byte aligned");
  const int64_t rows = (int64_t)B * T * H;
  {
    Probe probe(prof, s, "attn_bwd_delta", 0.0, rows * HD * 2.0 * 2 + rows * 4.0);
    attn_bwd_delta_kernel<<<(unsigned)(((int64_t)B * T + kDeltaTok - 1) / kDeltaTok), 256, 0, s>>>(
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, ldo, delta, B, T, H);
    NC_CUDA_TRY(cudaGetLastError());
  }
  NC_TRY(attention_bwd_tc_ex(q, ldq, k, v, ldkv, dout, ldo, lse, delta, nullptr, dk, dv, ldg, B, T,
                             H, Hkv, window, rope_tab, rope_T, rstd_k, ds, ld_ds, status, s, prof));
  return attention_dq_ex(ds, ld_ds, k, ldkv, B, T, H, Hkv, window, q, ldq, rstd_q, rope_tab, rope_T,
                         dq_out, ldg, status, s, prof);
}

nc_status attention_bwd(const void* q, const void* k, const void* v, int64_t ld, const void* o,
                        const void* dout, int64_t ldo, const float* lse, float* dq, void* dk,
                        void* dv, int64_t ldg, float* delta, int B, int T, int H, int* status,
                        cudaStream_t s, Profiler* prof) {
  return attention_bwd_ex(q, ld, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, delta, B, T, H, H, -1,
                          status, s, prof);
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
  int* st = nullptr;
  NC_TRY(op_status_word(&st));
  return attention_bwd(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, delta, B, T, H, st,
                       static_cast<cudaStream_t>(stream), nullptr);
}
