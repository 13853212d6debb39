// attention.cu -- causal softmax attention backward, head_dim 128 (the
// forward is in attention_tc.cu).
//
// Backward: one CTA (8 warps) per 64-key block; loops over the query blocks
// at or after it.  Recomputes P^T = exp(S^T - lse) from the saved lse,
//   dV += P^T dO,  dP^T = V dO^T,  dS^T = P^T (dP^T - D),  dK += dS^T Q,
//   dQ += dS K  (fp32 atomics into a dense accumulator),
// with D = rowsum(dO * O) from a separate pass.  Scale 1/sqrt(128) is folded
// into S, dK and dQ.

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace nc {
namespace {

constexpr int HD = 128;
constexpr int BQ = 64;
constexpr int BKV = 64;
constexpr int LDS = HD + 8;      // padded smem row (elements): 272 B, conflict-free ldmatrix
constexpr int LDP = BQ + 8;      // padded row of the P^T / dS^T tiles
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t s_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // zero-fill rows past the end
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s_u32(dst)), "l"(src),
               "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Copy a 64 x 128 bf16 tile (rows r0.., stride ld elements) into padded smem;
// rows >= T are zero-filled.  `nthr` threads cooperate.
template <int NTHR>
__device__ __forceinline__ void load_tile(__nv_bfloat16* s, const __nv_bfloat16* g, int64_t ld,
                                          int r0, int T) {
  for (int i = threadIdx.x; i < 64 * 16; i += NTHR) {
    const int r = i >> 4, c = (i & 15) * 8;
    const bool ok = (r0 + r) < T;
    const __nv_bfloat16* src = g + (int64_t)(ok ? r0 + r : 0) * ld + c;
    cp_async16(s + r * LDS + c, src, ok);
  }
}

// ------------------------------------------------------------------ backward
// D[b, h, t] = sum_i dO[b, t, h, i] * O[b, t, h, i]; one warp per (token, head).
__global__ void attn_bwd_delta_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                                      int64_t ldo, float* __restrict__ delta, int B, int T, int H) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (int64_t)B * T * H) return;
  const int h = (int)(w % H);
  const int64_t tok = w / H;
  const int64_t off = tok * ldo + (int64_t)h * HD + lane * 4;
  const uint2 a = *reinterpret_cast<const uint2*>(o + off);
  const uint2 c = *reinterpret_cast<const uint2*>(dout + off);
  const float2 a0 = unpack_bf16x2(a.x), a1 = unpack_bf16x2(a.y);
  const float2 c0 = unpack_bf16x2(c.x), c1 = unpack_bf16x2(c.y);
  float s = a0.x * c0.x + a0.y * c0.y + a1.x * c1.x + a1.y * c1.y;
  s = warp_sum(s);
  if (lane == 0) {
    const int64_t bb = tok / T, t = tok % T;
    delta[(bb * H + h) * T + t] = s;
  }
}

__global__ void __launch_bounds__(256) attn_bwd_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, int64_t ld, const __nv_bfloat16* __restrict__ dout,
    int64_t ldo, const float* __restrict__ lse, const float* __restrict__ delta,
    float* __restrict__ dq, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
    int64_t ldg, int T, int H) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sV = sK + 64 * LDS;
  __nv_bfloat16* sQ = sV + 64 * LDS;
  __nv_bfloat16* sdO = sQ + 64 * LDS;
  __nv_bfloat16* sPt = sdO + 64 * LDS;   // [64 keys][LDP]
  __nv_bfloat16* sdSt = sPt + 64 * LDP;  // [64 keys][LDP]
  float* sL = reinterpret_cast<float*>(sdSt + 64 * LDP);
  float* sD = sL + 64;

  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int wm = warp & 3, wn = warp >> 2;
  const int nqb = (T + BQ - 1) / BQ;
  const int k0 = kb * BKV;

  const int64_t base = (int64_t)b * T * ld + (int64_t)h * HD;
  const int64_t obase = (int64_t)b * T * ldo + (int64_t)h * HD;
  load_tile<256>(sK, k + base, ld, k0, T);
  load_tile<256>(sV, v + base, ld, k0, T);
  cp_commit();

  float dka[8][4], dva[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dka[i][e] = dva[i][e] = 0.f;

  const float scale = rsqrtf((float)HD);
  const float sl2 = kLog2e * scale;
  const float* lg = lse + ((int64_t)b * H + h) * T;
  const float* dg = delta + ((int64_t)b * H + h) * T;

  for (int qb = kb; qb < nqb; ++qb) {
    const int q0 = qb * BQ;
    load_tile<256>(sQ, q + base, ld, q0, T);
    load_tile<256>(sdO, dout + obase, ldo, q0, T);
    cp_commit();
    if (threadIdx.x < 64) {
      const int qi = q0 + threadIdx.x;
      sL[threadIdx.x] = qi < T ? lg[qi] * kLog2e : INFINITY;
      sD[threadIdx.x] = qi < T ? dg[qi] : 0.f;
    }
    cp_wait<0>();
    __syncthreads();

    // Phase 1: S^T and dP^T for keys wm*16.., queries wn*32..
    {
      float st[4][4], dpt[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[i][e] = dpt[i][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t ka[4], va[4];
        ldsm_x4(ka, s_u32(sK + (wm * 16 + (lane & 15)) * LDS + ks * 16 + (lane >> 4) * 8));
        ldsm_x4(va, s_u32(sV + (wm * 16 + (lane & 15)) * LDS + ks * 16 + (lane >> 4) * 8));
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          const int j = lane >> 3;
          const int qr = wn * 32 + (np * 2 + (j >> 1)) * 8 + (lane & 7);
          uint32_t bq[4], bo[4];
          ldsm_x4(bq, s_u32(sQ + qr * LDS + ks * 16 + (j & 1) * 8));
          ldsm_x4(bo, s_u32(sdO + qr * LDS + ks * 16 + (j & 1) * 8));
          mma16816(st[2 * np], ka, bq[0], bq[1]);
          mma16816(st[2 * np + 1], ka, bq[2], bq[3]);
          mma16816(dpt[2 * np], va, bo[0], bo[1]);
          mma16816(dpt[2 * np + 1], va, bo[2], bo[3]);
        }
      }
      const int kr0 = wm * 16 + g, kr1 = kr0 + 8;  // key rows within the block
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
        const int qc = wn * 32 + nb * 8 + 2 * t4;  // query column within the block
        float p[4], ds[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kr = (e < 2) ? kr0 : kr1;
          const int qcol = qc + (e & 1);
          const int kj = k0 + kr, qi = q0 + qcol;
          float pv = exp2f(st[nb][e] * sl2 - sL[qcol]);
          if (kj > qi || qi >= T || kj >= T) pv = 0.f;
          p[e] = pv;
          ds[e] = pv * (dpt[nb][e] - sD[qcol]);
        }
        *reinterpret_cast<uint32_t*>(sPt + kr0 * LDP + qc) = pack_bf16x2(p[0], p[1]);
        *reinterpret_cast<uint32_t*>(sPt + kr1 * LDP + qc) = pack_bf16x2(p[2], p[3]);
        *reinterpret_cast<uint32_t*>(sdSt + kr0 * LDP + qc) = pack_bf16x2(ds[0], ds[1]);
        *reinterpret_cast<uint32_t*>(sdSt + kr1 * LDP + qc) = pack_bf16x2(ds[2], ds[3]);
      }
    }
    __syncthreads();

    // Phase 2: dV += P^T dO, dK += dS^T Q for keys wm*16.., dims wn*64..
#pragma unroll
    for (int kq = 0; kq < 4; ++kq) {
      uint32_t pa[4], sa[4];
      ldsm_x4(pa, s_u32(sPt + (wm * 16 + (lane & 15)) * LDP + kq * 16 + (lane >> 4) * 8));
      ldsm_x4(sa, s_u32(sdSt + (wm * 16 + (lane & 15)) * LDP + kq * 16 + (lane >> 4) * 8));
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int j = lane >> 3;
        const int row = kq * 16 + (j & 1) * 8 + (lane & 7);
        const int col = wn * 64 + (np * 2 + (j >> 1)) * 8;
        uint32_t bo[4], bq[4];
        ldsm_x4_t(bo, s_u32(sdO + row * LDS + col));
        ldsm_x4_t(bq, s_u32(sQ + row * LDS + col));
        mma16816(dva[2 * np], pa, bo[0], bo[1]);
        mma16816(dva[2 * np + 1], pa, bo[2], bo[3]);
        mma16816(dka[2 * np], sa, bq[0], bq[1]);
        mma16816(dka[2 * np + 1], sa, bq[2], bq[3]);
      }
    }

    // Phase 3: dQ(rows wm*16.., dims wn*64..) = scale * dS K, atomically.
    {
      float dqa[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) dqa[i][0] = dqa[i][1] = dqa[i][2] = dqa[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        const int j = lane >> 3;
        // A = dS [query][key] read transposed from dS^T [key][query].
        ldsm_x4_t(a, s_u32(sdSt + (kk * 16 + (j >> 1) * 8 + (lane & 7)) * LDP + wm * 16 + (j & 1) * 8));
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          const int row = kk * 16 + (j & 1) * 8 + (lane & 7);
          const int col = wn * 64 + (np * 2 + (j >> 1)) * 8;
          uint32_t bk[4];
          ldsm_x4_t(bk, s_u32(sK + row * LDS + col));
          mma16816(dqa[2 * np], a, bk[0], bk[1]);
          mma16816(dqa[2 * np + 1], a, bk[2], bk[3]);
        }
      }
      const int qi0 = q0 + wm * 16 + g, qi1 = qi0 + 8;
      float* dqg = dq + ((int64_t)b * T) * ((int64_t)H * HD) + (int64_t)h * HD;
#pragma unroll
      for (int nd = 0; nd < 8; ++nd) {
        const int c = wn * 64 + nd * 8 + 2 * t4;
        if (qi0 < T) {
          atomicAdd(dqg + (int64_t)qi0 * H * HD + c, dqa[nd][0] * scale);
          atomicAdd(dqg + (int64_t)qi0 * H * HD + c + 1, dqa[nd][1] * scale);
        }
        if (qi1 < T) {
          atomicAdd(dqg + (int64_t)qi1 * H * HD + c, dqa[nd][2] * scale);
          atomicAdd(dqg + (int64_t)qi1 * H * HD + c + 1, dqa[nd][3] * scale);
        }
      }
    }
    __syncthreads();
  }

  // dK, dV for keys wm*16 + g (+8), dims wn*64 + nd*8 + 2*t4.
  const int64_t gbase = (int64_t)b * T * ldg + (int64_t)h * HD;
  const int kr0 = k0 + wm * 16 + g, kr1 = kr0 + 8;
#pragma unroll
  for (int nd = 0; nd < 8; ++nd) {
    const int c = wn * 64 + nd * 8 + 2 * t4;
    if (kr0 < T) {
      *reinterpret_cast<uint32_t*>(dk + gbase + (int64_t)kr0 * ldg + c) =
          pack_bf16x2(dka[nd][0] * scale, dka[nd][1] * scale);
      *reinterpret_cast<uint32_t*>(dv + gbase + (int64_t)kr0 * ldg + c) =
          pack_bf16x2(dva[nd][0], dva[nd][1]);
    }
    if (kr1 < T) {
      *reinterpret_cast<uint32_t*>(dk + gbase + (int64_t)kr1 * ldg + c) =
          pack_bf16x2(dka[nd][2] * scale, dka[nd][3] * scale);
      *reinterpret_cast<uint32_t*>(dv + gbase + (int64_t)kr1 * ldg + c) =
          pack_bf16x2(dva[nd][2], dva[nd][3]);
    }
  }
}

constexpr int kBwdSmem = 4 * 64 * LDS * 2 + 2 * 64 * LDP * 2 + 2 * 64 * 4;

}  // namespace

nc_status attention_bwd(const void* q, const void* k, const void* v, int64_t ld, const void* o,
                        const void* dout, int64_t ldo, const float* lse, float* dq, void* dk,
                        void* dv, int64_t ldg, float* delta, int B, int T, int H, cudaStream_t s,
                        Profiler* prof) {
  if (B < 1 || T < 1 || H < 1 || !q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv ||
      !delta)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: bad arguments");
  if (ld % 8 || ldo % 8 || ldg % 2)
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: bad strides");
  static bool attr = false;
  if (!attr) {
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem));
    attr = true;
  }
  const int64_t rows = (int64_t)B * T * H;
  {
    Probe probe(prof, s, "attn_bwd_delta", 0.0, rows * HD * 2.0 * 2 + rows * 4.0);
    attn_bwd_delta_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)dout, ldo, delta, B, T, H);
    NC_CUDA_TRY(cudaGetLastError());
  }
  NC_CUDA_TRY(cudaMemsetAsync(dq, 0, sizeof(float) * rows * HD, s));
  const double flops = 10.0 * B * H * HD * ((double)T * (T + 1) / 2.0);  // 5 causal products
  Probe probe(prof, s, "attn_bwd", flops, 0.0);
  dim3 grid((T + BKV - 1) / BKV, H, B);
  attn_bwd_kernel<<<grid, 256, kBwdSmem, s>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, ld,
      (const __nv_bfloat16*)dout, ldo, lse, delta, dq, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, ldg,
      T, H);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
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
  return attention_bwd(q, k, v, ld, o, dout, ldo, lse, dq, dk, dv, ldg, delta, B, T, H,
                       static_cast<cudaStream_t>(stream), nullptr);
}
