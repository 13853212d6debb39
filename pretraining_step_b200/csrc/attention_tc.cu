// attention_tc.cu -- causal attention forward on the tcgen05 tensor cores.
//
// One CTA per (128-query tile, head, batch row), heaviest tiles first.
// 192 threads in three roles:
//   warp 0      TMA: the Q tile once, then K and V tiles of 128 keys through
//               two-stage rings (128-byte swizzle, zero fill past T);
//   warp 1      TMEM owner and single-thread MMA issue:
//                 S_j = Q K_j^T  -> TMEM S[j % 2]   (M 128, N 128, K 128)
//                 O  += P_j V_j  -> TMEM O          (P from shared memory,
//                                                    V read MN-major)
//               S_{j+1} is issued before O += P_j V_j, so the tensor pipe
//               computes the next scores while the softmax warps work;
//   warps 2..5  softmax: each thread owns one query row.  It reads its row of
//               S from TMEM, applies scale and causal mask, and writes
//               P = exp2(S - m) as bf16 into a K-major shared tile.  The row
//               maximum m is raised only when the block maximum exceeds it by
//               more than 2^8 (the factor then rescales the O row in TMEM);
//               otherwise the stale maximum is kept and P stays below 2^8.
//               At the end: O / l to global memory, lse = (m + log2 l) ln 2.
// All mbarrier waits are bounded; a timeout sets the status word and every
// role drains (in-flight copies and MMAs) before TMEM is released.

#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nc {
namespace {

constexpr int HD = 128;
constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int kThreads = 192;
constexpr int TILE = 128 * 128 * 2;  // one 128 x 128 bf16 tile: two 64-column swizzled boxes
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE;      // 2 stages
constexpr int OFF_V = OFF_K + 2 * TILE;  // 2 stages
constexpr int OFF_P = OFF_V + 2 * TILE;
constexpr int OFF_BAR = OFF_P + TILE;
constexpr int kSmem = OFF_BAR + 256 + 1024;
constexpr uint32_t TM_S0 = 0, TM_O = 256, kTmemCols = 512;
constexpr float kRescaleThreshold = 8.f;  // log2 units

struct FwdArgs {
  int T, nqb;
  float sl2;  // softmax scale * log2(e)
  __nv_bfloat16* o;
  int64_t ldo;
  float* lse;
  int H;
  int* status;
};

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!tc::mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kWaitTimeoutNs) return;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* s_empty = bars + 11; // [2]
  uint64_t* p_full = bars + 13;
  uint64_t* pv_done = bars + 14;
  uint64_t* drained = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = a.nqb - 1 - (int)blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int n = qb + 1;  // causal: key tiles 0..qb (BQ == BKV)

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&k_full[i], 1);
      tc::mbar_init(&k_empty[i], 1);
      tc::mbar_init(&v_full[i], 1);
      tc::mbar_init(&v_empty[i], 1);
      tc::mbar_init(&s_full[i], 1);
      tc::mbar_init(&s_empty[i], 128);
    }
    tc::mbar_init(p_full, 128);
    tc::mbar_init(pv_done, 1);
    tc::mbar_init(drained, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int col0 = h * HD;

  if (warp == 0) {
    if (lane == 0) {
      tc::tma_prefetch_desc(&tq);
      tc::tma_prefetch_desc(&tk);
      tc::tma_prefetch_desc(&tv);
      tc::mbar_arrive_expect_tx(q_full, TILE);
      tc::tma_load_3d(smem + OFF_Q, &tq, q_full, col0, qb * BQ, b);
      tc::tma_load_3d(smem + OFF_Q + TILE / 2, &tq, q_full, col0 + 64, qb * BQ, b);
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!tc::mbar_wait(&k_empty[s], ph ^ 1, abort_flag, a.status)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&k_full[s], TILE);
        tc::tma_load_3d(smem + OFF_K + s * TILE, &tk, &k_full[s], col0, j * BKV, b);
        tc::tma_load_3d(smem + OFF_K + s * TILE + TILE / 2, &tk, &k_full[s], col0 + 64, j * BKV, b);
        ++issued_k;
        if (!tc::mbar_wait(&v_empty[s], ph ^ 1, abort_flag, a.status)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&v_full[s], TILE);
        tc::tma_load_3d(smem + OFF_V + s * TILE, &tv, &v_full[s], col0, j * BKV, b);
        tc::tma_load_3d(smem + OFF_V + s * TILE + TILE / 2, &tv, &v_full[s], col0 + 64, j * BKV, b);
        ++issued_v;
      }
      if (!ok) {
        // Let in-flight copies land before the CTA can exit.
        drain_wait(q_full, 0);
        for (int j = max(0, issued_k - 2); j < issued_k; ++j) drain_wait(&k_full[j & 1], (j >> 1) & 1);
        for (int j = max(0, issued_v - 2); j < issued_v; ++j) drain_wait(&v_full[j & 1], (j >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t q_addr = tc::smem_u32(smem + OFF_Q);
      const uint32_t p_addr = tc::smem_u32(smem + OFF_P);
      bool ok = tc::mbar_wait(q_full, 0, abort_flag, a.status);
      for (int j = 0; j <= n && ok; ++j) {
        if (j < n) {
          const int s = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          if (!tc::mbar_wait(&k_full[s], ph, abort_flag, a.status) ||
              !tc::mbar_wait(&s_empty[s], ph ^ 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t k_addr = tc::smem_u32(smem + OFF_K + s * TILE);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
            tc::umma_bf16_ss(tmem + TM_S0 + s * 128, tc::smem_desc_sw128(q_addr + off, 16, 1024),
                             tc::smem_desc_sw128(k_addr + off, 16, 1024), id_s, kk > 0 ? 1u : 0u);
          }
          tc::umma_commit(&s_full[s]);
          tc::umma_commit(&k_empty[s]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int s = jj & 1;
          const uint32_t ph = (jj >> 1) & 1;
          if (!tc::mbar_wait(&v_full[s], ph, abort_flag, a.status) ||
              !tc::mbar_wait(p_full, jj & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t v_addr = tc::smem_u32(smem + OFF_V + s * TILE);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            const uint32_t poff = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
            tc::umma_bf16_ss(tmem + TM_O, tc::smem_desc_sw128(p_addr + poff, 16, 1024),
                             tc::smem_desc_sw128(v_addr + kk * 2048, TILE / 2, 1024), id_pv,
                             (jj > 0 || kk > 0) ? 1u : 0u);
          }
          tc::umma_commit(pv_done);
          tc::umma_commit(&v_empty[s]);
        }
      }
      tc::umma_commit(drained);
      drain_wait(drained, 0);
    }
  } else {
    const int qw = warp & 3;
    const int row = qw * 32 + lane;
    const int qi = qb * BQ + row;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t p_row = tc::smem_u32(smem + OFF_P) + row * 128;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int s = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      ok = tc::mbar_wait(&s_full[s], ph, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc::tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld_32x32b_x32(lane_base + TM_S0 + s * 128 + c * 32, r[c]);
      tc::tmem_ld_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(&s_empty[s]);
      // Scale, mask, block maximum.
      const int k0 = j * BKV;
      const bool diag = (j == qb);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float x = __uint_as_float(r[c][i]) * a.sl2;
          const int kj = k0 + c * 32 + i;
          if ((diag && kj > qi) || kj >= a.T) x = -INFINITY;
          r[c][i] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      float alpha = 1.f;
      if (mx > m_used + kRescaleThreshold) {
        alpha = exp2f(m_used - mx);  // 0 on the first tile
        m_used = mx;
      }
      const float mu = (m_used == -INFINITY) ? 0.f : m_used;
      l *= alpha;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = exp2f(__uint_as_float(r[c][2 * i]) - mu);
          const float p1 = exp2f(__uint_as_float(r[c][2 * i + 1]) - mu);
          l += p0 + p1;
          pk[c * 16 + i] = pack_bf16x2(p0, p1);
        }
      // The P tile and the O accumulator are free once the previous P V landed.
      if (j >= 1) {
        ok = tc::mbar_wait(pv_done, (j - 1) & 1, abort_flag, a.status);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc::tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tc::tmem_ld_32x32b_x32(lane_base + TM_O + c * 32, o);
            tc::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tc::tmem_st_32x32b_x32(lane_base + TM_O + c * 32, o);
          }
          tc::tmem_st_wait();
        }
      }
      // P row -> K-major swizzled tile: 16-byte unit u of key chunk ch sits at
      // row*128 + ((u ^ (row & 7)) * 16) inside the chunk.
#pragma unroll
      for (int ch = 0; ch < 2; ++ch)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t* q4 = &pk[ch * 32 + u * 4];
          tc::st_shared_v4(p_row + ch * (TILE / 2) + ((u ^ (row & 7)) << 4), q4[0], q4[1], q4[2],
                           q4[3]);
        }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(p_full);
    }
    if (ok) {
      ok = tc::mbar_wait(pv_done, (n - 1) & 1, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = a.o + ((int64_t)b * a.T + qi) * a.ldo + col0;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tc::tmem_ld_32x32b_x32(lane_base + TM_O + c * 32, o);
        tc::tmem_ld_wait();
        if (qi < a.T) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * u + 0]) * inv, __uint_as_float(o[8 * u + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv);
            reinterpret_cast<uint4*>(orow + c * 32)[u] = v;
          }
        }
      }
      if (qi < a.T)
        a.lse[((int64_t)b * a.H + h) * a.T + qi] = (m_used + log2f(l)) * 0.69314718055994531f;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

nc_status attention_fwd(const void* q, const void* k, const void* v, int64_t ld, void* o,
                        int64_t ldo, float* lse, int B, int T, int H, int* status, cudaStream_t s,
                        Profiler* prof) {
  if (B < 1 || T < 1 || H < 1 || !q || !k || !v || !o || !lse)
    return fail(NC_ERR_INVALID_ARG, "attention_fwd: bad arguments");
  if (ld % 8 || ldo % 8 ||
      ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o)) & 15))
    return fail(NC_ERR_INVALID_ARG, "attention_fwd: rows must be 16-byte aligned");
  static bool attr = false;
  if (!attr) {
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmem));
    attr = true;
  }
  CUtensorMap mq, mk, mv;
  const uint64_t cols = (uint64_t)H * HD;
  if (!make_tmap_bf16_3d(&mq, q, cols, T, B, ld, (int64_t)T * ld, 128) ||
      !make_tmap_bf16_3d(&mk, k, cols, T, B, ld, (int64_t)T * ld, 128) ||
      !make_tmap_bf16_3d(&mv, v, cols, T, B, ld, (int64_t)T * ld, 128))
    return fail(NC_ERR_INVALID_ARG, "attention_fwd: cuTensorMapEncodeTiled rejected q/k/v");
  FwdArgs a;
  a.T = T;
  a.nqb = (T + BQ - 1) / BQ;
  a.sl2 = (float)(1.4426950408889634 / std::sqrt((double)HD));
  a.o = static_cast<__nv_bfloat16*>(o);
  a.ldo = ldo;
  a.lse = lse;
  a.H = H;
  a.status = status;
  const double flops = 4.0 * B * H * HD * ((double)T * (T + 1) / 2.0);
  Probe probe(prof, s, "attn_fwd", flops, 0.0);
  dim3 grid(a.nqb, H, B);
  attn_fwd_tc_kernel<<<grid, kThreads, kSmem, s>>>(mq, mk, mv, a);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

}  // namespace nc
