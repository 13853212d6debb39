// attention_tc.cu -- causal attention forward and backward on the tcgen05
// tensor cores.
//
// Forward: one CTA per (128-query tile, head, batch row), heaviest tiles
// first, two CTAs per SM.  320 threads in three roles:
//   warp 0      TMA: the Q tile once, then K and V tiles of 128 keys
//               (128-byte swizzle, zero fill past T), one buffer each;
//   warp 1      TMEM owner and single-thread MMA issue, per key tile j:
//                 S  = Q K_j^T  -> TMEM [0, 128)     (M 128, N 128, K 128)
//                 O += P_j V_j  -> TMEM [128, 256)   (A = P_j from TMEM,
//                                                     V read MN-major)
//               All operands keep N = 128: with A and B both in shared
//               memory a 64-wide N is bound by shared-memory bandwidth;
//               P never touches shared memory at all;
//   warps 2..9  softmax, two threads per query row (warps 2..5 keys
//               [0, 64) of each tile, warps 6..9 keys [64, 128)).  Each
//               reads its 64 scores once, the pair agrees on the block
//               maximum through shared memory, and each writes its
//               P = exp2(S - m) as bf16 over its own first scores.  The row
//               maximum m is raised only when the block maximum exceeds it
//               by more than 2^8 (the factor then rescales the O row in
//               TMEM); otherwise the stale maximum is kept and P stays below
//               2^8.  At the end: O / l to global memory,
//               lse = (m + log2 l) ln 2.
// The MMAs of a CTA run in issue order, so S_{j+1} (issued after P_j V_j)
// never overwrites P_j early, and the commit that publishes S_j also
// guarantees P_{j-1} V_{j-1} has finished with P_{j-1} and with O.  The other
// CTA on the SM keeps the tensor pipe busy while this one's softmax runs.
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
constexpr int BKV = 128;  // key tile (forward and backward)
constexpr int kThreads = 320;  // forward: TMA warp, MMA warp, 8 softmax warps
constexpr int TILE = 128 * 128 * 2;  // one 128 x 128 bf16 tile: two 64-column swizzled boxes
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE;
constexpr int OFF_V = OFF_K + TILE;
constexpr int OFF_BAR = OFF_V + TILE;
// 96 KB + barriers: two CTAs and their 1 KB system reservations fit the SM's
// 228 KB.  The dynamic window starts 1024-byte aligned; the kernel checks
// that before using it (no slack is reserved to realign).
constexpr int OFF_X = OFF_BAR + 256;   // [2 tiles][2 halves][128 rows] partial row maxima
constexpr int OFF_L = OFF_X + 2048;    // [2 halves][128 rows] partial row sums
constexpr int kSmem = OFF_L + 1024;
constexpr uint32_t TM_S = 0, TM_O = 128, kFwdTmemCols = 256;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.f;  // log2 units

struct FwdArgs {
  int T, nqb;
  float sl2;  // softmax scale * log2(e)
  __nv_bfloat16* o;
  int64_t ldo;
  float* lse;
  int H;
  int group;   // query heads per KV head (1: one KV head per query head)
  int window;  // query t sees keys [t - window, t]; < 0: every key up to t
  int* status;
};

// 2^x by the MUFU instruction (ex2.approx, flush-to-zero): the softmax
// arguments are <= 0 (or <= 8 with a stale maximum), far from its range limits.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!tc::mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kWaitTimeoutNs) return;
}

// GW: grouped KV heads or a window in play; the plain instance (every query
// head its own KV head, no window) compiles with those as constants.
template <bool GW>
__global__ void __launch_bounds__(kThreads, 2)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const FwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((tc::smem_u32(smem_raw) & 1023u) != 0) {  // never expected; no room to realign
    if (threadIdx.x == 0 && a.status) atomicExch(a.status, kDevTimeout);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 2;
  uint64_t* v_full = bars + 3;
  uint64_t* v_empty = bars + 4;
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* o_full = bars + 7;
  uint64_t* drained = bars + 8;
  uint64_t* mx_ready = bars + 9;
  uint64_t* l_ready = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = a.nqb - 1 - (int)blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int group = GW ? a.group : 1;
  const int window = GW ? a.window : -1;
  // Key tiles from the first one the window reaches to the diagonal (BKV == BQ).
  const int lo_key = window < 0 ? 0 : qb * BQ - window;
  const int j_lo = lo_key <= 0 ? 0 : lo_key / BKV;
  const int n = qb - j_lo + 1;

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    tc::mbar_init(k_full, 1);
    tc::mbar_init(k_empty, 1);
    tc::mbar_init(v_full, 1);
    tc::mbar_init(v_empty, 1);
    tc::mbar_init(s_full, 1);
    tc::mbar_init(p_full, 256);
    tc::mbar_init(o_full, 1);
    tc::mbar_init(drained, 1);
    tc::mbar_init(mx_ready, 256);
    tc::mbar_init(l_ready, 256);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kFwdTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int col0 = h * HD;
  const int kcol0 = (h / group) * HD;  // this query head's KV head

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
        const uint32_t ph = j & 1;
        if (!tc::mbar_wait(k_empty, ph ^ 1, abort_flag, a.status)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(k_full, TILE);
        tc::tma_load_3d(smem + OFF_K, &tk, k_full, kcol0, (j_lo + j) * BKV, b);
        tc::tma_load_3d(smem + OFF_K + TILE / 2, &tk, k_full, kcol0 + 64, (j_lo + j) * BKV, b);
        ++issued_k;
        if (!tc::mbar_wait(v_empty, ph ^ 1, abort_flag, a.status)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(v_full, TILE);
        tc::tma_load_3d(smem + OFF_V, &tv, v_full, kcol0, (j_lo + j) * BKV, b);
        tc::tma_load_3d(smem + OFF_V + TILE / 2, &tv, v_full, kcol0 + 64, (j_lo + j) * BKV, b);
        ++issued_v;
      }
      if (!ok) {
        // Let in-flight copies land before the CTA can exit.
        drain_wait(q_full, 0);
        if (issued_k > 0) drain_wait(k_full, (issued_k - 1) & 1);
        if (issued_v > 0) drain_wait(v_full, (issued_v - 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_bf16_f32(128, BKV, 0, 0);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, HD, 0, 1);
      // Descriptors are built once; each MMA adds a constant byte offset.
      const uint64_t qdesc = tc::smem_desc_sw128(tc::smem_u32(smem + OFF_Q), 16, 1024);
      const uint64_t kdesc = tc::smem_desc_sw128(tc::smem_u32(smem + OFF_K), 16, 1024);
      const uint64_t vdesc = tc::smem_desc_sw128(tc::smem_u32(smem + OFF_V), TILE / 2, 1024);
      bool ok = tc::mbar_wait(q_full, 0, abort_flag, a.status);
      for (int j = 0; j < n && ok; ++j) {
        const uint32_t ph = j & 1;
        if (!tc::mbar_wait(k_full, ph, abort_flag, a.status)) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
          tc::umma_bf16_ss(tmem + TM_S, tc::desc_add(qdesc, off), tc::desc_add(kdesc, off), id_s,
                           kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(s_full);
        tc::umma_commit(k_empty);
        if (!tc::mbar_wait(p_full, ph, abort_flag, a.status) ||
            !tc::mbar_wait(v_full, ph, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        // P_j is bf16 in TMEM: keys [64 h, 64 h + 64) in columns [64 h, 64 h + 32)
        // (over the scores of the softmax half that owns them); key step kk
        // (16 keys) is 8 columns.
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          tc::umma_bf16_ts(tmem + TM_O, tmem + TM_S + (kk >> 2) * 64 + (kk & 3) * 8,
                           tc::desc_add(vdesc, kk * 2048), id_pv, (j > 0 || kk > 0) ? 1u : 0u);
        tc::umma_commit(v_empty);
      }
      if (ok) tc::umma_commit(o_full);
      tc::umma_commit(drained);
      drain_wait(drained, 0);
    }
  } else {
    // Two threads per query row: warps 2..5 take keys [0, 64) of every tile,
    // warps 6..9 keys [64, 128) (a warp may only reach the TMEM lanes of
    // quarter warp % 4, which both warps of a pair share).
    const int qw = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = qw * 32 + lane;
    const int qi = qb * BQ + row;
    // Keys this row sees: [key_lo, key_hi].
    const int key_hi = min(qi, a.T - 1);
    const int key_lo = window < 0 ? 0 : qi - window;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t s_base = lane_base + TM_S + half * 64;
    const uint32_t o_base = lane_base + TM_O + half * 64;
    float* xm = reinterpret_cast<float*>(smem + OFF_X);
    float* lsum = reinterpret_cast<float*>(smem + OFF_L);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = tc::mbar_wait(s_full, j & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc::tc_fence_after();
      const int kt0 = (j_lo + j) * BKV;  // first key of the tile
      const int k0 = kt0 + half * 64;
      // The tile reaches the diagonal, T, or below the window of some row.
      const bool edge = kt0 + BKV > min(qb * BQ, a.T) ||
                        (window >= 0 && kt0 + window < qb * BQ + BQ - 1);
      // This half's 64 scores, read once; masked ones become -inf.
      uint32_t r[2][32];
      tc::tmem_ld_32x32b_x32(s_base, r[0]);
      tc::tmem_ld_32x32b_x32(s_base + 32, r[1]);
      tc::tmem_ld_wait();
      if (edge) {
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kj = k0 + c2 * 32 + i;
            if (kj > key_hi || kj < key_lo) r[c2][i] = __float_as_uint(-INFINITY);
          }
      }
      // Block maximum of the raw scores (the scale is positive): eight
      // independent chains here, then the two halves of the row combined
      // through shared memory.
      float pm[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
        for (int i = 0; i < 32; ++i) pm[i & 7] = fmaxf(pm[i & 7], __uint_as_float(r[c2][i]));
      float* xmj = xm + (j & 1) * 256;
      xmj[half * 128 + row] = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                    fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      tc::mbar_arrive(mx_ready);
      ok = tc::mbar_wait(mx_ready, j & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const float mx = fmaxf(xmj[row], xmj[128 + row]) * a.sl2;
      float alpha = 1.f;
      if (mx > m_used + kRescaleThreshold) {
        alpha = ex2(m_used - mx);  // 0 on the first tile
        m_used = mx;
      }
      const float neg_mu = (m_used == -INFINITY) ? 0.f : -m_used;
      l *= alpha;
      // p = 2^(s * scale * log2 e - m), one FFMA feeding ex2 per score; P
      // chunk c2 (32 keys, 16 packed columns) over this half's first scores.
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2(fmaf(__uint_as_float(r[c2][2 * i]), a.sl2, neg_mu));
          const float p1 = ex2(fmaf(__uint_as_float(r[c2][2 * i + 1]), a.sl2, neg_mu));
          ls[(2 * i) & 3] += p0;
          ls[(2 * i + 1) & 3] += p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tc::tmem_st_32x32b_x16(s_base + c2 * 16, pk);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // O is idle here: the commit that published S_j also covers P_{j-1} V_{j-1}.
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t o[32];
          tc::tmem_ld_32x32b_x32(o_base + c * 32, o);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc::tmem_st_32x32b_x32(o_base + c * 32, o);
        }
      }
      tc::tmem_st_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(p_full);
    }
    if (ok) {
      ok = tc::mbar_wait(o_full, 0, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {  // the row sum is split over the two halves
      lsum[half * 128 + row] = l;
      tc::mbar_arrive(l_ready);
      ok = tc::mbar_wait(l_ready, 0, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc::tc_fence_after();
      const float lt = lsum[row] + lsum[128 + row];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      __nv_bfloat16* orow = a.o + ((int64_t)b * a.T + qi) * a.ldo + col0 + half * 64;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tc::tmem_ld_32x32b_x32(o_base + c * 32, o);
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
      if (half == 0 && qi < a.T)
        a.lse[((int64_t)b * a.H + h) * a.T + qi] = (m_used + log2f(lt)) * 0.69314718055994531f;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kFwdTmemCols);
  }
}


// ------------------------------------------------------------------ backward
// One CTA per (128-key tile, head, batch row); loops over the 64-query tiles
// at or after it.  448 threads:
//   warp 0      TMA: K and V once, then Q_i and dO_i through a 4-stage ring
//               (tile i's Q/dO stay operands of dV/dK(i) while tile i+1's
//               scores are computed, so two stages would leave no prefetch);
//               its lanes also stage lse * log2(e) and D of each tile;
//   warp 1      MMA issue, per query tile i:
//                 S^T  = K Q_i^T        TMEM [  0, 64)   M 128 keys, N 64
//                 dP^T = V dO_i^T       TMEM [ 64,128)
//                 dV  += P^T dO_i       TMEM [256,384)   N 128 (dO MN-major)
//                 dK  += dS^T Q_i       TMEM [384,512)   N 128 (Q MN-major)
//                 dQ^T = K^T dS^T       TMEM [128,256)   M 128 dims, N 64, 2 buffers
//               (K^T and dS^T are the same shared tiles read MN-major), with
//               S^T/dP^T of tile i+1 issued before the gradient products of i;
//   warps 2..9  two warps per key row group, each half of the 64 columns:
//               P^T = exp(S^T/sqrt(d) - lse), dS^T = P^T (dP^T - D) as bf16
//               into K-major shared tiles; at the end dV (warps 2..5) and dK
//               (warps 6..9) rows to global memory;
//   warps 10..13 one head-dim row each: dQ^T row -> fp32 atomic adds into dq
//               (a warp covers 32 consecutive dims of one query: coalesced).
constexpr int BQB = 64;                  // query tile of the backward
constexpr int QT = BQB * 128 * 2;        // 16 KB: [64 rows x 128 dims]
constexpr int PT = 128 * BQB * 2;        // 16 KB: [128 keys x 64 queries]
constexpr int QST = 4;                   // Q / dO stages
constexpr int B_OFF_K = 0;
constexpr int B_OFF_V = B_OFF_K + TILE;
constexpr int B_OFF_Q = B_OFF_V + TILE;         // QST stages
constexpr int B_OFF_DO = B_OFF_Q + QST * QT;    // QST stages
constexpr int B_OFF_P = B_OFF_DO + QST * QT;
constexpr int B_OFF_DS = B_OFF_P + PT;
constexpr int B_OFF_LD = B_OFF_DS + PT;         // per stage: lse * log2(e) [64], D [64] (f32)
constexpr int B_OFF_BAR = B_OFF_LD + QST * 2 * BQB * 4;
constexpr int kBwdNeeded = B_OFF_BAR + 256;
constexpr int kBwdSmem = 232448;                // the per-block maximum; slack absorbs alignment
static_assert(kBwdNeeded + 512 <= kBwdSmem, "attention backward shared memory budget");
constexpr int kBwdThreads = 448;
constexpr uint32_t TB_S = 0, TB_DP = 64, TB_DQ = 128, TB_DV = 256, TB_DK = 384;

struct BwdArgs {
  int T, H, nkb, nqb;
  int group;   // query heads per KV head
  int window;  // query t sees keys [t - window, t]; < 0: every key up to t
  float sl2, scale;
  const float* lse;
  const float* delta;
  float* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int64_t ldg;
  int* status;
};

// GW: grouped KV heads or a window in play; the plain instance compiles
// with group 1 and no window as constants (its tile t is query tile i0 + t
// of head hk).
template <bool GW>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                       const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if ((smem - smem_raw) + kBwdNeeded > kBwdSmem) {  // never expected: base misaligned past slack
    if (threadIdx.x == 0 && a.status) atomicExch(a.status, kDevTimeout);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + B_OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* qd_full = bars + 1;              // [QST]
  uint64_t* qd_empty = bars + 1 + QST;       // [QST]
  uint64_t* sdp_full = bars + 1 + 2 * QST;
  uint64_t* sdp_empty = sdp_full + 1;
  uint64_t* pds_full = sdp_full + 2;
  uint64_t* pds_empty = sdp_full + 3;
  uint64_t* dq_full = sdp_full + 4;          // [2]
  uint64_t* dq_empty = sdp_full + 6;         // [2]
  uint64_t* dkv_full = sdp_full + 8;
  uint64_t* drained = sdp_full + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sdp_full + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;  // hk: the KV head
  const int group = GW ? a.group : 1;
  const int window = GW ? a.window : -1;
  const int i0 = (kb * BKV) / BQB;
  // Query tiles at or after this key tile, up to the last one a window reaches;
  // every query head of the KV head's group in turn (tile t: head
  // hk * group + t / nqt, query tile i0 + t % nqt), so dK and dV accumulate
  // over the whole group in TMEM.
  const int i_hi = window < 0 ? a.nqb - 1 : min(a.nqb - 1, (kb * BKV + BKV - 1 + window) / BQB);
  const int nqt = i_hi - i0 + 1;
  const int nblk = group * nqt;
  const int kcol0 = hk * HD;

  if (threadIdx.x == 0) {
    tc::mbar_init(kv_full, 1);
    for (int i = 0; i < QST; ++i) {
      tc::mbar_init(&qd_full[i], 32);  // the TMA lane (with its bytes) + 31 lse/D loader lanes
      tc::mbar_init(&qd_empty[i], 1);
    }
    tc::mbar_init(sdp_full, 1);
    tc::mbar_init(sdp_empty, 256);
    tc::mbar_init(pds_full, 256);
    tc::mbar_init(pds_empty, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&dq_full[i], 1);
      tc::mbar_init(&dq_empty[i], 128);
    }
    tc::mbar_init(dkv_full, 1);
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

  if (warp == 0) {
    // Lane 0 issues the TMA copies; all 32 lanes stage lse * log2(e) and D of
    // the query tile into shared memory and arrive on the same barrier.
    if (lane == 0) {
      tc::tma_prefetch_desc(&tq);
      tc::tma_prefetch_desc(&tk);
      tc::tma_prefetch_desc(&tv);
      tc::tma_prefetch_desc(&tdo);
      tc::mbar_arrive_expect_tx(kv_full, 2 * TILE);
      for (int c = 0; c < 2; ++c) {
        tc::tma_load_3d(smem + B_OFF_K + c * (TILE / 2), &tk, kv_full, kcol0 + 64 * c, kb * BKV, b);
        tc::tma_load_3d(smem + B_OFF_V + c * (TILE / 2), &tv, kv_full, kcol0 + 64 * c, kb * BKV, b);
      }
    }
    int issued = 0;
    bool ok = true;
    for (int t = 0; t < nblk; ++t) {
      const int st = t % QST;
      const uint32_t ph = (t / QST) & 1;
      bool w = true;
      if (lane == 0) w = tc::mbar_wait(&qd_empty[st], ph ^ 1, abort_flag, a.status);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) { ok = false; break; }
      const int hq = GW ? hk * group + t / nqt : hk;
      const int q0 = (i0 + (GW ? t % nqt : t)) * BQB;
      const int qcol0 = hq * HD;
      const float* lse_bh = a.lse + ((int64_t)b * a.H + hq) * a.T;
      const float* d_bh = a.delta + ((int64_t)b * a.H + hq) * a.T;
      float* ld = reinterpret_cast<float*>(smem + B_OFF_LD) + st * 2 * BQB;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = lane + 32 * u;
        const int q = q0 + c;
        ld[c] = q < a.T ? lse_bh[q] * 1.4426950408889634f : INFINITY;
        ld[BQB + c] = q < a.T ? d_bh[q] : 0.f;
      }
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&qd_full[st], 2 * QT);
        for (int c = 0; c < 2; ++c) {
          tc::tma_load_3d(smem + B_OFF_Q + st * QT + c * (QT / 2), &tq, &qd_full[st], qcol0 + 64 * c, q0, b);
          tc::tma_load_3d(smem + B_OFF_DO + st * QT + c * (QT / 2), &tdo, &qd_full[st], qcol0 + 64 * c, q0, b);
        }
      } else {
        tc::mbar_arrive(&qd_full[st]);
      }
      ++issued;
    }
    if (!ok && lane == 0) {
      drain_wait(kv_full, 0);
      for (int t = max(0, issued - QST); t < issued; ++t) drain_wait(&qd_full[t % QST], (t / QST) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_sdp = tc::idesc_bf16_f32(128, BQB, 0, 0);
      const uint32_t id_acc = tc::idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t id_dq = tc::idesc_bf16_f32(128, BQB, 1, 1);
      // Descriptors are built once; each MMA adds a constant byte offset.
      const uint64_t kK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_K), 16, 1024);
      const uint64_t vK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_V), 16, 1024);
      const uint64_t kMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_K), TILE / 2, 1024);
      const uint64_t qK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_Q), 16, 1024);
      const uint64_t doK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DO), 16, 1024);
      const uint64_t qMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_Q), QT / 2, 1024);
      const uint64_t doMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DO), QT / 2, 1024);
      const uint64_t pK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_P), 16, 1024);
      const uint64_t dsK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DS), 16, 1024);
      const uint64_t dsMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DS), PT, 1024);
      bool ok = tc::mbar_wait(kv_full, 0, abort_flag, a.status);
      // S^T and dP^T of query tile t into TMEM once the tile has landed and the
      // softmax warps have read the previous scores.
      auto issue_sdp = [&](int t) -> bool {
        const int st = t % QST;
        if (!tc::mbar_wait(&qd_full[st], (t / QST) & 1, abort_flag, a.status)) return false;
        if (t > 0 && !tc::mbar_wait(sdp_empty, (t - 1) & 1, abort_flag, a.status)) return false;
        tc::tc_fence_after();
        const uint64_t qd = qK + (uint64_t)((st * QT) >> 4);
        const uint64_t dod = doK + (uint64_t)((st * QT) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
          const uint32_t bo = (kk >> 2) * (QT / 2) + (kk & 3) * 32;
          tc::umma_bf16_ss(tmem + TB_S, tc::desc_add(kK, ao), tc::desc_add(qd, bo), id_sdp,
                           kk > 0 ? 1u : 0u);
          tc::umma_bf16_ss(tmem + TB_DP, tc::desc_add(vK, ao), tc::desc_add(dod, bo), id_sdp,
                           kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(sdp_full);
        return true;
      };
      if (ok) ok = issue_sdp(0);
      for (int t = 0; t < nblk && ok; ++t) {
        const int st = t % QST;
        if (t + 1 < nblk && !issue_sdp(t + 1)) { ok = false; break; }
        const int db = t & 1;  // dQ accumulator of this tile
        if (!tc::mbar_wait(pds_full, t & 1, abort_flag, a.status) ||
            !tc::mbar_wait(&dq_empty[db], ((t >> 1) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t qmn = qMN + (uint64_t)((st * QT) >> 4);
        const uint64_t domn = doMN + (uint64_t)((st * QT) >> 4);
#pragma unroll
        for (int kk = 0; kk < BQB / 16; ++kk) {
          const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
          tc::umma_bf16_ss(tmem + TB_DV, tc::desc_add(pK, kk * 32), tc::desc_add(domn, kk * 2048),
                           id_acc, acc);
          tc::umma_bf16_ss(tmem + TB_DK, tc::desc_add(dsK, kk * 32), tc::desc_add(qmn, kk * 2048),
                           id_acc, acc);
        }
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          tc::umma_bf16_ss(tmem + TB_DQ + db * BQB, tc::desc_add(kMN, kk * 2048),
                           tc::desc_add(dsMN, kk * 2048), id_dq, kk > 0 ? 1u : 0u);
        tc::umma_commit(pds_empty);
        tc::umma_commit(&qd_empty[st]);
        tc::umma_commit(&dq_full[db]);
      }
      if (ok) tc::umma_commit(dkv_full);
      tc::umma_commit(drained);
      drain_wait(drained, 0);
    }
  } else if (warp < 10) {
    // ---------------- P^T and dS^T: one key row per thread, half the columns per warp
    const int qw = warp & 3;
    const int ch = (warp - 2) >> 2;  // column half: queries [32 ch, 32 ch + 32) of the tile
    const int row = qw * 32 + lane;
    const int key = kb * BKV + row;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t p_row = tc::smem_u32(smem + B_OFF_P) + row * 128;
    const uint32_t ds_row = tc::smem_u32(smem + B_OFF_DS) + row * 128;
    bool ok = true;
    for (int t = 0; t < nblk; ++t) {
      const int q0 = (i0 + (GW ? t % nqt : t)) * BQB + 32 * ch;
      const float* ld = reinterpret_cast<const float*>(smem + B_OFF_LD) + (t % QST) * 2 * BQB + 32 * ch;
      ok = tc::mbar_wait(sdp_full, t & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc::tc_fence_after();
      uint32_t sv[32], dp[32];
      tc::tmem_ld_32x32b_x32(lane_base + TB_S + 32 * ch, sv);
      tc::tmem_ld_32x32b_x32(lane_base + TB_DP + 32 * ch, dp);
      tc::tmem_ld_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(sdp_empty);
      // The tile's lse/D, staged by the TMA warp and published by the stage's
      // qd_full barrier (already complete: the scores came from it).
      ok = tc::mbar_wait(&qd_full[t % QST], (t / QST) & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      uint32_t pp[16], pd[16];
      const bool edge = (q0 < key + 1) || (q0 + 32 > a.T) || (key >= a.T) ||
                        (window >= 0 && q0 + 31 > key + window);  // diagonal, T or window
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float p0 = ex2(__uint_as_float(sv[2 * c]) * a.sl2 - ld[2 * c]);
        float p1 = ex2(__uint_as_float(sv[2 * c + 1]) * a.sl2 - ld[2 * c + 1]);
        if (edge) {
          const int qa = q0 + 2 * c, qb2 = qa + 1;
          if (qa < key || qa >= a.T || key >= a.T || (window >= 0 && qa > key + window)) p0 = 0.f;
          if (qb2 < key || qb2 >= a.T || key >= a.T || (window >= 0 && qb2 > key + window)) p1 = 0.f;
        }
        const float d0 = p0 * (__uint_as_float(dp[2 * c]) - ld[BQB + 2 * c]);
        const float d1 = p1 * (__uint_as_float(dp[2 * c + 1]) - ld[BQB + 2 * c + 1]);
        pp[c] = pack_bf16x2(p0, p1);
        pd[c] = pack_bf16x2(d0, d1);
      }
      ok = tc::mbar_wait(pds_empty, (t & 1) ^ 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t sw = (uint32_t)(((4 * ch + u) ^ (row & 7)) << 4);
        tc::st_shared_v4(p_row + sw, pp[4 * u], pp[4 * u + 1], pp[4 * u + 2], pp[4 * u + 3]);
        tc::st_shared_v4(ds_row + sw, pd[4 * u], pd[4 * u + 1], pd[4 * u + 2], pd[4 * u + 3]);
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(pds_full);
    }
    if (ok) {
      ok = tc::mbar_wait(dkv_full, 0, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      // Warps of column half 0 write dV rows, those of half 1 dK rows.
      tc::tc_fence_after();
      const int64_t grow = ((int64_t)b * a.T + key) * a.ldg + kcol0;
      const uint32_t base = lane_base + (ch ? TB_DK : TB_DV);
      const float mul = ch ? a.scale : 1.f;
      __nv_bfloat16* dst = (ch ? a.dk : a.dv) + grow;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tc::tmem_ld_32x32b_x32(base + c * 32, o);
        tc::tmem_ld_wait();
        if (key < a.T) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * u + 0]) * mul, __uint_as_float(o[8 * u + 1]) * mul);
            v.y = pack_bf16x2(__uint_as_float(o[8 * u + 2]) * mul, __uint_as_float(o[8 * u + 3]) * mul);
            v.z = pack_bf16x2(__uint_as_float(o[8 * u + 4]) * mul, __uint_as_float(o[8 * u + 5]) * mul);
            v.w = pack_bf16x2(__uint_as_float(o[8 * u + 6]) * mul, __uint_as_float(o[8 * u + 7]) * mul);
            reinterpret_cast<uint4*>(dst + c * 32)[u] = v;
          }
        }
      }
    }
  } else {
    // ---------------- dQ^T rows: one head-dim per thread, atomics into dq
    const int qw = warp & 3;
    const int dim = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const int64_t dq_row = (int64_t)a.H * HD;
    for (int t = 0; t < nblk; ++t) {
      const int q0 = (i0 + (GW ? t % nqt : t)) * BQB;
      float* dq_bh = a.dq + (int64_t)b * a.T * dq_row + (GW ? hk * group + t / nqt : hk) * HD + dim;
      bool ok = tc::mbar_wait(&dq_full[t & 1], (t >> 1) & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::tc_fence_after();
      float* dst = dq_bh + (int64_t)q0 * dq_row;
      const int nq = min(BQB, a.T - q0);
#pragma unroll 1
      for (int c0 = 0; c0 < BQB; c0 += 16) {
        uint32_t v[16];
        tc::tmem_ld_32x32b_x16(lane_base + TB_DQ + (t & 1) * BQB + c0, v);
        tc::tmem_ld_wait();
        if (c0 + 16 == BQB) {  // the whole tile has been read: TMEM may be reused
          tc::tc_fence_before();
          tc::mbar_arrive(&dq_empty[t & 1]);
        }
        float vv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) vv[j] = __uint_as_float(v[j]) * a.scale;
        if (c0 + 16 <= nq) {
#pragma unroll
          for (int j = 0; j < 16; ++j) atomicAdd(dst + (int64_t)(c0 + j) * dq_row, vv[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < nq) atomicAdd(dst + (int64_t)(c0 + j) * dq_row, vv[j]);
        }
      }
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

// Query-key pairs a causal window keeps: sum over t of min(t, window) + 1
// (every key up to t when window < 0).
double causal_pairs(int T, int window) {
  if (window < 0 || window >= T - 1) return (double)T * (T + 1) / 2.0;
  const double w = window;
  return (w + 1) * (w + 2) / 2.0 + (T - w - 1) * (w + 1);  // rows t <= w, then rows t > w
}

nc_status attention_fwd_ex(const void* q, int64_t ldq, const void* k, const void* v, int64_t ldkv,
                           void* o, int64_t ldo, float* lse, int B, int T, int H, int Hkv,
                           int window, int* status, cudaStream_t s, Profiler* prof) {
  if (B < 1 || T < 1 || H < 1 || Hkv < 1 || H % Hkv || !q || !k || !v || !o || !lse)
    return fail(NC_ERR_INVALID_ARG, "attention_fwd: bad arguments (H must be a multiple of Hkv)");
  if (ldq % 8 || ldkv % 8 || ldo % 8 ||
      ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(o)) & 15))
    return fail(NC_ERR_INVALID_ARG, "attention_fwd: rows must be 16-byte aligned");
  static DeviceOnce attr;
  NC_TRY(once_per_device(attr, []() -> nc_status {
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_tc_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem));
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_tc_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem));
    return NC_OK;
  }));
  CUtensorMap mq, mk, mv;
  // Box heights must match the tile sizes the kernel's byte counts assume.
  if (!make_tmap_bf16_3d(&mq, q, (uint64_t)H * HD, T, B, ldq, (int64_t)T * ldq, BQ) ||
      !make_tmap_bf16_3d(&mk, k, (uint64_t)Hkv * HD, T, B, ldkv, (int64_t)T * ldkv, BKV) ||
      !make_tmap_bf16_3d(&mv, v, (uint64_t)Hkv * HD, T, B, ldkv, (int64_t)T * ldkv, BKV))
    return fail(NC_ERR_INVALID_ARG, "attention_fwd: cuTensorMapEncodeTiled rejected q/k/v");
  FwdArgs a;
  a.T = T;
  a.nqb = (T + BQ - 1) / BQ;
  a.sl2 = (float)(1.4426950408889634 / std::sqrt((double)HD));
  a.o = static_cast<__nv_bfloat16*>(o);
  a.ldo = ldo;
  a.lse = lse;
  a.H = H;
  a.group = H / Hkv;
  // A window of T - 1 or more keys is full causal: such a window runs as
  // unbounded, which also keeps the kernels' window sums (up to ~2T) in range.
  a.window = (window < 0 || window >= T - 1) ? -1 : window;
  a.status = status;
  const double flops = 4.0 * B * H * HD * causal_pairs(T, a.window);
  Probe probe(prof, s, "attn_fwd", flops, 0.0);
  dim3 grid(a.nqb, H, B);
  if (a.group > 1 || a.window >= 0)
    attn_fwd_tc_kernel<true><<<grid, kThreads, kSmem, s>>>(mq, mk, mv, a);
  else
    attn_fwd_tc_kernel<false><<<grid, kThreads, kSmem, s>>>(mq, mk, mv, a);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status attention_fwd(const void* q, const void* k, const void* v, int64_t ld, void* o,
                        int64_t ldo, float* lse, int B, int T, int H, int* status, cudaStream_t s,
                        Profiler* prof) {
  return attention_fwd_ex(q, ld, k, v, ld, o, ldo, lse, B, T, H, H, -1, status, s, prof);
}


nc_status attention_bwd_tc_ex(const void* q, int64_t ldq, const void* k, const void* v, int64_t ldkv,
                              const void* dout, int64_t ldo, const float* lse, const float* delta,
                              float* dq, void* dk, void* dv, int64_t ldg, int B, int T, int H,
                              int Hkv, int window, int* status, cudaStream_t s, Profiler* prof) {
  static DeviceOnce attr;
  NC_TRY(once_per_device(attr, []() -> nc_status {
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_tc_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem));
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_tc_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem));
    return NC_OK;
  }));
  if (Hkv < 1 || H % Hkv) return fail(NC_ERR_INVALID_ARG, "attention_bwd: H must be a multiple of Hkv");
  if (ldq % 8 || ldkv % 8 || ldo % 8 || ldg % 8 ||
      ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(dout) |
        reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 15))
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: rows must be 16-byte aligned");
  CUtensorMap mq, mk, mv, mdo;
  const uint64_t qcols = (uint64_t)H * HD, kvcols = (uint64_t)Hkv * HD;
  if (!make_tmap_bf16_3d(&mq, q, qcols, T, B, ldq, (int64_t)T * ldq, BQB) ||
      !make_tmap_bf16_3d(&mk, k, kvcols, T, B, ldkv, (int64_t)T * ldkv, BKV) ||
      !make_tmap_bf16_3d(&mv, v, kvcols, T, B, ldkv, (int64_t)T * ldkv, BKV) ||
      !make_tmap_bf16_3d(&mdo, dout, qcols, T, B, ldo, (int64_t)T * ldo, BQB))
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: cuTensorMapEncodeTiled rejected an operand");
  BwdArgs a;
  a.T = T;
  a.H = H;
  a.nkb = (T + BKV - 1) / BKV;
  a.nqb = (T + BQB - 1) / BQB;
  a.group = H / Hkv;
  a.window = (window < 0 || window >= T - 1) ? -1 : window;  // as in the forward
  a.scale = (float)(1.0 / std::sqrt((double)HD));
  a.sl2 = (float)(1.4426950408889634 / std::sqrt((double)HD));
  a.lse = lse;
  a.delta = delta;
  a.dq = dq;
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.ldg = ldg;
  a.status = status;
  const double flops = 10.0 * B * H * HD * causal_pairs(T, a.window);
  Probe probe(prof, s, "attn_bwd", flops, 0.0);
  dim3 grid(a.nkb, Hkv, B);  // one CTA per key tile and KV head; it loops over the group
  if (a.group > 1 || a.window >= 0)
    attn_bwd_tc_kernel<true><<<grid, kBwdThreads, kBwdSmem, s>>>(mq, mk, mv, mdo, a);
  else
    attn_bwd_tc_kernel<false><<<grid, kBwdThreads, kBwdSmem, s>>>(mq, mk, mv, mdo, a);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status attention_bwd_tc(const void* q, const void* k, const void* v, int64_t ld,
                           const void* dout, int64_t ldo, const float* lse, const float* delta,
                           float* dq, void* dk, void* dv, int64_t ldg, int B, int T, int H,
                           int* status, cudaStream_t s, Profiler* prof) {
  return attention_bwd_tc_ex(q, ld, k, v, ld, dout, ldo, lse, delta, dq, dk, dv, ldg, B, T, H, H, -1,
                             status, s, prof);
}

}  // namespace nc
