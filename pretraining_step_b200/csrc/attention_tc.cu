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
#include "exp2_poly.cuh"

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
  int B;
};

// 2^x by the MUFU instruction (ex2.approx, flush-to-zero): the softmax
// arguments are <= 0 (or <= 8 with a stale maximum), far from its range limits.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// In the key-side backward's P^T phase one pair of exponentials in every
// kPolyPeriod goes to the FMA pipe (exp2_fma2) instead of the exponential
// unit, which then needs 3/4 of its time per score tile.  (Measured on the
// step: the key side about 1% faster with one pair in four, slower with one
// in two; the forward was slower with any share, so it keeps the unit.)
constexpr int kPolyPeriod = 4;
__device__ __forceinline__ constexpr bool poly_pair(int pair) { return pair % kPolyPeriod == kPolyPeriod - 1; }

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
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


// ------------------------------------------------------------------ forward, two query tiles, persistent
// The plain forward (one KV head per query head, no window): one CTA per SM
// walks work items, each two query tiles (2p, 2p + 1) of one (head, batch
// row) whose shared key/value tiles it streams once.  The two score chains
// interleave on the tensor pipe, so one tile's softmax runs while the other
// tile's products execute:
//   tensor:  ... PV_a(j)  S_a(j+1)  PV_b(j)  S_b(j+1)  PV_a(j+1) ...
// Items come in pairs of one (head, row), query-tile pair npairs - 1 - j and
// then j: their key-tile counts add up to the same total whatever j is, so
// dealing item pair s to CTA s mod gridDim.x balances the work, and the CTAs
// working at the same time share a (head, row)'s K and V tiles in L2.  The
// K/V ring runs on across items, the next item's Q tiles load as soon as the
// current item's last products that read them are done, and the next item's
// first scores are computed while the softmax warps still write the current
// item's output (its first P V product waits for that).
// 320 threads:
//   warp 0       TMA: Q_a and Q_b per item, K_j and V_j through two stages
//                each (a stage is released when both tiles' products that
//                read it are done);
//   warp 1       TMEM owner and single-thread MMA issue in the order above;
//   warps 2..5   softmax of tile a, warps 6..9 softmax of tile b: one thread
//                per query row holding its 128 scores, so the row maximum
//                needs no exchange between threads; the maximum is raised
//                only past 2^8 (O rescaled in TMEM then), and P is written as
//                bf16 over the scores it replaces (key k in column k / 2);
//                at the item's end O / l and lse of the row.
// TMEM columns: S_a [0,128), S_b [128,256), O_a [256,384), O_b [384,512).
// The MMAs run in issue order, so S_x(j+1) never overwrites P_x(j) before
// PV_x(j) has read it, and the commit that publishes S_x(j+1) also covers
// PV_x(j): O_x is idle while tile x's softmax runs.
constexpr int kPPThreads = 320;
constexpr int PP_OFF_QA = 0;       // Q_a, then Q_b at + TILE
constexpr int PP_OFF_K = 2 * TILE;   // 2 stages
constexpr int PP_OFF_V = 4 * TILE;   // 2 stages
constexpr int PP_OFF_BAR = 6 * TILE;
constexpr int kPPSmem = PP_OFF_BAR + 512;

// This CTA's items in order: item pair s (stride gridDim.x) is query-tile
// pairs npairs - 1 - j (sub 0) and j (sub 1) of one (head, row).
struct FwdWalk {
  int s, sub;
  __device__ __forceinline__ void start() {
    s = blockIdx.x;
    sub = 0;
  }
  __device__ __forceinline__ bool valid(int nsuper) const { return s < nsuper; }
  // Query-tile pair, head and batch row of the current item.
  __device__ __forceinline__ void item(const FwdArgs& a, int npairs, int& pr, int& h, int& b) const {
    const int spg = (npairs + 1) / 2;
    const int grp = s / spg;
    const int j = s - grp * spg;
    pr = sub ? j : npairs - 1 - j;
    h = grp % a.H;
    b = grp / a.H;
  }
  __device__ __forceinline__ void next(int npairs) {
    const int j = s % ((npairs + 1) / 2);
    if (sub == 0 && npairs - 1 - j != j) {
      sub = 1;
    } else {
      sub = 0;
      s += gridDim.x;
    }
  }
};

__global__ void __launch_bounds__(kPPThreads, 1)
    attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const FwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((tc::smem_u32(smem_raw) & 1023u) != 0) {  // never expected; no room to realign
    if (threadIdx.x == 0 && a.status) atomicExch(a.status, kDevTimeout);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PP_OFF_BAR);
  uint64_t* q_full = bars + 0;    // [2 tiles]
  uint64_t* q_empty = bars + 2;   // [2 tiles]
  uint64_t* k_full = bars + 4;    // [2]
  uint64_t* k_empty = bars + 6;   // [2]
  uint64_t* v_full = bars + 8;    // [2]
  uint64_t* v_empty = bars + 10;  // [2]
  uint64_t* s_full = bars + 12;   // [2 tiles]
  uint64_t* p_full = bars + 14;   // [2 tiles]
  uint64_t* o_full = bars + 16;   // [2 tiles]
  uint64_t* o_empty = bars + 18;  // [2 tiles]
  uint64_t* drained = bars + 20;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 21);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int npairs = (a.nqb + 1) / 2;
  const int nsuper = (npairs + 1) / 2 * a.H * a.B;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&q_full[i], 1);
      tc::mbar_init(&q_empty[i], 1);
      tc::mbar_init(&k_full[i], 1);
      tc::mbar_init(&k_empty[i], 1);
      tc::mbar_init(&v_full[i], 1);
      tc::mbar_init(&v_empty[i], 1);
      tc::mbar_init(&s_full[i], 1);
      tc::mbar_init(&p_full[i], 128);
      tc::mbar_init(&o_full[i], 1);
      tc::mbar_init(&o_empty[i], 128);
    }
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
    if (lane == 0) {
      tc::tma_prefetch_desc(&tq);
      tc::tma_prefetch_desc(&tk);
      tc::tma_prefetch_desc(&tv);
      int nq[2] = {0, 0};  // loads into each Q slot so far
      int g = 0;           // K/V tiles loaded so far (ring position)
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      FwdWalk w;
      for (w.start(); w.valid(nsuper) && ok; w.next(npairs)) {
        int pr, h, b;
        w.item(a, npairs, pr, h, b);
        const int qt0 = 2 * pr;
        const bool has_b = qt0 + 1 < a.nqb;
        const int nkv = has_b ? qt0 + 2 : qt0 + 1;
        const int col0 = h * HD;
        for (int x = 0; x < (has_b ? 2 : 1); ++x) {
          // The slot is free once the products of the previous item that
          // read it are done.
          if (nq[x] > 0 && !tc::mbar_wait(&q_empty[x], (nq[x] - 1) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&q_full[x], TILE);
          for (int c = 0; c < 2; ++c)
            tc::tma_load_3d(smem + PP_OFF_QA + x * TILE + c * (TILE / 2), &tq, &q_full[x], col0 + 64 * c,
                            (qt0 + x) * BQ, b);
          ++nq[x];
        }
        for (int j = 0; j < nkv && ok; ++j, ++g) {
          const int st = g & 1;
          const uint32_t ph = (g >> 1) & 1;
          if (!tc::mbar_wait(&k_empty[st], ph ^ 1, abort_flag, a.status)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&k_full[st], TILE);
          for (int c = 0; c < 2; ++c)
            tc::tma_load_3d(smem + PP_OFF_K + st * TILE + c * (TILE / 2), &tk, &k_full[st],
                            col0 + 64 * c, j * BKV, b);
          ++issued_k;
          if (!tc::mbar_wait(&v_empty[st], ph ^ 1, abort_flag, a.status)) { ok = false; break; }
          tc::mbar_arrive_expect_tx(&v_full[st], TILE);
          for (int c = 0; c < 2; ++c)
            tc::tma_load_3d(smem + PP_OFF_V + st * TILE + c * (TILE / 2), &tv, &v_full[st],
                            col0 + 64 * c, j * BKV, b);
          ++issued_v;
        }
      }
      if (!ok) {
        for (int x = 0; x < 2; ++x)
          if (nq[x] > 0) drain_wait(&q_full[x], (nq[x] - 1) & 1);
        for (int j = max(0, issued_k - 2); j < issued_k; ++j) drain_wait(&k_full[j & 1], (j >> 1) & 1);
        for (int j = max(0, issued_v - 2); j < issued_v; ++j) drain_wait(&v_full[j & 1], (j >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_bf16_f32(128, BKV, 0, 0);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, HD, 0, 1);
      const uint64_t qdesc = tc::smem_desc_sw128(tc::smem_u32(smem + PP_OFF_QA), 16, 1024);
      const uint64_t kdesc = tc::smem_desc_sw128(tc::smem_u32(smem + PP_OFF_K), 16, 1024);
      const uint64_t vdesc = tc::smem_desc_sw128(tc::smem_u32(smem + PP_OFF_V), TILE / 2, 1024);
      // S_x = Q_x K^T (K from ring slot ks) into tile x's score columns.
      auto issue_s = [&](int x, int ks) {
        const uint64_t qd = tc::desc_add(qdesc, x * TILE);
        const uint64_t kd = tc::desc_add(kdesc, ks * TILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
          tc::umma_bf16_ss(tmem + 128 * x, tc::desc_add(qd, off), tc::desc_add(kd, off), id_s,
                           kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(&s_full[x]);
      };
      // O_x (+)= P_x V (V from ring slot vs), P from TMEM (key k in column
      // k / 2 of the tile's score block; 16 keys per MMA).
      auto issue_pv = [&](int x, int vs, bool acc) {
        const uint64_t vd = tc::desc_add(vdesc, vs * TILE);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          tc::umma_bf16_ts(tmem + 256 + 128 * x, tmem + 128 * x + kk * 8,
                           tc::desc_add(vd, kk * 2048), id_pv, (acc || kk > 0) ? 1u : 0u);
      };
      int nq[2] = {0, 0}, np[2] = {0, 0}, no[2] = {0, 0};
      int g = 0;
      bool ok = true;
      FwdWalk w;
      for (w.start(); w.valid(nsuper) && ok; w.next(npairs)) {
        int pr, h, b;
        w.item(a, npairs, pr, h, b);
        const int qt0 = 2 * pr;
        const bool has_b = qt0 + 1 < a.nqb;
        const int xs = has_b ? 2 : 1;
        const int nkv = has_b ? qt0 + 2 : qt0 + 1;
        const int last[2] = {qt0, qt0 + 1};  // each tile's last key tile (its diagonal)
        if (!tc::mbar_wait(&k_full[g & 1], (g >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
        for (int x = 0; x < xs && ok; ++x) {
          ok = tc::mbar_wait(&q_full[x], nq[x] & 1, abort_flag, a.status);
          ++nq[x];
          if (!ok) break;
          tc::tc_fence_after();
          issue_s(x, g & 1);
          if (last[x] == 0) tc::umma_commit(&q_empty[x]);  // the item's only scores of tile x
        }
        if (!ok) break;
        tc::umma_commit(&k_empty[g & 1]);
        for (int j = 0; j < nkv && ok; ++j) {
          const int st = (g + j) & 1;
          if (!tc::mbar_wait(&v_full[st], ((g + j) >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
          bool k_next = false;  // K_{j+1} has landed
          for (int x = 0; x < xs; ++x) {
            if (j > last[x]) continue;
            if (!tc::mbar_wait(&p_full[x], np[x] & 1, abort_flag, a.status)) { ok = false; break; }
            ++np[x];
            // The item's first product overwrites O_x: the softmax warps
            // must have written out the previous item's.
            if (j == 0 && no[x] > 0 && !tc::mbar_wait(&o_empty[x], (no[x] - 1) & 1, abort_flag, a.status)) {
              ok = false;
              break;
            }
            tc::tc_fence_after();
            issue_pv(x, st, j > 0);
            if (j == last[x]) {
              tc::umma_commit(&o_full[x]);
              ++no[x];
              continue;
            }
            if (!k_next) {
              if (!tc::mbar_wait(&k_full[(g + j + 1) & 1], ((g + j + 1) >> 1) & 1, abort_flag, a.status)) {
                ok = false;
                break;
              }
              tc::tc_fence_after();
              k_next = true;
            }
            issue_s(x, (g + j + 1) & 1);
            if (j + 1 == last[x]) tc::umma_commit(&q_empty[x]);  // Q_x's last reader
          }
          if (!ok) break;
          tc::umma_commit(&v_empty[st]);
          if (k_next) tc::umma_commit(&k_empty[(g + j + 1) & 1]);
        }
        g += nkv;
      }
      tc::umma_commit(drained);
      drain_wait(drained, 0);
    }
  } else {
    // Softmax of tile x: warps 2..5 (x = 0) and 6..9 (x = 1), one thread per
    // query row (a warp may only reach the TMEM lanes of quarter warp % 4).
    const int x = (warp - 2) >> 2;
    const int qw = warp & 3;
    const int row = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t s_base = lane_base + 128 * x;
    const uint32_t o_base = lane_base + 256 + 128 * x;
    int ns = 0, no = 0;  // score tiles and items of tile x so far
    bool ok = true;
    FwdWalk w;
    for (w.start(); w.valid(nsuper) && ok; w.next(npairs)) {
      int pr, h, b;
      w.item(a, npairs, pr, h, b);
      const int qb = 2 * pr + x;
      if (qb >= a.nqb) continue;  // no tile b in this item
      const int qi = qb * BQ + row;
      const int key_hi = min(qi, a.T - 1);
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j <= qb; ++j, ++ns) {
        ok = tc::mbar_wait(&s_full[x], ns & 1, abort_flag, a.status);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc::tc_fence_after();
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_ld_32x32b_x32(s_base + 32 * c, r[c]);
        tc::tmem_ld_wait();
        // The diagonal tile or the tile that reaches T: keys past this row's
        // last visible key become -inf.
        const bool edge = j * BKV + BKV > min(qb * BQ, a.T);
        if (edge) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (j * BKV + 32 * c + i > key_hi) r[c][i] = __float_as_uint(-INFINITY);
        }
        // Row maximum with the three-input max: two scores per instruction.
        float pm[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            pm[(i >> 1) & 7] = fmax3(pm[(i >> 1) & 7], __uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1]));
        const float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7])) * a.sl2;
        float alpha = 1.f;
        if (mx > m_used + kRescaleThreshold) {
          alpha = ex2(m_used - mx);  // 0 on the first tile
          m_used = mx;
        }
        const float neg_mu = (m_used == -INFINITY) ? 0.f : -m_used;
        l *= alpha;
        // Arguments two at a time (packed fp32 pairs: one issue slot per two
        // scores, the same rounding as scalar fma).
        const float2 sl2v = make_float2(a.sl2, a.sl2), nmu = make_float2(neg_mu, neg_mu);
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(r[c][2 * i]), __uint_as_float(r[c][2 * i + 1])),
                                        sl2v, nmu);
            const float p0 = ex2(x.x), p1 = ex2(x.y);
            ls[(2 * i) & 3] += p0;
            ls[(2 * i + 1) & 3] += p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          // Keys [32 c, 32 c + 32) to columns [16 c, 16 c + 16): over scores
          // already held in registers.
          tc::tmem_st_32x32b_x16(s_base + 16 * c, pk);
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        // O is idle here: the commit that published S_j also covers P_{j-1} V_{j-1}.
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          const float2 al = make_float2(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tc::tmem_ld_32x32b_x32(o_base + c * 32, o);
            tc::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), al);
              o[i] = __float_as_uint(v.x);
              o[i + 1] = __float_as_uint(v.y);
            }
            tc::tmem_st_32x32b_x32(o_base + c * 32, o);
          }
        }
        tc::tmem_st_wait();
        tc::tc_fence_before();
        tc::mbar_arrive(&p_full[x]);
      }
      if (!ok) break;
      ok = tc::mbar_wait(&o_full[x], no & 1, abort_flag, a.status);
      ++no;
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = a.o + ((int64_t)b * a.T + qi) * a.ldo + h * HD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tc::tmem_ld_32x32b_x32(o_base + c * 32, o);
        tc::tmem_ld_wait();
        if (c == 3) {  // O_x is read: the next item's first product may overwrite it
          tc::tc_fence_before();
          tc::mbar_arrive(&o_empty[x]);
        }
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

// ------------------------------------------------------------------ backward
// One CTA per (128-key tile, KV head, batch row); it loops over the 128-query
// tiles at or after its keys (every query head of the KV head's group in
// turn).  Every product is a 128 x 128 x 128 tcgen05 MMA, and the two score
// gradients that feed the key-side products (P^T and dS^T) reach the tensor
// core from TMEM, so their shared-memory operand traffic is one tile per
// product instead of two.  448 threads:
//   warp 0      TMA: K and V once, then Q_i and dO_i (two stages each, their
//               own barriers, so dO of tile i + 2 can land while Q_i is still
//               an operand); its lanes also stage lse * log2(e) (with Q) and
//               D (with dO) of the tile;
//   warp 1      TMEM owner and single-thread MMA issue, per query tile i:
//                 dV  += P_i^T dO_i     (A = P^T from TMEM, dO MN-major)
//                 S^T_{i+1} = K Q_{i+1}^T            -> TMEM S
//                 dK  += dS_i^T Q_i     (A = dS^T from TMEM, Q MN-major)
//                 dQ_i = dS_i K         -> TMEM DP   (dS and K read MN-major)
//                 dP^T_{i+1} = V dO_{i+1}^T          -> TMEM DP, once the dQ
//                                                       warps have read dQ_i
//               The MMAs of a CTA run in issue order, so S^T_{i+1} never
//               overwrites P_i^T before dV has read it, and dQ_i never
//               overwrites dS_i^T before dK has read it;
//   warps 2..9  two per key row group (TMEM lane quarter), each half of the
//               tile's 128 queries: P^T = exp2(S^T sl2 - lse2) written back
//               as bf16 over its own first scores; then dS^T = P^T (dP^T - D)
//               as bf16 over its own first dP^T columns and into the shared
//               dS tile the dQ product reads; at the end dV (warps 2..5) and
//               dK (warps 6..9) rows to global memory;
//   warps 10..13 one query row each: the tile's dQ rows leave TMEM through
//               the shared dS tile (free once the dQ product has read it),
//               staged as fp32 boxes of 32 queries x 32 dims with the 128-byte
//               swizzle, and are added into dq by TMA bulk reductions
//               (cp.reduce.async.bulk.tensor ... .add): the sums happen in L2
//               on whole lines, with no per-thread atomics.
// TMEM columns: dV [0,128), dK [128,256), S^T/P^T [256,384), dP^T/dS^T and
// dQ [384,512).  All mbarrier waits are bounded; on a timeout every role
// drains its in-flight copies and MMAs before TMEM is released.
constexpr int BQB = 128;                 // query tile of the backward
constexpr int B_OFF_K = 0;
constexpr int B_OFF_V = B_OFF_K + TILE;
constexpr int B_OFF_Q = B_OFF_V + TILE;       // 2 stages
constexpr int B_OFF_DO = B_OFF_Q + 2 * TILE;  // 2 stages
constexpr int B_OFF_DS = B_OFF_DO + 2 * TILE; // [2 query halves][128 keys][64 queries] bf16
constexpr int B_OFF_LQ = B_OFF_DS + TILE;     // [2 stages][128] lse * log2(e)
constexpr int B_OFF_LD = B_OFF_LQ + 2 * BQB * 4;  // [2 stages][128] D
constexpr int B_OFF_BAR = B_OFF_LD + 2 * BQB * 4;
constexpr int kBwdSmem = B_OFF_BAR + 256;
static_assert(kBwdSmem <= 232448, "attention backward shared memory budget");
constexpr int kBwdThreads = 448;
constexpr uint32_t TB_DV = 0, TB_DK = 128, TB_S = 256, TB_DP = 384;

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
  int B;
  // Persistent key-side kernel: dK leaves through the backward of the k-side
  // RoPE + QK-norm (the forward applies them in the q|k|v projection's
  // epilogue), using the saved normalised k (the K operand itself), rstd_k
  // [B*T, Hkv] and the cos/sin table (rope_table()'s buffer).
  const float2* rope_tab;
  int rope_T;  // positions of the table (its grouped copy starts at rope_tab + rope_T * 64)
  const float* rstd_k;
  int Hkv;
};

// GW: grouped KV heads or a window in play; the plain instance compiles
// with group 1 and no window as constants (its tile t is query tile i0 + t
// of head hk).  This form computes dQ itself (fp32, TMA bulk reductions);
// the model's backward uses the persistent key-side kernel and the dQ
// kernel instead.
template <bool GW>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                       const __grid_constant__ CUtensorMap tdq, const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((tc::smem_u32(smem_raw) & 1023u) != 0) {  // never expected; no room to realign
    if (threadIdx.x == 0 && a.status) atomicExch(a.status, kDevTimeout);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + B_OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;    // [2]
  uint64_t* q_empty = bars + 3;   // [2]
  uint64_t* do_full = bars + 5;   // [2]
  uint64_t* do_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;
  uint64_t* p_full = bars + 10;
  uint64_t* dp_full = bars + 11;
  uint64_t* ds_full = bars + 12;
  uint64_t* ds_empty = bars + 13;
  uint64_t* dq_full = bars + 14;
  uint64_t* dq_empty = bars + 15;
  uint64_t* dkv_full = bars + 16;
  uint64_t* drained = bars + 17;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;  // hk: the KV head
  const int group = GW ? a.group : 1;
  const int window = GW ? a.window : -1;
  const int i0 = kb;  // BQB == BKV: the first query tile that reaches these keys
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
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&q_full[i], 32);  // the TMA lane (with its bytes) + 31 staging lanes
      tc::mbar_init(&q_empty[i], 1);
      tc::mbar_init(&do_full[i], 32);
      tc::mbar_init(&do_empty[i], 1);
    }
    tc::mbar_init(s_full, 1);
    tc::mbar_init(p_full, 256);
    tc::mbar_init(dp_full, 1);
    tc::mbar_init(ds_full, 256);
    // One lane of each dQ warp once its staging is read.
    tc::mbar_init(ds_empty, 4);
    tc::mbar_init(dq_full, 1);
    tc::mbar_init(dq_empty, 128);
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
    // Lane 0 issues the TMA copies; all 32 lanes stage lse * log2(e) (with Q)
    // and D (with dO) of the query tile and arrive on the same barriers.
    if (lane == 0) {
      tc::tma_prefetch_desc(&tq);
      tc::tma_prefetch_desc(&tk);
      tc::tma_prefetch_desc(&tv);
      tc::tma_prefetch_desc(&tdo);
      tc::tma_prefetch_desc(&tdq);
      tc::mbar_arrive_expect_tx(kv_full, 2 * TILE);
      for (int c = 0; c < 2; ++c) {
        tc::tma_load_3d(smem + B_OFF_K + c * (TILE / 2), &tk, kv_full, kcol0 + 64 * c, kb * BKV, b);
        tc::tma_load_3d(smem + B_OFF_V + c * (TILE / 2), &tv, kv_full, kcol0 + 64 * c, kb * BKV, b);
      }
    }
    int issued_q = 0, issued_do = 0;
    bool ok = true;
    for (int t = 0; t < nblk; ++t) {
      const int st = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      const int hq = GW ? hk * group + t / nqt : hk;
      const int q0 = (i0 + (GW ? t % nqt : t)) * BQB;
      const int qcol0 = hq * HD;
      bool w = true;
      if (lane == 0) w = tc::mbar_wait(&q_empty[st], ph ^ 1, abort_flag, a.status);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) { ok = false; break; }
      const float* lse_bh = a.lse + ((int64_t)b * a.H + hq) * a.T;
      float* lq = reinterpret_cast<float*>(smem + B_OFF_LQ) + st * BQB;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = q0 + lane + 32 * u;
        lq[lane + 32 * u] = q < a.T ? lse_bh[q] * 1.4426950408889634f : INFINITY;
      }
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&q_full[st], TILE);
        for (int c = 0; c < 2; ++c)
          tc::tma_load_3d(smem + B_OFF_Q + st * TILE + c * (TILE / 2), &tq, &q_full[st], qcol0 + 64 * c, q0, b);
      } else {
        tc::mbar_arrive(&q_full[st]);
      }
      ++issued_q;
      if (lane == 0) w = tc::mbar_wait(&do_empty[st], ph ^ 1, abort_flag, a.status);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) { ok = false; break; }
      const float* d_bh = a.delta + ((int64_t)b * a.H + hq) * a.T;
      float* ldd = reinterpret_cast<float*>(smem + B_OFF_LD) + st * BQB;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = q0 + lane + 32 * u;
        ldd[lane + 32 * u] = q < a.T ? d_bh[q] : 0.f;
      }
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&do_full[st], TILE);
        for (int c = 0; c < 2; ++c)
          tc::tma_load_3d(smem + B_OFF_DO + st * TILE + c * (TILE / 2), &tdo, &do_full[st], qcol0 + 64 * c, q0, b);
      } else {
        tc::mbar_arrive(&do_full[st]);
      }
      ++issued_do;
    }
    if (!ok && lane == 0) {
      drain_wait(kv_full, 0);
      for (int t = max(0, issued_q - 2); t < issued_q; ++t) drain_wait(&q_full[t & 1], (t >> 1) & 1);
      for (int t = max(0, issued_do - 2); t < issued_do; ++t) drain_wait(&do_full[t & 1], (t >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_ss = tc::idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
      const uint32_t id_ts = tc::idesc_bf16_f32(128, 128, 0, 1);  // dV, dK: A from TMEM
      const uint32_t id_dq = tc::idesc_bf16_f32(128, 128, 1, 1);  // dQ: both MN-major
      // Descriptors are built once; each MMA adds a constant byte offset.
      const uint64_t kK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_K), 16, 1024);
      const uint64_t vK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_V), 16, 1024);
      const uint64_t kMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_K), TILE / 2, 1024);
      const uint64_t qK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_Q), 16, 1024);
      const uint64_t doK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DO), 16, 1024);
      const uint64_t qMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_Q), TILE / 2, 1024);
      const uint64_t doMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DO), TILE / 2, 1024);
      const uint64_t dsMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DS), TILE / 2, 1024);
      bool ok = tc::mbar_wait(kv_full, 0, abort_flag, a.status);
      // S^T of tile t once its Q has landed; the S columns are free because
      // every earlier MMA that reads them (dV of tile t - 1) was issued first.
      auto issue_s = [&](int t) -> bool {
        const int st = t & 1;
        if (!tc::mbar_wait(&q_full[st], (t >> 1) & 1, abort_flag, a.status)) return false;
        tc::tc_fence_after();
        const uint64_t qd = tc::desc_add(qK, st * TILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
          tc::umma_bf16_ss(tmem + TB_S, tc::desc_add(kK, off), tc::desc_add(qd, off), id_ss,
                           kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(s_full);
        return true;
      };
      // dP^T of tile t once its dO has landed (the DP columns are free: the
      // dQ warps have read the previous tile's dQ).
      auto issue_dp = [&](int t) -> bool {
        const int st = t & 1;
        if (!tc::mbar_wait(&do_full[st], (t >> 1) & 1, abort_flag, a.status)) return false;
        tc::tc_fence_after();
        const uint64_t dod = tc::desc_add(doK, st * TILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
          tc::umma_bf16_ss(tmem + TB_DP, tc::desc_add(vK, off), tc::desc_add(dod, off), id_ss,
                           kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(dp_full);
        return true;
      };
      if (ok) ok = issue_s(0) && issue_dp(0);
      for (int t = 0; t < nblk && ok; ++t) {
        const int st = t & 1;
        if (!tc::mbar_wait(p_full, t & 1, abort_flag, a.status)) { ok = false; break; }
        tc::tc_fence_after();
        // dV += P^T dO: query step kk (16 queries) is 8 packed columns of the
        // softmax half that owns it (half h at column 64 h).
        const uint64_t domn = tc::desc_add(doMN, st * TILE);
#pragma unroll
        for (int kk = 0; kk < BQB / 16; ++kk)
          tc::umma_bf16_ts(tmem + TB_DV, tmem + TB_S + (kk >> 2) * 64 + (kk & 3) * 8,
                           tc::desc_add(domn, kk * 2048), id_ts, (t > 0 || kk > 0) ? 1u : 0u);
        tc::umma_commit(&do_empty[st]);
        if (t + 1 < nblk && !issue_s(t + 1)) { ok = false; break; }
        if (!tc::mbar_wait(ds_full, t & 1, abort_flag, a.status)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t qmn = tc::desc_add(qMN, st * TILE);
#pragma unroll
        for (int kk = 0; kk < BQB / 16; ++kk)
          tc::umma_bf16_ts(tmem + TB_DK, tmem + TB_DP + (kk >> 2) * 64 + (kk & 3) * 8,
                           tc::desc_add(qmn, kk * 2048), id_ts, (t > 0 || kk > 0) ? 1u : 0u);
        tc::umma_commit(&q_empty[st]);
        // dQ = dS K (one query per TMEM lane): key step kk (16 keys) is 2 KB
        // into both MN-major tiles.
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          tc::umma_bf16_ss(tmem + TB_DP, tc::desc_add(dsMN, kk * 2048),
                           tc::desc_add(kMN, kk * 2048), id_dq, kk > 0 ? 1u : 0u);
        tc::umma_commit(dq_full);
        if (t + 1 < nblk) {
          if (!tc::mbar_wait(dq_empty, t & 1, abort_flag, a.status)) { ok = false; break; }
          tc::tc_fence_after();
          if (!issue_dp(t + 1)) { ok = false; break; }
        }
      }
      if (ok) tc::umma_commit(dkv_full);
      tc::umma_commit(drained);
      drain_wait(drained, 0);
    }
  } else if (warp < 10) {
    // ---------------- P^T and dS^T: one key row per thread, half the queries per warp
    const int qw = warp & 3;
    const int hf = (warp - 2) >> 2;  // query half: [64 hf, 64 hf + 64) of the tile
    const int row = qw * 32 + lane;
    const int key = kb * BKV + row;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t s_col = lane_base + TB_S + 64 * hf;
    const uint32_t dp_col = lane_base + TB_DP + 64 * hf;
    const uint32_t ds_row = tc::smem_u32(smem + B_OFF_DS) + hf * (TILE / 2) + row * 128;
    bool ok = true;
    for (int t = 0; t < nblk; ++t) {
      const int st = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      const int qh = (i0 + (GW ? t % nqt : t)) * BQB + 64 * hf;  // first query of this half
      ok = tc::mbar_wait(s_full, t & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc::tc_fence_after();
      // The tile's lse, staged by the TMA warp and published by the stage's
      // q_full barrier (already complete: the scores came from it).
      ok = tc::mbar_wait(&q_full[st], ph, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const float* lq = reinterpret_cast<const float*>(smem + B_OFF_LQ) + st * BQB + 64 * hf;
      // The half reaches the diagonal, T, or past the window of this key.
      const bool edge = (qh < key) || (qh + 63 >= a.T) || (key >= a.T) ||
                        (window >= 0 && qh + 63 > key + window);
      uint32_t pk[2][16];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sv[32];
        tc::tmem_ld_32x32b_x32(s_col + 32 * c, sv);
        // The chunk's 32 lse values as eight 16-byte shared loads, issued
        // while the scores are in flight.
        float l[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 v = reinterpret_cast<const float4*>(lq + 32 * c)[u];
          l[4 * u] = v.x;
          l[4 * u + 1] = v.y;
          l[4 * u + 2] = v.z;
          l[4 * u + 3] = v.w;
        }
        tc::tmem_ld_wait();
        // Every argument first, then the 32 independent exponentials.
        float p[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) p[i] = fmaf(__uint_as_float(sv[i]), a.sl2, -l[i]);
#pragma unroll
        for (int i = 0; i < 32; ++i) p[i] = ex2(p[i]);
        if (edge) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int qa = qh + 32 * c + i;
            if (qa < key || qa >= a.T || key >= a.T || (window >= 0 && qa > key + window)) p[i] = 0.f;
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[c][i] = pack_bf16x2(p[2 * i], p[2 * i + 1]);
      }
      tc::tmem_st_32x32b_x16(s_col, pk[0]);
      tc::tmem_st_32x32b_x16(s_col + 16, pk[1]);
      tc::tmem_st_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(p_full);
      // dS^T = P^T (dP^T - D), from the bf16 P the dV product reads.
      ok = tc::mbar_wait(dp_full, t & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc::tc_fence_after();
      ok = tc::mbar_wait(&do_full[st], ph, abort_flag, a.status);  // D, staged with dO
      // The shared dS tile is free once the previous tile's dQ product is done.
      ok = ok && tc::mbar_wait(ds_empty, (t & 1) ^ 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const float* ld = reinterpret_cast<const float*>(smem + B_OFF_LD) + st * BQB + 64 * hf;
      // 32 queries at a time: chunk c's dS^T goes over the dP^T columns of
      // queries [16 c, 16 c + 16), which chunk 0 has already read.
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dpv[32];
        tc::tmem_ld_32x32b_x32(dp_col + 32 * c, dpv);
        float dl[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 v = reinterpret_cast<const float4*>(ld + 32 * c)[u];
          dl[4 * u] = v.x;
          dl[4 * u + 1] = v.y;
          dl[4 * u + 2] = v.z;
          dl[4 * u + 3] = v.w;
        }
        tc::tmem_ld_wait();
        uint32_t pd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 p = unpack_bf16x2(pk[c][i]);
          const float d0 = p.x * (__uint_as_float(dpv[2 * i]) - dl[2 * i]);
          const float d1 = p.y * (__uint_as_float(dpv[2 * i + 1]) - dl[2 * i + 1]);
          pd[i] = pack_bf16x2(d0, d1);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t sw = (uint32_t)(((4 * c + u) ^ (row & 7)) << 4);
          tc::st_shared_v4(ds_row + sw, pd[4 * u], pd[4 * u + 1], pd[4 * u + 2], pd[4 * u + 3]);
        }
        tc::tmem_st_32x32b_x16(dp_col + 16 * c, pd);
      }
      tc::tmem_st_wait();
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(ds_full);
    }
    if (ok) {
      ok = tc::mbar_wait(dkv_full, 0, abort_flag, a.status);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      // Warps of query half 0 write dV rows, those of half 1 dK rows.
      tc::tc_fence_after();
      const int64_t grow = ((int64_t)b * a.T + key) * a.ldg + kcol0;
      const uint32_t base = lane_base + (hf ? TB_DK : TB_DV);
      const float mul = hf ? a.scale : 1.f;
      __nv_bfloat16* dst = (hf ? a.dk : a.dv) + grow;
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
    // ---------------- dQ rows: one query per thread, TMA bulk reductions into dq
    const int qw = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    // This warp's 8 KB of the dS tile: its 32 queries x 64 dims as two
    // swizzled 32 x 32 fp32 boxes.
    const uint32_t slot = tc::smem_u32(smem + B_OFF_DS) + qw * 8192;
    bool pending = false;  // this warp has bulk reductions in flight
    for (int t = 0; t < nblk; ++t) {
      const int q0 = (i0 + (GW ? t % nqt : t)) * BQB + 32 * qw;
      const int dcol = (GW ? hk * group + t / nqt : hk) * HD;
      bool ok = tc::mbar_wait(dq_full, t & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {  // dims [64 hh, 64 hh + 64)
        uint32_t v[2][32];
        tc::tmem_ld_32x32b_x32(lane_base + TB_DP + 64 * hh, v[0]);
        tc::tmem_ld_32x32b_x32(lane_base + TB_DP + 64 * hh + 32, v[1]);
        tc::tmem_ld_wait();
        if (hh == 1) {  // every dQ column read: the MMA warp may reuse them
          tc::tc_fence_before();
          tc::mbar_arrive(dq_empty);
        }
        if (hh == 1 && lane == 0) tc::bulk_wait_group_read0();  // the first half's boxes are read
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int u = 0; u < 8; ++u)
            tc::st_shared_v4(slot + c * 4096 + lane * 128 + ((u ^ (lane & 7)) << 4),
                             __float_as_uint(__uint_as_float(v[c][4 * u]) * a.scale),
                             __float_as_uint(__uint_as_float(v[c][4 * u + 1]) * a.scale),
                             __float_as_uint(__uint_as_float(v[c][4 * u + 2]) * a.scale),
                             __float_as_uint(__uint_as_float(v[c][4 * u + 3]) * a.scale));
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int c = 0; c < 2; ++c)
            tc::tma_reduce_add_3d(&tdq, slot + c * 4096, dcol + 64 * hh + 32 * c, q0, b);
          tc::bulk_commit_group();
        }
      }
      pending = true;
      // The dS tile is the next tile's again once these boxes are read.
      if (lane == 0) {
        tc::bulk_wait_group_read0();
        tc::mbar_arrive(ds_empty);
      }
      __syncwarp();
    }
    if (pending && lane == 0) tc::bulk_wait_group0();
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}


// ------------------------------------------------------------------ key side, persistent
// The key-side backward of the split form as a persistent kernel: one CTA
// per SM walks work items (128-key tile, KV head, batch row) in balanced
// pairs (KvCursor).  Per item it accumulates dV and dK in TMEM
// over the query tiles (and query heads of the KV head's group) that reach
// its keys, exactly as the one-item-per-CTA form does, and stores every dS^T
// tile for the query-side kernel; in addition the tile pipeline runs on
// across item boundaries:
//   * K and V of the next item are loaded as soon as the MMAs that read the
//     current ones (the item's last S^T and dP^T) are done, so the next
//     item's first scores follow the current item's last ones directly;
//   * the dV / dK epilogue (k-side RoPE + QK-norm backward included) runs on
//     warps of its own while the next item's tiles are processed; the MMA
//     warp only waits for it before the next item's first dV and dK
//     products, which overwrite the accumulators.
// 512 threads (128 registers each), four warps per role group so that each
// group's warps cover the four TMEM lane quarters:
//   warp 0      TMA: K and V per item, Q_i and dO_i of every tile (two stages
//               each), lse * log2(e) and D staged by all its lanes;
//   warp 1      TMEM owner and single-thread MMA issue (products as in the
//               one-item-per-CTA form);
//   warp 2      one lane stores each dS^T tile (TMA) once the softmax warps
//               have written it to shared memory; warp 3 idles;
//   warps 4..11 P^T and dS^T, two threads per key row;
//   warps 12..15 epilogue, one key row per thread: the row of yhat (the
//               normalised k, the K operand itself) is copied from shared
//               memory into registers while the item runs, so K's buffer
//               can take the next item; at the item's end dV goes out, then
//               dK through dr = r (g - yhat mean(g yhat)), dk = R(-theta) dr.
constexpr int kKvThreads = 512;
constexpr int KV_OFF_TI = B_OFF_BAR;        // [2 stages] (first query, key tile) of the tile
constexpr int KV_OFF_BAR = KV_OFF_TI + 64;
constexpr int kKvSmem = KV_OFF_BAR + 256;
static_assert(kKvSmem <= 232448, "persistent key-side shared memory budget");

// Work item: key tile, KV head, batch row, and its tile count.
struct KvItem {
  int kb, hk, b, nqt, nblk;
};

// This CTA's work items in order.  Items come in pairs of one (KV head,
// row): key tile j, then key tile nkb - 1 - j.  Under the causal mask the
// pair's tile counts add up to nqb + 1 whatever j is, so dealing pair p to
// CTA p mod gridDim.x balances the work; the pairs of one (KV head, row) are
// consecutive, so the CTAs working at the same time read the same Q and dO
// tiles, which then come from L2.  t is the tile of the current item and n
// counts the items walked.
struct KvCursor {
  int p, sub, n, t;
  bool valid;
  KvItem m;
  __device__ __forceinline__ void load(const BwdArgs& a, int npairs, int group, int window) {
    valid = p < npairs;
    if (!valid) return;
    const int ppg = (a.nkb + 1) / 2;
    const int grp = p / ppg;
    const int j = p - grp * ppg;
    m.kb = sub ? a.nkb - 1 - j : j;
    m.hk = grp % a.Hkv;
    m.b = grp / a.Hkv;
    const int i_hi = window < 0 ? a.nqb - 1 : min(a.nqb - 1, (m.kb * BKV + BKV - 1 + window) / BQB);
    m.nqt = i_hi - m.kb + 1;
    m.nblk = group * m.nqt;
  }
  __device__ __forceinline__ void start(const BwdArgs& a, int npairs, int group, int window) {
    p = blockIdx.x;
    sub = 0;
    n = 0;
    t = 0;
    load(a, npairs, group, window);
  }
  __device__ __forceinline__ void next_item(const BwdArgs& a, int npairs, int group, int window) {
    const int j = p % ((a.nkb + 1) / 2);
    if (sub == 0 && a.nkb - 1 - j != j) {
      sub = 1;
    } else {
      sub = 0;
      p += gridDim.x;
    }
    ++n;
    t = 0;
    load(a, npairs, group, window);
  }
  __device__ __forceinline__ void next(const BwdArgs& a, int npairs, int group, int window) {
    if (++t == m.nblk) next_item(a, npairs, group, window);
  }
  // Query head and first query of the current tile.
  __device__ __forceinline__ int hq(int group) const { return m.hk * group + t / m.nqt; }
  __device__ __forceinline__ int q0() const { return (m.kb + t % m.nqt) * BQB; }
};

// Tiles of all this CTA's items.
__device__ __forceinline__ int kv_tiles_total(const BwdArgs& a, int npairs, int group, int window) {
  KvCursor c;
  int total = 0;
  for (c.start(a, npairs, group, window); c.valid; c.next_item(a, npairs, group, window)) total += c.m.nblk;
  return total;
}

template <bool GW>
__global__ void __launch_bounds__(kKvThreads)
    attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                       const __grid_constant__ CUtensorMap tds, const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((tc::smem_u32(smem_raw) & 1023u) != 0) {  // never expected; no room to realign
    if (threadIdx.x == 0 && a.status) atomicExch(a.status, kDevTimeout);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + KV_OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;   // the item's MMAs have read K and V
  uint64_t* k_copied = bars + 2;   // the epilogue has copied its yhat rows
  uint64_t* q_full = bars + 3;     // [2]
  uint64_t* q_empty = bars + 5;    // [2]
  uint64_t* do_full = bars + 7;    // [2]
  uint64_t* do_empty = bars + 9;   // [2]
  uint64_t* s_full = bars + 11;
  uint64_t* p_full = bars + 12;
  uint64_t* dp_full = bars + 13;
  uint64_t* ds_full = bars + 14;
  uint64_t* ds_empty = bars + 15;
  uint64_t* dkv_full = bars + 16;  // the item's dV and dK are final
  uint64_t* dv_empty = bars + 17;  // the epilogue has read dV
  uint64_t* dk_empty = bars + 18;  // ... and dK
  uint64_t* drained = bars + 19;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int group = GW ? a.group : 1;
  const int window = GW ? a.window : -1;
  const int npairs = (a.nkb + 1) / 2 * a.Hkv * a.B;

  if (threadIdx.x == 0) {
    tc::mbar_init(kv_full, 1);
    tc::mbar_init(kv_empty, 1);
    tc::mbar_init(k_copied, 128);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&q_full[i], 32);  // the TMA lane (with its bytes) + 31 staging lanes
      tc::mbar_init(&q_empty[i], 1);
      tc::mbar_init(&do_full[i], 32);
      tc::mbar_init(&do_empty[i], 1);
    }
    tc::mbar_init(s_full, 1);
    tc::mbar_init(p_full, 256);
    tc::mbar_init(dp_full, 1);
    tc::mbar_init(ds_full, 256);
    tc::mbar_init(ds_empty, 1);
    tc::mbar_init(dkv_full, 1);
    tc::mbar_init(dv_empty, 128);
    tc::mbar_init(dk_empty, 128);
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
    // Lane 0 issues the TMA copies; all 32 lanes stage lse * log2(e) (with Q)
    // and D (with dO) of the query tile and arrive on the same barriers.
    if (lane == 0) {
      tc::tma_prefetch_desc(&tq);
      tc::tma_prefetch_desc(&tk);
      tc::tma_prefetch_desc(&tv);
      tc::tma_prefetch_desc(&tdo);
      tc::tma_prefetch_desc(&tds);
    }
    KvCursor c;
    c.start(a, npairs, group, window);
    int issued_q = 0, issued_do = 0, issued_kv = 0;
    bool ok = true;
    for (int g = 0; c.valid; ++g) {
      const int st = g & 1;
      const uint32_t ph = (g >> 1) & 1;
      bool w = true;
      if (c.t == 0) {
        // K and V of the item, once the previous item's MMAs have read them.
        if (lane == 0 && c.n > 0)
          w = tc::mbar_wait(kv_empty, (c.n - 1) & 1, abort_flag, a.status) &&
              tc::mbar_wait(k_copied, (c.n - 1) & 1, abort_flag, a.status);
        if (!__shfl_sync(0xffffffffu, (int)w, 0)) { ok = false; break; }
        if (lane == 0) {
          tc::mbar_arrive_expect_tx(kv_full, 2 * TILE);
          for (int h = 0; h < 2; ++h) {
            tc::tma_load_3d(smem + B_OFF_K + h * (TILE / 2), &tk, kv_full, c.m.hk * HD + 64 * h,
                            c.m.kb * BKV, c.m.b);
            tc::tma_load_3d(smem + B_OFF_V + h * (TILE / 2), &tv, kv_full, c.m.hk * HD + 64 * h,
                            c.m.kb * BKV, c.m.b);
          }
        }
        ++issued_kv;
      }
      const int hq = GW ? c.hq(group) : c.m.hk;
      const int q0 = GW ? c.q0() : (c.m.kb + c.t) * BQB;
      const int qcol0 = hq * HD;
      if (lane == 0) w = tc::mbar_wait(&q_empty[st], ph ^ 1, abort_flag, a.status);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) { ok = false; break; }
      const float* lse_bh = a.lse + ((int64_t)c.m.b * a.H + hq) * a.T;
      float* lq = reinterpret_cast<float*>(smem + B_OFF_LQ) + st * BQB;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = q0 + lane + 32 * u;
        lq[lane + 32 * u] = q < a.T ? -lse_bh[q] * 1.4426950408889634f : -INFINITY;  // negated
      }
      if (lane == 0) {
        reinterpret_cast<int2*>(smem + KV_OFF_TI)[st] = make_int2(q0, c.m.kb);
        tc::mbar_arrive_expect_tx(&q_full[st], TILE);
        for (int h = 0; h < 2; ++h)
          tc::tma_load_3d(smem + B_OFF_Q + st * TILE + h * (TILE / 2), &tq, &q_full[st], qcol0 + 64 * h,
                          q0, c.m.b);
      } else {
        tc::mbar_arrive(&q_full[st]);
      }
      ++issued_q;
      if (lane == 0) w = tc::mbar_wait(&do_empty[st], ph ^ 1, abort_flag, a.status);
      if (!__shfl_sync(0xffffffffu, (int)w, 0)) { ok = false; break; }
      const float* d_bh = a.delta + ((int64_t)c.m.b * a.H + hq) * a.T;
      float* ldd = reinterpret_cast<float*>(smem + B_OFF_LD) + st * BQB;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = q0 + lane + 32 * u;
        ldd[lane + 32 * u] = q < a.T ? -d_bh[q] : 0.f;  // negated
      }
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&do_full[st], TILE);
        for (int h = 0; h < 2; ++h)
          tc::tma_load_3d(smem + B_OFF_DO + st * TILE + h * (TILE / 2), &tdo, &do_full[st],
                          qcol0 + 64 * h, q0, c.m.b);
      } else {
        tc::mbar_arrive(&do_full[st]);
      }
      ++issued_do;
      c.next(a, npairs, group, window);
    }
    if (!ok && lane == 0) {
      if (issued_kv > 0) drain_wait(kv_full, (issued_kv - 1) & 1);
      for (int t = max(0, issued_q - 2); t < issued_q; ++t) drain_wait(&q_full[t & 1], (t >> 1) & 1);
      for (int t = max(0, issued_do - 2); t < issued_do; ++t) drain_wait(&do_full[t & 1], (t >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_ss = tc::idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
      const uint32_t id_ts = tc::idesc_bf16_f32(128, 128, 0, 1);  // dV, dK: A from TMEM
      const uint64_t kK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_K), 16, 1024);
      const uint64_t vK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_V), 16, 1024);
      const uint64_t qK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_Q), 16, 1024);
      const uint64_t doK = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DO), 16, 1024);
      const uint64_t qMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_Q), TILE / 2, 1024);
      const uint64_t doMN = tc::smem_desc_sw128(tc::smem_u32(smem + B_OFF_DO), TILE / 2, 1024);
      // S^T of tile g once its Q has landed; the S columns are free because
      // every earlier MMA that reads them (dV of tile g - 1) was issued first.
      auto issue_s = [&](int g) -> bool {
        const int st = g & 1;
        if (!tc::mbar_wait(&q_full[st], (g >> 1) & 1, abort_flag, a.status)) return false;
        tc::tc_fence_after();
        const uint64_t qd = tc::desc_add(qK, st * TILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
          tc::umma_bf16_ss(tmem + TB_S, tc::desc_add(kK, off), tc::desc_add(qd, off), id_ss,
                           kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(s_full);
        return true;
      };
      // dP^T of tile g once its dO has landed (the DP columns are free: dK of
      // tile g - 1, which reads dS^T from them, was issued first).
      auto issue_dp = [&](int g) -> bool {
        const int st = g & 1;
        if (!tc::mbar_wait(&do_full[st], (g >> 1) & 1, abort_flag, a.status)) return false;
        tc::tc_fence_after();
        const uint64_t dod = tc::desc_add(doK, st * TILE);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (TILE / 2) + (kk & 3) * 32;
          tc::umma_bf16_ss(tmem + TB_DP, tc::desc_add(vK, off), tc::desc_add(dod, off), id_ss,
                           kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(dp_full);
        return true;
      };
      KvCursor c, nx;
      c.start(a, npairs, group, window);
      bool ok = c.valid && tc::mbar_wait(kv_full, 0, abort_flag, a.status);
      if (ok) ok = issue_s(0) && issue_dp(0);
      // The item's last S^T and dP^T have been issued: K and V are free once
      // they complete.
      if (ok && c.m.nblk == 1) tc::umma_commit(kv_empty);
      for (int g = 0; c.valid && ok; ++g) {
        const int st = g & 1;
        nx = c;
        nx.next(a, npairs, group, window);
        if (!tc::mbar_wait(p_full, g & 1, abort_flag, a.status)) { ok = false; break; }
        // The first product of an item overwrites dV: the epilogue must have
        // read the previous item's.
        if (c.t == 0 && c.n > 0 && !tc::mbar_wait(dv_empty, (c.n - 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        // dV += P^T dO: query step kk (16 queries) is 8 packed columns of the
        // softmax half that owns it (half h at column 64 h).
        const uint64_t domn = tc::desc_add(doMN, st * TILE);
#pragma unroll
        for (int kk = 0; kk < BQB / 16; ++kk)
          tc::umma_bf16_ts(tmem + TB_DV, tmem + TB_S + (kk >> 2) * 64 + (kk & 3) * 8,
                           tc::desc_add(domn, kk * 2048), id_ts, (c.t > 0 || kk > 0) ? 1u : 0u);
        tc::umma_commit(&do_empty[st]);
        if (nx.valid) {
          if (nx.t == 0 && !tc::mbar_wait(kv_full, nx.n & 1, abort_flag, a.status)) { ok = false; break; }
          if (!issue_s(g + 1)) { ok = false; break; }
        }
        if (!tc::mbar_wait(ds_full, g & 1, abort_flag, a.status)) { ok = false; break; }
        if (c.t == 0 && c.n > 0 && !tc::mbar_wait(dk_empty, (c.n - 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint64_t qmn = tc::desc_add(qMN, st * TILE);
#pragma unroll
        for (int kk = 0; kk < BQB / 16; ++kk)
          tc::umma_bf16_ts(tmem + TB_DK, tmem + TB_DP + (kk >> 2) * 64 + (kk & 3) * 8,
                           tc::desc_add(qmn, kk * 2048), id_ts, (c.t > 0 || kk > 0) ? 1u : 0u);
        tc::umma_commit(&q_empty[st]);
        if (c.t == c.m.nblk - 1) tc::umma_commit(dkv_full);
        if (nx.valid) {
          if (!issue_dp(g + 1)) { ok = false; break; }
          if (nx.t == nx.m.nblk - 1) tc::umma_commit(kv_empty);
        }
        c = nx;
      }
      tc::umma_commit(drained);
      drain_wait(drained, 0);
    }
  } else if (warp == 2) {
    // ---------------- dS^T tiles to global memory (one lane of warp 2)
    if (lane == 0) {
      KvCursor c;
      c.start(a, npairs, group, window);
      bool pending = false;
      for (int g = 0; c.valid; ++g, c.next(a, npairs, group, window)) {
        const int q0 = GW ? c.q0() : (c.m.kb + c.t) * BQB;
        const int hq = GW ? c.hq(group) : c.m.hk;
        if (!tc::mbar_wait(ds_full, g & 1, abort_flag, a.status)) break;
        for (int h = 0; h < 2; ++h)
          tc::tma_store_3d(&tds, tc::smem_u32(smem + B_OFF_DS) + h * (TILE / 2), q0 + 64 * h,
                           c.m.kb * BKV, c.m.b * a.H + hq);
        tc::bulk_commit_group();
        pending = true;
        tc::bulk_wait_group_read0();  // the tile may be rewritten once read
        tc::mbar_arrive(ds_empty);
      }
      if (pending) tc::bulk_wait_group0();
    }
  } else if (warp < 4) {
    // warp 3: no role
  } else if (warp < 12) {
    // ---------------- P^T and dS^T: one key row per thread, half the queries per warp
    const int qw = warp & 3;
    const int hf = (warp - 4) >> 2;  // query half: [64 hf, 64 hf + 64) of the tile
    const int row = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    const uint32_t s_col = lane_base + TB_S + 64 * hf;
    const uint32_t dp_col = lane_base + TB_DP + 64 * hf;
    const uint32_t ds_row = tc::smem_u32(smem + B_OFF_DS) + hf * (TILE / 2) + row * 128;
    const int total = kv_tiles_total(a, npairs, group, window);
    for (int g = 0; g < total; ++g) {
      const int st = g & 1;
      const uint32_t ph = (g >> 1) & 1;
      bool ok = tc::mbar_wait(s_full, g & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::tc_fence_after();
      // The tile's lse and coordinates, staged by the TMA warp and published
      // by the stage's q_full barrier (already complete: the scores came
      // from it).
      ok = tc::mbar_wait(&q_full[st], ph, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int2 ti = reinterpret_cast<const int2*>(smem + KV_OFF_TI)[st];
      const int key = ti.y * BKV + row;
      const int qh = ti.x + 64 * hf;  // first query of this half
      const float* lq = reinterpret_cast<const float*>(smem + B_OFF_LQ) + st * BQB + 64 * hf;
      // The half reaches the diagonal, T, or past the window of this key.
      const bool edge = (qh < key) || (qh + 63 >= a.T) || (key >= a.T) ||
                        (window >= 0 && qh + 63 > key + window);
      uint32_t pk[2][16];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t sv[32];
        tc::tmem_ld_32x32b_x32(s_col + 32 * cc, sv);
        // The chunk's 32 lse values as eight 16-byte shared loads, issued
        // while the scores are in flight.
        float l[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 v = reinterpret_cast<const float4*>(lq + 32 * cc)[u];
          l[4 * u] = v.x;
          l[4 * u + 1] = v.y;
          l[4 * u + 2] = v.z;
          l[4 * u + 3] = v.w;
        }
        tc::tmem_ld_wait();
        // Every argument first (packed fp32 pairs, the same rounding as scalar
        // fma; l holds -lse log2(e)), then the 32 independent exponentials.
        float p[32];
        const float2 sl2v = make_float2(a.sl2, a.sl2);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), sl2v,
                                      make_float2(l[i], l[i + 1]));
          p[i] = x.x;
          p[i + 1] = x.y;
        }
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          if (poly_pair(i / 2)) {
            const float2 e = exp2_fma2(make_float2(p[i], p[i + 1]));
            p[i] = e.x;
            p[i + 1] = e.y;
          } else {
            p[i] = ex2(p[i]);
            p[i + 1] = ex2(p[i + 1]);
          }
        }
        if (edge) {  // masked scores (exp2_fma2 leaves them near 2^-125) become 0
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int qa = qh + 32 * cc + i;
            if (qa < key || qa >= a.T || key >= a.T || (window >= 0 && qa > key + window)) p[i] = 0.f;
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[cc][i] = pack_bf16x2(p[2 * i], p[2 * i + 1]);
      }
      tc::tmem_st_32x32b_x16(s_col, pk[0]);
      tc::tmem_st_32x32b_x16(s_col + 16, pk[1]);
      tc::tmem_st_wait();
      tc::tc_fence_before();
      tc::mbar_arrive(p_full);
      // dS^T = P^T (dP^T - D), from the bf16 P the dV product reads.
      ok = tc::mbar_wait(dp_full, g & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::tc_fence_after();
      ok = tc::mbar_wait(&do_full[st], ph, abort_flag, a.status);  // D, staged with dO
      // The shared dS tile is free once the previous tile's store has read it.
      ok = ok && tc::mbar_wait(ds_empty, (g & 1) ^ 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      const float* ld = reinterpret_cast<const float*>(smem + B_OFF_LD) + st * BQB + 64 * hf;
      // 32 queries at a time: chunk cc's dS^T goes over the dP^T columns of
      // queries [16 cc, 16 cc + 16), which chunk 0 has already read.
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t dpv[32];
        tc::tmem_ld_32x32b_x32(dp_col + 32 * cc, dpv);
        float dl[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 v = reinterpret_cast<const float4*>(ld + 32 * cc)[u];
          dl[4 * u] = v.x;
          dl[4 * u + 1] = v.y;
          dl[4 * u + 2] = v.z;
          dl[4 * u + 3] = v.w;
        }
        tc::tmem_ld_wait();
        uint32_t pd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // dl holds -D: dS = P (dP - D) as a packed add and multiply.
          const float2 dd = __fadd2_rn(make_float2(__uint_as_float(dpv[2 * i]), __uint_as_float(dpv[2 * i + 1])),
                                       make_float2(dl[2 * i], dl[2 * i + 1]));
          const float2 d = __fmul2_rn(unpack_bf16x2(pk[cc][i]), dd);
          pd[i] = pack_bf16x2(d.x, d.y);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t sw = (uint32_t)(((4 * cc + u) ^ (row & 7)) << 4);
          tc::st_shared_v4(ds_row + sw, pd[4 * u], pd[4 * u + 1], pd[4 * u + 2], pd[4 * u + 3]);
        }
        tc::tmem_st_32x32b_x16(dp_col + 16 * cc, pd);
      }
      tc::tmem_st_wait();
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(ds_full);
    }
  } else {
    // ---------------- epilogue: one key row per thread
    const int qw = warp & 3;
    const int row = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    KvCursor c;
    c.start(a, npairs, group, window);
    for (; c.valid; c.next_item(a, npairs, group, window)) {
      const int n = c.n;
      const int key = c.m.kb * BKV + row;
      // Keys at or past T (a ragged last tile) take part in the warp-wide
      // TMEM loads but write nothing (their global loads read key 0's row).
      const bool live = key < a.T;
      const int64_t tok = (int64_t)c.m.b * a.T + (live ? key : 0);
      const int kcol0 = c.m.hk * HD;
      // yhat of this key row (dims [8 u, 8 u + 8) in yv[u]) from the K tile
      // in shared memory as soon as it lands, then 1/rms and the first
      // (cos, sin) groups, all before the item's accumulators are waited for.
      bool okk = tc::mbar_wait(kv_full, n & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, okk)) break;
      uint4 yv[16];
      {
        const uint32_t krow = tc::smem_u32(smem + B_OFF_K) + row * 128;
#pragma unroll
        for (int u = 0; u < 16; ++u)
          yv[u] = tc::ld_shared_v4(krow + (u >> 3) * (TILE / 2) + (((u & 7) ^ (row & 7)) << 4));
      }
      tc::mbar_arrive(k_copied);
      const float r = a.rstd_k[tok * a.Hkv + c.m.hk];
      // (cos, sin) of four consecutive pairs of this key are 32 contiguous
      // bytes of the grouped table, so a warp's 32 keys read 1 KB at once;
      // a three-slot ring keeps two groups in flight ahead of their use.
      const float* csg = reinterpret_cast<const float*>(a.rope_tab + (int64_t)a.rope_T * 64) +
                         (int64_t)(live ? key : 0) * 8;
      const int64_t cs_step = (int64_t)a.rope_T * 8;  // floats from one group of 4 pairs to the next
      float cs0[8], cs1[8], cs2[8];
      tc::ld_global_v8f(csg, cs0);
      tc::ld_global_v8f(csg + cs_step, cs1);
      bool ok = tc::mbar_wait(dkv_full, n & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::tc_fence_after();
      {
        __nv_bfloat16* dst = a.dv + tok * a.ldg + kcol0;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tc::tmem_ld_32x32b_x32(lane_base + TB_DV + 32 * cc, o);
          tc::tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1]));
          if (live) {
            tc::st_global_v8(dst + 32 * cc, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
            tc::st_global_v8(dst + 32 * cc + 16, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
          }
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(dv_empty);
      // yhat element j from the packed row.
      auto yel = [&](int j) -> float {
        const uint4 v = yv[j >> 3];
        const uint32_t wv = (j & 7) < 2 ? v.x : (j & 7) < 4 ? v.y : (j & 7) < 6 ? v.z : v.w;
        const float2 f = unpack_bf16x2(wv);
        return (j & 1) ? f.y : f.x;
      };
      // The same element, unpacked by an instruction the compiler may not
      // merge with the first pass's: yhat then stays packed (64 registers)
      // between the two passes instead of as 128 floats.
      auto yel2 = [&](int j) -> float {
        const uint4 v = yv[j >> 3];
        const uint32_t wv = (j & 7) < 2 ? v.x : (j & 7) < 4 ? v.y : (j & 7) < 6 ? v.z : v.w;
        uint32_t u;
        if (j & 1)
          asm volatile("and.b32 %0, %1, 0xffff0000;" : "=r"(u) : "r"(wv));
        else
          asm volatile("shl.b32 %0, %1, 16;" : "=r"(u) : "r"(wv));
        return __uint_as_float(u);
      };
      float dot = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t gv[32];
        tc::tmem_ld_32x32b_x32(lane_base + TB_DK + 32 * cc, gv);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) dot = fmaf(__uint_as_float(gv[i]), yel(32 * cc + i), dot);
      }
      const float mean = dot * a.scale / 128.f;
      __nv_bfloat16* dst = a.dk + tok * a.ldg + kcol0;
      uint32_t lo[8], hi[8];  // four groups' outputs, stored as 32 bytes each
#pragma unroll
      for (int j = 0; j < 16; ++j) {  // pairs [4 j, 4 j + 4): dims 4 j + i and 64 + 4 j + i
        // Ring slot of group j: j % 3; group j + 2 goes into the slot group
        // j - 1 has just freed.
        float* cur = (j % 3 == 0) ? cs0 : (j % 3 == 1) ? cs1 : cs2;
        if (j + 2 < 16) {
          float* nxt = ((j + 2) % 3 == 0) ? cs0 : ((j + 2) % 3 == 1) ? cs1 : cs2;
          tc::ld_global_v8f(csg + (j + 2) * cs_step, *reinterpret_cast<float (*)[8]>(nxt));
        }
        uint32_t g0[4], g1[4];
        tc::tmem_ld_32x32b_x4(lane_base + TB_DK + 4 * j, g0);
        tc::tmem_ld_32x32b_x4(lane_base + TB_DK + 64 + 4 * j, g1);
        tc::tmem_ld_wait();
        if (j == 15) {  // dK is read: the MMA warp may overwrite it
          tc::tc_fence_before();
          tc::mbar_arrive(dk_empty);
        }
#pragma unroll
        for (int i = 0; i < 4; i += 2) {
          float o_lo[2], o_hi[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float cv = cur[2 * (i + e)], sv = cur[2 * (i + e) + 1];
            const float d0 = r * (__uint_as_float(g0[i + e]) * a.scale - yel2(4 * j + i + e) * mean);
            const float d1 = r * (__uint_as_float(g1[i + e]) * a.scale - yel2(64 + 4 * j + i + e) * mean);
            o_lo[e] = d0 * cv + d1 * sv;
            o_hi[e] = d1 * cv - d0 * sv;
          }
          lo[(j & 3) * 2 + i / 2] = pack_bf16x2(o_lo[0], o_lo[1]);
          hi[(j & 3) * 2 + i / 2] = pack_bf16x2(o_hi[0], o_hi[1]);
        }
        if ((j & 3) == 3 && live) {
          tc::st_global_v8(dst + 4 * (j - 3), lo[0], lo[1], lo[2], lo[3], lo[4], lo[5], lo[6], lo[7]);
          tc::st_global_v8(dst + 64 + 4 * (j - 3), hi[0], hi[1], hi[2], hi[3], hi[4], hi[5], hi[6], hi[7]);
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

// ------------------------------------------------------------------ dQ from stored dS
// Query side of the backward when the key-side kernel stored dS^T: a
// persistent kernel (one CTA per SM) walks the work items (128-query tile,
// query head, batch row) in balanced pairs (see DqWalk), and for each accumulates
//   dQ = sum over key tiles kb of dS(i, kb) K_kb        (M 128 queries, N 128 dims)
// in TMEM from the dS^T tile ([128 keys][128 queries], read MN-major) and the
// K tile ([128 keys][128 dims], MN-major), each through its own TMA ring.
// Two TMEM accumulators alternate between items, so one item's epilogue
// runs while the next item's tiles stream in and multiply.  The epilogue
// takes dQ through the backward of the q-side RoPE + QK-norm: with
// g = dQ / sqrt(128), yhat the saved normalised q and r its 1/rms,
//   dr = r (g - yhat mean(g yhat)),  dq = R(-theta) dr  (pairs i, i + 64),
// written as bf16 into the q slice of the q|k|v gradient.  320 threads:
// warp 0 TMA, warp 1 TMEM owner and MMA issue, warps 2..9 the epilogue, two
// threads per query row, each holding 32 whole RoPE pairs (dims
// [32 s, 32 s + 32) and [64 + 32 s, 96 + 32 s) for side s): the saved q row
// and its cos/sin are loaded before the accumulator is waited for, and the
// pair of threads combines its two halves of mean(g yhat) through shared
// memory.
constexpr int kDqThreads = 320;
// The dS^T tiles come from HBM (written by the key-side kernel, far larger
// than L2) and get a four-deep ring; a K tile is shared by the query tiles
// of its (head, row), which the item order keeps close together in time, so
// it mostly hits L2 and three stages cover that latency.
constexpr int kDqDsStages = 4;
constexpr int kDqKStages = 3;
constexpr int DQ_OFF_K = kDqDsStages * TILE;
constexpr int DQ_OFF_DOT = DQ_OFF_K + kDqKStages * TILE;  // [2 accumulators][2 sides][128 rows] f32
constexpr int DQ_OFF_BAR = DQ_OFF_DOT + 2 * 2 * 128 * 4;
constexpr int kDqSmem = DQ_OFF_BAR + 256;
static_assert(kDqSmem <= 232448, "dQ kernel shared memory budget");

struct DqArgs {
  int T, H, B, nqb;
  int group;   // query heads per KV head
  int window;  // query t sees keys [t - window, t]; < 0: every key up to t
  float scale;
  const __nv_bfloat16* yhat;  // saved normalised q: row tok at yhat + tok * ldy, head h at + h * 128
  int64_t ldy;
  const float* rstd_q;        // [B * T, H]
  const float2* rope_tab;     // [rope_T][64] (cos, sin), then the grouped copy
  int rope_T;
  __nv_bfloat16* out;         // dq rows: out + tok * ldo + h * 128
  int64_t ldo;
  int* status;
};

// Work item: query tile, head, batch row, and the key tiles [kb_lo, qi]
// whose dS^T tiles the key-side kernel stored for it.
struct DqItem {
  int qi, h, b, kb_lo, n;
};

// This CTA's work items in order.  Items come in pairs of one (head, row):
// query tile nqb - 1 - j, then tile j.  Under the causal mask the pair's tile
// counts add up to nqb + 1 whatever j is, so dealing pair p to CTA
// p mod gridDim.x balances the work; the pairs of one (head, row) are
// consecutive, so the CTAs working at the same time share its K tiles in L2.
struct DqWalk {
  int p, sub;
  __device__ __forceinline__ void start() {
    p = blockIdx.x;
    sub = 0;
  }
  __device__ __forceinline__ bool valid(int npairs) const { return p < npairs; }
  __device__ __forceinline__ DqItem item(const DqArgs& a, int window) const {
    const int ppg = (a.nqb + 1) / 2;
    const int grp = p / ppg;
    const int j = p - grp * ppg;
    DqItem it;
    it.qi = sub ? j : a.nqb - 1 - j;
    it.h = grp % a.H;
    it.b = grp / a.H;
    const int lo = window < 0 ? 0 : it.qi * BQB - BKV + 1 - window;
    it.kb_lo = lo <= 0 ? 0 : (lo + BKV - 1) / BKV;
    it.n = it.qi - it.kb_lo + 1;
    return it;
  }
  __device__ __forceinline__ void next(const DqArgs& a) {
    const int ppg = (a.nqb + 1) / 2;
    const int j = p % ppg;
    if (sub == 0 && a.nqb - 1 - j != j) {
      sub = 1;
    } else {
      sub = 0;
      p += gridDim.x;
    }
  }
};

// Walks this CTA's key tiles in order: tile t of the walk's current item.
struct DqCursor {
  DqWalk wk;
  int t;
  DqItem m;
  __device__ __forceinline__ bool valid(int npairs) const { return wk.valid(npairs); }
  __device__ __forceinline__ void start(const DqArgs& a, int window, int npairs) {
    wk.start();
    t = 0;
    if (wk.valid(npairs)) m = wk.item(a, window);
  }
  __device__ __forceinline__ void next(const DqArgs& a, int window, int npairs) {
    if (++t == m.n) {
      t = 0;
      wk.next(a);
      if (wk.valid(npairs)) m = wk.item(a, window);
    }
  }
};

template <bool GW>
__global__ void __launch_bounds__(kDqThreads, 1)
    attn_dq_kernel(const __grid_constant__ CUtensorMap tds, const __grid_constant__ CUtensorMap tk,
                   const DqArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((tc::smem_u32(smem_raw) & 1023u) != 0) {  // never expected; no room to realign
    if (threadIdx.x == 0 && a.status) atomicExch(a.status, kDevTimeout);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + DQ_OFF_BAR);
  uint64_t* ds_full = bars;                        // [kDqDsStages]
  uint64_t* ds_empty = bars + kDqDsStages;         // [kDqDsStages]
  uint64_t* k_full = bars + 2 * kDqDsStages;       // [kDqKStages]
  uint64_t* k_empty = k_full + kDqKStages;         // [kDqKStages]
  uint64_t* acc_full = k_empty + kDqKStages;       // [2]
  uint64_t* acc_empty = acc_full + 2;              // [2]
  uint64_t* dot_ready = acc_empty + 2;             // [2]
  uint64_t* drained = dot_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int window = GW ? a.window : -1;
  const int npairs = (a.nqb + 1) / 2 * a.H * a.B;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDqDsStages; ++i) {
      tc::mbar_init(&ds_full[i], 1);
      tc::mbar_init(&ds_empty[i], 1);
    }
    for (int i = 0; i < kDqKStages; ++i) {
      tc::mbar_init(&k_full[i], 1);
      tc::mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&acc_full[i], 1);
      tc::mbar_init(&acc_empty[i], 256);
      tc::mbar_init(&dot_ready[i], 256);
    }
    tc::mbar_init(drained, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 256);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tc::tma_prefetch_desc(&tds);
      tc::tma_prefetch_desc(&tk);
      // dS^T tile u and K tile u - (ring depth difference): the dS^T ring
      // runs kDqDsStages tiles ahead of the tensor core, the K ring kDqKStages.
      constexpr int lag = kDqDsStages - kDqKStages;
      DqCursor cd, ck;
      cd.start(a, window, npairs);
      ck.start(a, window, npairs);
      int issued_d = 0, issued_k = 0;
      bool ok = true;
      for (int u = 0; ok && (cd.valid(npairs) || ck.valid(npairs)); ++u) {
        if (cd.valid(npairs)) {
          const int st = issued_d % kDqDsStages;
          if (!tc::mbar_wait(&ds_empty[st], ((issued_d / kDqDsStages) & 1) ^ 1, abort_flag,
                             a.status)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&ds_full[st], TILE);
          for (int c = 0; c < 2; ++c)
            tc::tma_load_3d(smem + st * TILE + c * (TILE / 2), &tds, &ds_full[st],
                            cd.m.qi * BQB + 64 * c, (cd.m.kb_lo + cd.t) * BKV, cd.m.b * a.H + cd.m.h);
          ++issued_d;
          cd.next(a, window, npairs);
        }
        if (u >= lag && ck.valid(npairs)) {
          const int st = issued_k % kDqKStages;
          if (!tc::mbar_wait(&k_empty[st], ((issued_k / kDqKStages) & 1) ^ 1, abort_flag,
                             a.status)) {
            ok = false;
            break;
          }
          const int hk = GW ? ck.m.h / a.group : ck.m.h;
          tc::mbar_arrive_expect_tx(&k_full[st], TILE);
          for (int c = 0; c < 2; ++c)
            tc::tma_load_3d(smem + DQ_OFF_K + st * TILE + c * (TILE / 2), &tk, &k_full[st],
                            hk * HD + 64 * c, (ck.m.kb_lo + ck.t) * BKV, ck.m.b);
          ++issued_k;
          ck.next(a, window, npairs);
        }
      }
      if (!ok) {
        for (int i = max(0, issued_d - kDqDsStages); i < issued_d; ++i)
          drain_wait(&ds_full[i % kDqDsStages], (i / kDqDsStages) & 1);
        for (int i = max(0, issued_k - kDqKStages); i < issued_k; ++i)
          drain_wait(&k_full[i % kDqKStages], (i / kDqKStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = tc::idesc_bf16_f32(128, 128, 1, 1);
      const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(smem), TILE / 2, 1024);
      const uint64_t bd = tc::smem_desc_sw128(tc::smem_u32(smem + DQ_OFF_K), TILE / 2, 1024);
      int it = 0, item = 0;
      bool ok = true;
      DqWalk wk;
      for (wk.start(); wk.valid(npairs) && ok; wk.next(a), ++item) {
        const DqItem m = wk.item(a, window);
        const int buf = item & 1;
        // The epilogue of the item two back has read this accumulator.
        if (!tc::mbar_wait(&acc_empty[buf], ((item >> 1) & 1) ^ 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        for (int t = 0; t < m.n; ++t, ++it) {
          const int sd = it % kDqDsStages, sk = it % kDqKStages;
          if (!tc::mbar_wait(&ds_full[sd], (it / kDqDsStages) & 1, abort_flag, a.status) ||
              !tc::mbar_wait(&k_full[sk], (it / kDqKStages) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint64_t a0 = tc::desc_add(ad, sd * TILE), b0 = tc::desc_add(bd, sk * TILE);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)
            tc::umma_bf16_ss(tmem + 128 * buf, tc::desc_add(a0, kk * 2048), tc::desc_add(b0, kk * 2048),
                             id, (t > 0 || kk > 0) ? 1u : 0u);
          tc::umma_commit(&ds_empty[sd]);
          tc::umma_commit(&k_empty[sk]);
        }
        if (ok) tc::umma_commit(&acc_full[buf]);
      }
      tc::umma_commit(drained);
      drain_wait(drained, 0);
    }
  } else {
    // Epilogue: warps 2..9, a TMEM lane quarter each (warp % 4) and one side
    // of the row's RoPE pairs ((warp - 2) / 4).
    const int qw = warp & 3;
    const int side = (warp - 2) >> 2;
    const int row = qw * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
    float* dots = reinterpret_cast<float*>(smem + DQ_OFF_DOT);
    int item = 0;
    DqWalk wk;
    for (wk.start(); wk.valid(npairs); wk.next(a), ++item) {
      const DqItem m = wk.item(a, window);
      const int buf = item & 1;
      const uint32_t acc = lane_base + 128 * buf;
      const int q = m.qi * BQB + row;
      const bool live = q < a.T;
      const int64_t tok = (int64_t)m.b * a.T + (live ? q : 0);
      // Everything the row needs besides the accumulator, loaded before it
      // is waited for: the saved normalised q (dims 32 side + [0, 32) and
      // 64 + 32 side + [0, 32)), 1/rms and the 32 pairs' (cos, sin).
      // 32-byte loads: the q row's halves (the row's address is 32-byte
      // aligned), and (cos, sin) of four consecutive pairs from the grouped
      // copy of the table, where a warp's 32 rows read 1 KB at once.
      const __nv_bfloat16* yrow = a.yhat + tok * a.ldy + m.h * HD + 32 * side;
      uint4 yv[8];
#pragma unroll
      for (int u = 0; u < 4; u += 2) {
        uint32_t w0[8], w1[8];
        tc::ld_global_v8u(yrow + 8 * u, w0);
        tc::ld_global_v8u(yrow + 64 + 8 * u, w1);
        yv[u] = make_uint4(w0[0], w0[1], w0[2], w0[3]);
        yv[u + 1] = make_uint4(w0[4], w0[5], w0[6], w0[7]);
        yv[4 + u] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
        yv[5 + u] = make_uint4(w1[4], w1[5], w1[6], w1[7]);
      }
      const float r = a.rstd_q[tok * a.H + m.h];
      const float* csg = reinterpret_cast<const float*>(a.rope_tab + (int64_t)a.rope_T * 64) +
                         ((int64_t)(8 * side) * a.rope_T + (live ? q : 0)) * 8;
      float cs[8][8];  // pairs 32 side + 4 u + [0, 4): (cos, sin) x 4
#pragma unroll
      for (int u = 0; u < 8; ++u) tc::ld_global_v8f(csg + (int64_t)u * a.rope_T * 8, cs[u]);
      bool ok = tc::mbar_wait(&acc_full[buf], (item >> 1) & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::tc_fence_after();
      // yhat element j of half hh (j < 32) from the packed row.
      auto yel = [&](int hh, int j) -> float {
        const uint4 v = yv[4 * hh + (j >> 3)];
        const uint32_t wv = (j & 7) < 2 ? v.x : (j & 7) < 4 ? v.y : (j & 7) < 6 ? v.z : v.w;
        const float2 f = unpack_bf16x2(wv);
        return (j & 1) ? f.y : f.x;
      };
      float dot = 0.f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t g[16];
          tc::tmem_ld_32x32b_x16(acc + 64 * hh + 32 * side + 16 * c, g);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) dot = fmaf(__uint_as_float(g[i]), yel(hh, 16 * c + i), dot);
        }
      // The row's two halves of sum(g yhat) meet in shared memory.
      float* dslot = dots + buf * 256;
      dslot[side * 128 + row] = dot;
      tc::mbar_arrive(&dot_ready[buf]);
      ok = tc::mbar_wait(&dot_ready[buf], (item >> 1) & 1, abort_flag, a.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      const float mean = (dslot[row] + dslot[128 + row]) * a.scale / 128.f;
      __nv_bfloat16* dst = a.out + tok * a.ldo + m.h * HD + 32 * side;
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // pairs 32 side + 16 c + [0, 16)
        uint32_t g0[16], g1[16];
        tc::tmem_ld_32x32b_x16(acc + 32 * side + 16 * c, g0);
        tc::tmem_ld_32x32b_x16(acc + 64 + 32 * side + 16 * c, g1);
        tc::tmem_ld_wait();
        if (c == 1) {  // the accumulator is read: the MMA warp may reuse it
          tc::tc_fence_before();
          tc::mbar_arrive(&acc_empty[buf]);
        }
        uint32_t lo_[8], hi_[8];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float* t4 = &cs[(16 * c + i) / 4][2 * ((16 * c + i) % 4)];  // pairs i, i + 1 of the chunk
          const float cc[2] = {t4[0], t4[2]}, sn[2] = {t4[1], t4[3]};
          float o_lo[2], o_hi[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float d0 = r * (__uint_as_float(g0[i + e]) * a.scale - yel(0, 16 * c + i + e) * mean);
            const float d1 = r * (__uint_as_float(g1[i + e]) * a.scale - yel(1, 16 * c + i + e) * mean);
            o_lo[e] = d0 * cc[e] + d1 * sn[e];
            o_hi[e] = d1 * cc[e] - d0 * sn[e];
          }
          lo_[i / 2] = pack_bf16x2(o_lo[0], o_lo[1]);
          hi_[i / 2] = pack_bf16x2(o_hi[0], o_hi[1]);
        }
        if (live) {
          tc::st_global_v8(dst + 16 * c, lo_[0], lo_[1], lo_[2], lo_[3], lo_[4], lo_[5], lo_[6], lo_[7]);
          tc::st_global_v8(dst + 64 + 16 * c, hi_[0], hi_[1], hi_[2], hi_[3], hi_[4], hi_[5], hi_[6], hi_[7]);
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 256);
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
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_pp_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kPPSmem));
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
  a.B = B;
  const double flops = 4.0 * B * H * HD * causal_pairs(T, a.window);
  Probe probe(prof, s, "attn_fwd", flops, 0.0);
  if (a.group > 1 || a.window >= 0) {
    dim3 grid(a.nqb, H, B);
    attn_fwd_tc_kernel<true><<<grid, kThreads, kSmem, s>>>(mq, mk, mv, a);
  } else {
    // Persistent: one CTA per SM over the items (two query tiles each).
    const int nsuper = ((a.nqb + 1) / 2 + 1) / 2 * H * B;
    attn_fwd_pp_kernel<<<(unsigned)std::min(nsuper, num_sms()), kPPThreads, kPPSmem, s>>>(mq, mk, mv, a);
  }
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
                              int Hkv, int window, const float2* rope_tab, int rope_T,
                              const float* rstd_k, void* ds, int64_t ld_ds, int* status,
                              cudaStream_t s, Profiler* prof) {
  static DeviceOnce attr;
  NC_TRY(once_per_device(attr, []() -> nc_status {
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_tc_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem));
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_tc_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem));
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_kv_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem));
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_bwd_kv_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem));
    return NC_OK;
  }));
  const bool sds = ds != nullptr;
  if (Hkv < 1 || H % Hkv) return fail(NC_ERR_INVALID_ARG, "attention_bwd: H must be a multiple of Hkv");
  if (ldq % 8 || ldkv % 8 || ldo % 8 || ldg % 8 ||
      ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(dout) |
        reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 15))
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: rows must be 16-byte aligned");
  CUtensorMap mq, mk, mv, mdo, mdq;
  const uint64_t qcols = (uint64_t)H * HD, kvcols = (uint64_t)Hkv * HD;
  if (!make_tmap_bf16_3d(&mq, q, qcols, T, B, ldq, (int64_t)T * ldq, BQB) ||
      !make_tmap_bf16_3d(&mk, k, kvcols, T, B, ldkv, (int64_t)T * ldkv, BKV) ||
      !make_tmap_bf16_3d(&mv, v, kvcols, T, B, ldkv, (int64_t)T * ldkv, BKV) ||
      !make_tmap_bf16_3d(&mdo, dout, qcols, T, B, ldo, (int64_t)T * ldo, BQB))
    return fail(NC_ERR_INVALID_ARG, "attention_bwd: cuTensorMapEncodeTiled rejected an operand");
  if (sds) {
    // dS^T (bf16 [B * H][T keys][T queries], row stride ld_ds): 64 x 128 boxes.
    if (ld_ds < T || ld_ds % 8 || (reinterpret_cast<uintptr_t>(ds) & 15) ||
        !make_tmap_bf16_3d(&mdq, ds, T, T, (uint64_t)B * H, ld_ds, (int64_t)T * ld_ds, BKV))
      return fail(NC_ERR_INVALID_ARG, "attention_bwd: dS buffer rejected");
    if (!rope_tab || rope_T < T || !rstd_k)
      return fail(NC_ERR_INVALID_ARG, "attention_bwd: the store-dS form needs the RoPE table and rstd_k");
    if (ldg % 16 || ((reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 31))
      return fail(NC_ERR_INVALID_ARG, "attention_bwd: dk and dv rows must be 32-byte aligned");
  } else {
    // dq (fp32, dense [B, T, H * 128]): 32 x 32 boxes, 128-byte swizzle.
    if ((reinterpret_cast<uintptr_t>(dq) & 15) ||
        !make_tmap_3d(&mdq, dq, true, qcols, T, B, (int64_t)qcols, (int64_t)T * qcols, 32, 32, 128))
      return fail(NC_ERR_INVALID_ARG, "attention_bwd: dq rejected (16-byte aligned fp32)");
  }
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
  a.rope_tab = rope_tab;
  a.rope_T = rope_T;
  a.rstd_k = rstd_k;
  a.Hkv = Hkv;
  a.B = B;
  // Five products per (query, key) pair, or four when dQ is left to the
  // query-side kernel.
  const double flops = (sds ? 8.0 : 10.0) * B * H * HD * causal_pairs(T, a.window);
  Probe probe(prof, s, "attn_bwd", flops, 0.0);
  dim3 grid(a.nkb, Hkv, B);  // one CTA per key tile and KV head; it loops over the group
  const bool gw = a.group > 1 || a.window >= 0;
  if (sds) {
    // Persistent form: one CTA per SM over the (key tile, KV head, row) items.
    const unsigned pgrid = (unsigned)std::min<int64_t>((int64_t)(a.nkb + 1) / 2 * Hkv * B, num_sms());
    if (gw)
      attn_bwd_kv_kernel<true><<<pgrid, kKvThreads, kKvSmem, s>>>(mq, mk, mv, mdo, mdq, a);
    else
      attn_bwd_kv_kernel<false><<<pgrid, kKvThreads, kKvSmem, s>>>(mq, mk, mv, mdo, mdq, a);
  } else if (gw) {
    attn_bwd_tc_kernel<true><<<grid, kBwdThreads, kBwdSmem, s>>>(mq, mk, mv, mdo, mdq, a);
  } else {
    attn_bwd_tc_kernel<false><<<grid, kBwdThreads, kBwdSmem, s>>>(mq, mk, mv, mdo, mdq, a);
  }
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status attention_bwd_tc(const void* q, const void* k, const void* v, int64_t ld,
                           const void* dout, int64_t ldo, const float* lse, const float* delta,
                           float* dq, void* dk, void* dv, int64_t ldg, int B, int T, int H,
                           int* status, cudaStream_t s, Profiler* prof) {
  return attention_bwd_tc_ex(q, ld, k, v, ld, dout, ldo, lse, delta, dq, dk, dv, ldg, B, T, H, H, -1,
                             nullptr, 0, nullptr, nullptr, 0, status, s, prof);
}

nc_status attention_dq_ex(const void* ds, int64_t ld_ds, const void* k, int64_t ldkv, int B, int T,
                          int H, int Hkv, int window, const void* yhat, int64_t ldy,
                          const float* rstd_q, const float2* rope_tab, int rope_T, void* out,
                          int64_t ldo, int* status, cudaStream_t s, Profiler* prof) {
  static DeviceOnce attr;
  NC_TRY(once_per_device(attr, []() -> nc_status {
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_dq_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem));
    NC_CUDA_TRY(cudaFuncSetAttribute(attn_dq_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem));
    return NC_OK;
  }));
  if (B < 1 || T < 1 || H < 1 || Hkv < 1 || H % Hkv || !ds || !k || !yhat || !rstd_q ||
      !rope_tab || rope_T < T || !out)
    return fail(NC_ERR_INVALID_ARG, "attention_dq: bad arguments");
  if (ldy % 16 || ldo % 16 ||
      ((reinterpret_cast<uintptr_t>(yhat) | reinterpret_cast<uintptr_t>(out)) & 31))
    return fail(NC_ERR_INVALID_ARG, "attention_dq: q and dq rows must be 32-byte aligned");
  if (ldkv % 8 || ldy % 8 || ldo % 8 || ld_ds < T || ld_ds % 8 ||
      ((reinterpret_cast<uintptr_t>(ds) | reinterpret_cast<uintptr_t>(k) |
        reinterpret_cast<uintptr_t>(yhat) | reinterpret_cast<uintptr_t>(out)) & 15))
    return fail(NC_ERR_INVALID_ARG, "attention_dq: rows must be 16-byte aligned");
  CUtensorMap mds, mk;
  if (!make_tmap_bf16_3d(&mds, ds, T, T, (uint64_t)B * H, ld_ds, (int64_t)T * ld_ds, BKV) ||
      !make_tmap_bf16_3d(&mk, k, (uint64_t)Hkv * HD, T, B, ldkv, (int64_t)T * ldkv, BKV))
    return fail(NC_ERR_INVALID_ARG, "attention_dq: cuTensorMapEncodeTiled rejected an operand");
  DqArgs a;
  a.T = T;
  a.H = H;
  a.B = B;
  a.nqb = (T + BQB - 1) / BQB;
  a.group = H / Hkv;
  a.window = (window < 0 || window >= T - 1) ? -1 : window;
  a.scale = (float)(1.0 / std::sqrt((double)HD));
  a.yhat = static_cast<const __nv_bfloat16*>(yhat);
  a.ldy = ldy;
  a.rstd_q = rstd_q;
  a.rope_tab = rope_tab;
  a.rope_T = rope_T;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.ldo = ldo;
  a.status = status;
  const double flops = 2.0 * B * H * HD * causal_pairs(T, a.window);
  Probe probe(prof, s, "attn_bwd_dq", flops, 0.0);
  // Persistent: one CTA per SM (or per work item when there are fewer).
  const int npairs = (a.nqb + 1) / 2 * H * B;
  const unsigned grid = (unsigned)std::min(npairs, num_sms());
  if (a.group > 1 || a.window >= 0)
    attn_dq_kernel<true><<<grid, kDqThreads, kDqSmem, s>>>(mds, mk, a);
  else
    attn_dq_kernel<false><<<grid, kDqThreads, kDqSmem, s>>>(mds, mk, a);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

}  // namespace nc
