// gemm.cu -- the tcgen05 GEMM engine (sm_100a).
//
// Persistent kernels (one CTA, or one CTA pair, per SM) walk a list of
// output tiles.  Warp roles inside a CTA (320 threads):
//   warp 0      TMA producer: streams 128-byte K slices of A and B (64 bf16
//               or 128 E4M3 elements per row) into a STAGES-deep
//               shared-memory ring (128-byte swizzle), one mbarrier pair
//               (full / empty) per slot;
//   warp 1      allocates TMEM; one elected thread issues tcgen05.mma into a
//               TMEM accumulator and releases ring slots and accumulators
//               with tcgen05.commit;
//   warps 2..9  epilogue: tcgen05.ld the accumulator (a thread owns one row
//               of its warp's 32-row lane quarter and half of the columns),
//               apply the fused epilogue, store to global memory through a
//               per-warp staging slot.
// gemm_tc_kernel computes 128 x BN tiles on one CTA; gemm_tc2_kernel and
// gemm_tc2_aux_kernel compute 256 x 256 tiles on a cluster of two CTAs with
// tcgen05.mma.cta_group::2 (each CTA stages its 128 rows of A and of B, the
// even CTA issues the MMAs), the aux form reading an epilogue operand
// through a per-warp TMA ring.  The pair kernels also take E4M3 operands
// (kind::f8f6f4, both K-major, dequantised by the epilogue's alpha).
// The accumulator is double-buffered in TMEM (2 x BN columns), so the
// epilogue of tile i overlaps the main loop of tile i + 1.
// bf16 operands may be K-major or MN-major (transposed) independently,
// which covers y = x W^T, dx = dy W and dW = dy^T x without transposes.
// Every mbarrier wait is bounded (see tc.cuh); a timeout sets the device
// status word and every role drains and exits.

#include <algorithm>
#include <cmath>
#include <type_traits>

#include "kernels.h"
#include "tc.cuh"

namespace nc {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 320;  // TMA warp, MMA warp, 8 epilogue warps
constexpr int kEpiThreads = 256;

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int X_WARP_BYTES = 4096;  // per epilogue warp: one staging slot (RoPE epilogue)
  static constexpr int X_BYTES = (kEpiThreads / 32) * X_WARP_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + X_BYTES + BAR_BYTES + 1024;
};

struct Args {
  int M, N, K, batch;
  int tiles_m, tiles_n, split_k, kb_per_split, num_kb;
  int a_mn, b_mn;
  int epi;
  union {
    struct {
      float alpha, beta;
    };
    // fp8: the two operands' quantisation scales (device); the epilogue's
    // alpha becomes 1 / (ab_scale[0] * ab_scale[1]).
    const float* ab_scale;
  };
  void* D;
  int64_t ldd;
  // The RoPE/QK-norm epilogue (batch 1, no aux operand) keeps its parameters
  // in fields it does not otherwise use: the kernel argument block stays at
  // its size (growing it by 32 bytes measurably slowed every GEMM).
  union {
    int64_t stride_d;
    struct {
      int rope_T;
      int16_t rope_H, rope_Hkv;  // query heads, KV heads
    };
    // fp8 kernels with one batch and a bf16 output: where max |output| goes
    // (the bits of a non-negative float, for integer atomicMax), or null.
    unsigned* amax_out;
  };
  union {
    const void* aux;
    const float2* rope_tab;
  };
  union {
    int64_t ldaux;
    float* rstd_q;
  };
  union {
    int64_t stride_aux;
    float* rstd_k;
  };
  int* status;
};

struct TileCoord {
  int b, mb, nb, kb0, kb1;
};

// Tile order inside one (split, batch) plane.  Column tiles run fastest, so
// the CTAs running at the same time share A rows.  On planes much wider than
// the grid (the 32768-wide lm_head) that order sweeps all of B once per row
// of tiles while the output stream evicts it from L2 (2.7x the algorithmic
// DRAM bytes); there tiles go in groups of kGroupM row tiles, column tiles
// outer and row tiles inner, so concurrent CTAs share a few B column tiles
// and a group's A rows, which stay in L2.
constexpr int kGroupM = 16;
constexpr int kGroupMinTilesN = 32;
// Tiles of one (split, batch) plane.  A symmetric output (tiles_m < 0, a
// square plane of tiles_n x tiles_n tiles) computes only the tiles on or
// above the diagonal; the epilogue also stores each off-diagonal tile's
// transpose.
__device__ __forceinline__ int plane_tiles(const Args& p) {
  return p.tiles_m >= 0 ? p.tiles_m * p.tiles_n : p.tiles_n * (p.tiles_n + 1) / 2;
}

__device__ __forceinline__ TileCoord decode(const Args& p, int t) {
  TileCoord c;
  const int plane = plane_tiles(p);
  const int r = t % plane;
  t /= plane;
  if (p.tiles_m < 0) {  // row mb holds column tiles mb .. tiles_n - 1
    int mb = 0, rem = r, len = p.tiles_n;
    while (rem >= len) {
      rem -= len;
      ++mb;
      --len;
    }
    c.mb = mb;
    c.nb = mb + rem;
  } else if (p.tiles_n > kGroupMinTilesN) {
    const int gsize = kGroupM * p.tiles_n;
    const int g = r / gsize;
    const int gm = min(kGroupM, p.tiles_m - g * kGroupM);  // rows in this (possibly last) group
    const int in = r - g * gsize;
    c.mb = g * kGroupM + in % gm;
    c.nb = in / gm;
  } else {
    c.nb = r % p.tiles_n;
    c.mb = r / p.tiles_n;
  }
  const int ks = t % p.split_k;
  c.b = t / p.split_k;
  c.kb0 = ks * p.kb_per_split;
  c.kb1 = min(c.kb0 + p.kb_per_split, p.num_kb);
  return c;
}

// Plain bounded wait used while draining after an abort.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitTimeoutNs) return;
  }
}

// ------------------------------------------------------------------ epilogue
__device__ __forceinline__ bool epi_has_aux(int epi) {
  return epi == NC_EPI_RESID_F32 || epi == NC_EPI_RELU2_BWD || epi == NC_EPI_AXPBY_BF16;
}

// The aux operand of one 32-column chunk of one row, as floats (0 past N).
__device__ __forceinline__ void load_aux(const Args& p, int b, int row, int col0,
                                         float (&x)[32]) {
  const int nvalid = min(32, p.N - col0);
  if (p.epi == NC_EPI_RESID_F32) {
    const float* R = (const float*)p.aux + (int64_t)b * p.stride_aux + (int64_t)row * p.ldaux + col0;
    if (nvalid == 32) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 r = reinterpret_cast<const float4*>(R)[j];
        x[4 * j] = r.x; x[4 * j + 1] = r.y; x[4 * j + 2] = r.z; x[4 * j + 3] = r.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = j < nvalid ? R[j] : 0.f;
    }
  } else {
    const __nv_bfloat16* X = (const __nv_bfloat16*)p.aux + (int64_t)b * p.stride_aux +
                             (int64_t)row * p.ldaux + col0;
    if (nvalid == 32) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 u = reinterpret_cast<const uint4*>(X)[j];
        float2 f;
        f = unpack_bf16x2(u.x); x[8 * j + 0] = f.x; x[8 * j + 1] = f.y;
        f = unpack_bf16x2(u.y); x[8 * j + 2] = f.x; x[8 * j + 3] = f.y;
        f = unpack_bf16x2(u.z); x[8 * j + 4] = f.x; x[8 * j + 5] = f.y;
        f = unpack_bf16x2(u.w); x[8 * j + 6] = f.x; x[8 * j + 7] = f.y;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = j < nvalid ? bf2f(X[j]) : 0.f;
    }
  }
}

__device__ __forceinline__ void store_bf16_chunk(__nv_bfloat16* D, int nvalid, const float (&w)[32]) {
  if (nvalid == 32) {
    uint4* d4 = reinterpret_cast<uint4*>(D);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 u;
      u.x = pack_bf16x2(w[8 * j + 0], w[8 * j + 1]);
      u.y = pack_bf16x2(w[8 * j + 2], w[8 * j + 3]);
      u.z = pack_bf16x2(w[8 * j + 4], w[8 * j + 5]);
      u.w = pack_bf16x2(w[8 * j + 6], w[8 * j + 7]);
      d4[j] = u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nvalid) D[j] = f2bf(w[j]);
  }
}

// Apply the epilogue to one 32-column chunk (v = accumulator, x = aux) and store.
__device__ __forceinline__ void store_row_chunk(const Args& p, int b, int row, int col0,
                                                const float (&v)[32], const float (&x)[32]) {
  const int nvalid = min(32, p.N - col0);
  const int64_t off = (int64_t)b * p.stride_d + (int64_t)row * p.ldd + col0;
  float w[32];
  switch (p.epi) {
    case NC_EPI_STORE_BF16:
    case NC_EPI_RELU2:
    case NC_EPI_RELU2_BWD:
    case NC_EPI_AXPBY_BF16: {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float a = v[j] * p.alpha;
        if (p.epi == NC_EPI_RELU2) {
          const float r = fmaxf(a, 0.f);
          w[j] = r * r;
        } else if (p.epi == NC_EPI_RELU2_BWD) {
          w[j] = 2.f * sqrt_approx(fmaxf(x[j], 0.f)) * a;
        } else if (p.epi == NC_EPI_AXPBY_BF16) {
          w[j] = a + p.beta * x[j];
        } else {
          w[j] = a;
        }
      }
      store_bf16_chunk((__nv_bfloat16*)p.D + off, nvalid, w);
      break;
    }
    case NC_EPI_STORE_F32:
    case NC_EPI_RESID_F32: {
      float* D = (float*)p.D + off;
      const bool resid = p.epi == NC_EPI_RESID_F32;
      if (nvalid == 32) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float4 o = make_float4(v[4 * j] * p.alpha, v[4 * j + 1] * p.alpha,
                                 v[4 * j + 2] * p.alpha, v[4 * j + 3] * p.alpha);
          if (resid) {
            o.x += x[4 * j]; o.y += x[4 * j + 1]; o.z += x[4 * j + 2]; o.w += x[4 * j + 3];
          }
          reinterpret_cast<float4*>(D)[j] = o;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) D[j] = v[j] * p.alpha + (resid ? x[j] : 0.f);
      }
      break;
    }
    case NC_EPI_ACC_F32: {
      float* D = (float*)p.D + off;
      if (nvalid == 32) {  // 16-byte vector reductions (rows are 32-byte aligned)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(D + 4 * j),
                       "f"(v[4 * j] * p.alpha), "f"(v[4 * j + 1] * p.alpha), "f"(v[4 * j + 2] * p.alpha),
                       "f"(v[4 * j + 3] * p.alpha)
                       : "memory");
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nvalid) atomicAdd(D + j, v[j] * p.alpha);
      }
      break;
    }
    default:
      break;
  }
}

// Store one finished 32 x 32 block of a warp (row `lane` in w) through its
// shared-memory slot: each lane writes its row (fp32: 128-byte rows with the
// 128-byte swizzle; bf16: 64-byte rows with the 64-byte swizzle), then the
// warp stores the block row by row (8 lanes per fp32 row, 4 per bf16 row), so
// each store instruction covers whole lines instead of 16 bytes of 32
// different lines.  Rows past M and columns past N are skipped.
__device__ __forceinline__ void stage_store_chunk(const Args& p, uint8_t* slot, int lane, bool f32, int b,
                                                  int row0, int col0, const float (&w)[32],
                                                  bool mirror = false) {
  const uint32_t base = tc::smem_u32(slot);
  if (f32) {
    const uint32_t rowa = base + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      tc::st_shared_v4(rowa + ((j ^ (lane & 7)) << 4), __float_as_uint(w[4 * j]), __float_as_uint(w[4 * j + 1]),
                       __float_as_uint(w[4 * j + 2]), __float_as_uint(w[4 * j + 3]));
  } else {
    const uint32_t rowa = base + lane * 64;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      tc::st_shared_v4(rowa + ((j ^ ((lane >> 1) & 3)) << 4), pack_bf16x2(w[8 * j], w[8 * j + 1]),
                       pack_bf16x2(w[8 * j + 2], w[8 * j + 3]), pack_bf16x2(w[8 * j + 4], w[8 * j + 5]),
                       pack_bf16x2(w[8 * j + 6], w[8 * j + 7]));
  }
  __syncwarp();
  const int ncol = p.N - col0;  // >= 1
  if (f32) {
    float* D = (float*)p.D + (int64_t)b * p.stride_d + col0;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int rr = it * 4 + (lane >> 3), cc = lane & 7;
      const uint4 u = tc::ld_shared_v4(base + rr * 128 + ((cc ^ (rr & 7)) << 4));
      if (row0 + rr < p.M) {
        float* d = D + (int64_t)(row0 + rr) * p.ldd + cc * 4;
        if (cc * 4 + 4 <= ncol) {
          *reinterpret_cast<uint4*>(d) = u;
        } else {
          const uint32_t e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (cc * 4 + i < ncol) d[i] = __uint_as_float(e[i]);
        }
      }
    }
  } else {
    __nv_bfloat16* D = (__nv_bfloat16*)p.D + (int64_t)b * p.stride_d + col0;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int rr = it * 8 + (lane >> 2), cc = lane & 3;
      const uint4 u = tc::ld_shared_v4(base + rr * 64 + ((cc ^ ((rr >> 1) & 3)) << 4));
      if (row0 + rr < p.M) {
        __nv_bfloat16* d = D + (int64_t)(row0 + rr) * p.ldd + cc * 8;
        if (cc * 8 + 8 <= ncol) {
          *reinterpret_cast<uint4*>(d) = u;
        } else {
          const uint32_t e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (cc * 8 + i < ncol) {
              const uint32_t h = (e[i >> 1] >> ((i & 1) * 16)) & 0xffffu;
              d[i] = __ushort_as_bfloat16((unsigned short)h);
            }
        }
      }
    }
    if (mirror) {
      // The block's transpose at rows col0.., columns row0.. (a symmetric
      // output's other triangle): lane l gathers 8 block rows of column
      // it * 8 + l / 4 and stores them as 16 contiguous bytes.
      const uint16_t* sh = reinterpret_cast<const uint16_t*>(slot);
      __nv_bfloat16* Dt = (__nv_bfloat16*)p.D + (int64_t)b * p.stride_d + row0;
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int cc = it * 8 + (lane >> 2), r0 = (lane & 3) * 8;
        uint32_t e[4];
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
          const int ra = r0 + k, rb = r0 + k + 1;
          const uint32_t lo = sh[(ra * 64 + (((cc >> 3) ^ ((ra >> 1) & 3)) << 4)) / 2 + (cc & 7)];
          const uint32_t hi = sh[(rb * 64 + (((cc >> 3) ^ ((rb >> 1) & 3)) << 4)) / 2 + (cc & 7)];
          e[k / 2] = lo | (hi << 16);
        }
        if (cc < ncol && col0 + cc < p.M && row0 + r0 + 8 <= p.N)
          *reinterpret_cast<uint4*>(Dt + (int64_t)(col0 + cc) * p.ldd + r0) = make_uint4(e[0], e[1], e[2], e[3]);
        else if (cc < ncol && col0 + cc < p.M)
          for (int i = 0; i < 8; ++i)
            if (row0 + r0 + i < p.N) {
              const uint32_t h = (e[i >> 1] >> ((i & 1) * 16)) & 0xffffu;
              Dt[(int64_t)(col0 + cc) * p.ldd + r0 + i] = __ushort_as_bfloat16((unsigned short)h);
            }
      }
    }
  }
  __syncwarp();  // the slot may be rewritten by the warp's next chunk
}

// Fused q|k|v epilogue: this warp's 128 accumulator columns are one head
// (col0 is a multiple of 128): rope_H q heads, then rope_Hkv k heads, then
// rope_Hkv v heads.  q and k heads are rotated (pairs i, i + 64, position
// row % T) and RMS-normalised; v heads are stored as computed.  The rotation
// preserves the norm of every pair, so a first pass over TMEM takes the
// head's norm and a second rotates, scales and stores column chunks c and
// c + 2 together.
__device__ __forceinline__ void rope_head_epilogue(const Args& p, uint32_t taddr, int b, int row,
                                                   int col0, uint8_t* slot, int lane) {
  const bool live = row < p.M && col0 < p.N;
  const int hq = col0 >> 7;  // head index over q|k|v (uniform across the warp)
  const int region = hq < p.rope_H ? 0 : (hq < p.rope_H + p.rope_Hkv ? 1 : 2);  // q, k, v
  float rs = 1.f;
  if (region < 2) {
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tc::tmem_ld_32x32b_x32(taddr + c * 32, r);
      tc::tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float x = __uint_as_float(r[j]) * p.alpha;
        ss += x * x;
      }
    }
    rs = rsqrtf(ss / 128.f + kNormEps);
    if (live) {
      if (region) p.rstd_k[(int64_t)row * p.rope_Hkv + (hq - p.rope_H)] = rs;
      else p.rstd_q[(int64_t)row * p.rope_H + hq] = rs;
    }
  }
  (void)b;  // batch 1: stride_d holds T and H here
  const float4* tab = reinterpret_cast<const float4*>(p.rope_tab + (int64_t)(row % p.rope_T) * 64);
#pragma unroll 1
  for (int cp = 0; cp < 2; ++cp) {
    uint32_t lo[32], hi[32];
    tc::tmem_ld_32x32b_x32(taddr + cp * 32, lo);
    tc::tmem_ld_32x32b_x32(taddr + (cp + 2) * 32, hi);
    tc::tmem_ld_wait();
    float w0[32], w1[32];
    if (region < 2) {
#pragma unroll
      for (int i2 = 0; i2 < 16; ++i2) {
        const float4 cs = live ? tab[cp * 16 + i2] : make_float4(1.f, 0.f, 1.f, 0.f);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 2 * i2 + e;
          const float c = e ? cs.z : cs.x, sn = e ? cs.w : cs.y;
          const float x0 = __uint_as_float(lo[i]) * p.alpha, x1 = __uint_as_float(hi[i]) * p.alpha;
          w0[i] = (x0 * c - x1 * sn) * rs;
          w1[i] = (x0 * sn + x1 * c) * rs;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        w0[i] = __uint_as_float(lo[i]) * p.alpha;
        w1[i] = __uint_as_float(hi[i]) * p.alpha;
      }
    }
    stage_store_chunk(p, slot, lane, false, 0, row - lane, col0 + cp * 32, w0);
    stage_store_chunk(p, slot, lane, false, 0, row - lane, col0 + (cp + 2) * 32, w1);
  }
}

// ------------------------------------------------------------------ kernel
template <int BN, bool ROPE>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const Args p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_slots = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::X_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drained = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&tfull[i], 1);
      tc::mbar_init(&tempty[i], kEpiThreads);
    }
    tc::mbar_init(drained, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total = p.tiles_m * p.tiles_n * p.split_k * p.batch;

  if (warp == 0) {
    if (lane == 0) {
      tc::tma_prefetch_desc(&tmA);
      tc::tma_prefetch_desc(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileCoord c = decode(p, t);
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          uint8_t* a_dst = smem + stage * C::STAGE_BYTES;
          uint8_t* b_dst = a_dst + C::A_BYTES;
          const int k0 = kb * BK;
          if (!p.a_mn) {
            tc::tma_load_3d(a_dst, &tmA, &full[stage], k0, c.mb * BM, c.b);
          } else {
            tc::tma_load_3d(a_dst, &tmA, &full[stage], c.mb * BM, k0, c.b);
            tc::tma_load_3d(a_dst + 8192, &tmA, &full[stage], c.mb * BM + 64, k0, c.b);
          }
          if (!p.b_mn) {
            tc::tma_load_3d(b_dst, &tmB, &full[stage], k0, c.nb * BN, c.b);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tc::tma_load_3d(b_dst + j * 8192, &tmB, &full[stage], c.nb * BN + 64 * j, k0, c.b);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits.
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < min(issued, C::STAGES); ++i) {
          if (--s < 0) {
            s = C::STAGES - 1;
            ph ^= 1;
          }
          drain_wait(&full[s], ph);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(BM, BN, p.a_mn, p.b_mn);
      // Descriptors of stage 0; a stage adds STAGE_BYTES, a 16-wide K step adds
      // 32 bytes (K-major) or 16 rows of 128 bytes (MN-major).
      const uint32_t s0 = tc::smem_u32(smem);
      const uint64_t adesc0 = p.a_mn ? tc::smem_desc_sw128(s0, 8192, 1024) : tc::smem_desc_sw128(s0, 16, 1024);
      const uint64_t bdesc0 = p.b_mn ? tc::smem_desc_sw128(s0 + C::A_BYTES, 8192, 1024)
                                     : tc::smem_desc_sw128(s0 + C::A_BYTES, 16, 1024);
      const uint32_t a_step = p.a_mn ? 2048 : 32, b_step = p.b_mn ? 2048 : 32;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileCoord c = decode(p, t);
        if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!tc::mbar_wait(&full[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint64_t ad = adesc0 + (uint64_t)((stage * C::STAGE_BYTES) >> 4);
          const uint64_t bd = bdesc0 + (uint64_t)((stage * C::STAGE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc::umma_bf16_ss(d_tmem, tc::desc_add(ad, kk * a_step), tc::desc_add(bd, kk * b_step),
                             idesc, (kb > c.kb0 || kk > 0) ? 1u : 0u);
          tc::umma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc::umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // Wait for every issued MMA before TMEM is released.
      tc::umma_commit(drained);
      drain_wait(drained, 0);
    }
  } else {
    // Two epilogue warps per TMEM lane quarter, each taking half the columns.
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;
    constexpr int CH = BN / 32 / 2;  // 32-column chunks per warp
    const int row_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const TileCoord c = decode(p, t);
      bool ok = tc::mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::tc_fence_after();
      const int row = c.mb * BM + row_in_tile;
      const bool aux = epi_has_aux(p.epi);
      if constexpr (ROPE) {  // separate instantiation: the other GEMMs carry no RoPE code
        rope_head_epilogue(p, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + half * CH * 32, c.b,
                           row, c.nb * BN + half * CH * 32, stage_slots + (warp - 2) * C::X_WARP_BYTES, lane);
      } else {
      // The aux chunk is loaded one chunk ahead so its HBM latency overlaps
      // the current chunk's TMEM load, arithmetic and stores.
      float xa[32], xb[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) xa[j] = xb[j] = 0.f;
      {
        const int col0 = c.nb * BN + half * CH * 32;
        if (aux && row < p.M && col0 < p.N) load_aux(p, c.b, row, col0, xa);
      }
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int ch = half * CH + k;
        uint32_t r[32];
        tc::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + ch * 32, r);
        const int col0 = c.nb * BN + ch * 32;
        float(&cur)[32] = (k & 1) ? xb : xa;
        float(&nxt)[32] = (k & 1) ? xa : xb;
        if (aux && k + 1 < CH && row < p.M && col0 + 32 < p.N) load_aux(p, c.b, row, col0 + 32, nxt);
        tc::tmem_ld_wait();
        if (row < p.M && col0 < p.N) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          store_row_chunk(p, c.b, row, col0, v, cur);
        }
      }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA-pair kernel
// Same roles, but a cluster of two CTAs computes one 256 x 256 tile with
// tcgen05.mma.cta_group::2: each CTA stages its 128 rows of A and its 128
// rows of B (32 KB per 64-wide K slice instead of 48 KB for 128 x 256 on one
// CTA), the even CTA's MMA thread issues M = 256 MMAs over both CTAs' shared
// memory, and each CTA's TMEM receives its own 128 rows of the accumulator,
// drained by its own epilogue warps.  Both CTAs' copies complete on the
// leader's full barrier; commits arrive on both CTAs' barriers; epilogue
// warps release an accumulator with a remote arrive on the leader.
struct Cfg2 {
  static constexpr int BN = 256;
  static constexpr int A_BYTES = BM * BK * 2;         // this CTA's 128 rows of A
  static constexpr int B_BYTES = (BN / 2) * BK * 2;   // this CTA's 128 rows of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 6;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int X_WARP_BYTES = 4096;  // per epilogue warp: one staging slot
  static constexpr int X_BYTES = (kEpiThreads / 32) * X_WARP_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + X_BYTES + 512 + 1024;
};
static_assert(Cfg2::SMEM_BYTES <= 232448, "pair GEMM exceeds shared memory");

// The pair kernel for epilogues that read an aux operand: one operand stage
// fewer, and each epilogue warp owns an 8 KB ring of aux chunks (its 32 rows
// x 32 columns: two fp32 or four bf16 slots) that it fills by TMA ahead of
// use, across tile boundaries, so the aux read overlaps the main loop.
struct Cfg2X : Cfg2 {
  static constexpr int STAGES = 5;
  static constexpr int X_WARP_BYTES = 8192;
  static constexpr int X_MAX_SLOTS = 4;
  static constexpr int X_BYTES = (kEpiThreads / 32) * X_WARP_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + X_BYTES + 512 + 1024;
};
static_assert(Cfg2X::SMEM_BYTES <= 232448, "aux-ring pair GEMM exceeds shared memory");

// Request aux chunk g of this warp (tile pair + (g / CH) * npairs, column
// chunk g % CH) into its ring slot; false when that tile does not exist.
template <int BN, int CH>
__device__ __forceinline__ bool aux_issue(const Args& p, const CUtensorMap* tmX, uint8_t* ring,
                                          uint64_t* xfull, int slot_bytes, int slots, int g, int pair,
                                          int npairs, int total, int rank, int q, int half) {
  const int t = pair + (g / CH) * npairs;
  if (t >= total) return false;
  const TileCoord c = decode(p, t);
  const int slot = g & (slots - 1);
  tc::mbar_arrive_expect_tx(&xfull[slot], slot_bytes);
  tc::tma_load_3d(ring + slot * slot_bytes, tmX, &xfull[slot], c.nb * BN + (half * CH + g % CH) * 32,
                  c.mb * 2 * BM + rank * BM + q * 32, c.b);
  return true;
}

// This lane's row of one ring slot, as floats.  The slot holds 32 rows of
// 128 bytes (fp32, 128-byte swizzle) or 64 bytes (bf16, 64-byte swizzle).
__device__ __forceinline__ void aux_read_slot(const uint8_t* slot, int lane, bool f32, float (&x)[32]) {
  const uint32_t base = tc::smem_u32(slot);
  if (f32) {
    const uint32_t row = base + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 u = tc::ld_shared_v4(row + ((j ^ (lane & 7)) << 4));
      x[4 * j] = __uint_as_float(u.x); x[4 * j + 1] = __uint_as_float(u.y);
      x[4 * j + 2] = __uint_as_float(u.z); x[4 * j + 3] = __uint_as_float(u.w);
    }
  } else {
    const uint32_t row = base + lane * 64;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 u = tc::ld_shared_v4(row + ((j ^ ((lane >> 1) & 3)) << 4));
      float2 f;
      f = unpack_bf16x2(u.x); x[8 * j + 0] = f.x; x[8 * j + 1] = f.y;
      f = unpack_bf16x2(u.y); x[8 * j + 2] = f.x; x[8 * j + 3] = f.y;
      f = unpack_bf16x2(u.z); x[8 * j + 4] = f.x; x[8 * j + 5] = f.y;
      f = unpack_bf16x2(u.w); x[8 * j + 6] = f.x; x[8 * j + 7] = f.y;
    }
  }
}

// Aux epilogues of the ring kernel: the output has the aux operand's type, so
// the finished rows go out through the slot that held the aux rows.
__device__ __forceinline__ void aux_epilogue_chunk(const Args& p, uint8_t* slot, int lane, bool f32,
                                                   int b, int row0, int col0, const uint32_t (&r)[32],
                                                   bool mirror, float& amx) {
  float x[32];
  aux_read_slot(slot, lane, f32, x);
  __syncwarp();  // every lane has read its aux row before any is overwritten
  float w[32];
  const bool relu2_bwd = p.epi == NC_EPI_RELU2_BWD;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float a = __uint_as_float(r[j]) * p.alpha;
    w[j] = f32 ? x[j] + a : (relu2_bwd ? 2.f * sqrt_approx(fmaxf(x[j], 0.f)) * a : a + p.beta * x[j]);
    amx = fmaxf(amx, fabsf(w[j]));
  }
  stage_store_chunk(p, slot, lane, f32, b, row0, col0, w, mirror);
}

// Plain epilogues (bf16 / fp32 store, ReLU^2) of the pair kernel through the
// warp's staging slot; the accumulate and aux forms keep their own path.
__device__ __forceinline__ bool epi_staged(int epi) {
  return epi == NC_EPI_STORE_BF16 || epi == NC_EPI_RELU2 || epi == NC_EPI_STORE_F32;
}

// FP8: E4M3 operands (a stage holds 128 bytes of K per row: 128 elements).
template <bool ROPE, bool XR, bool FP8>
__device__ __forceinline__ void gemm_tc2_body(const CUtensorMap* tmA, const CUtensorMap* tmB,
                                              const CUtensorMap* tmX, const Args& p) {
  using C = std::conditional_t<XR, Cfg2X, Cfg2>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xring_all = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::SMEM_BYTES - 512 - 1024);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drained = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* xbar = drained + 2;  // XR: X_MAX_SLOTS per epilogue warp

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_ctarank();
  const bool leader = (rank == 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&tfull[i], 1);
      tc::mbar_init(&tempty[i], 2 * (kEpiThreads / 32));  // one arrive per epilogue warp of the pair
    }
    tc::mbar_init(drained, 1);
    if constexpr (XR) {
      for (int i = 0; i < (kEpiThreads / 32) * Cfg2X::X_MAX_SLOTS; ++i) tc::mbar_init(&xbar[i], 1);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc2(tmem_slot, C::TMEM_COLS);
    tc::tmem_relinquish2();
  }
  tc::tc_fence_before();
  tc::cluster_sync();  // both CTAs' barriers exist before any cross-CTA traffic
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int total = plane_tiles(p) * p.split_k * p.batch;  // tiles_m counts 256-row tiles

  if (warp == 0) {
    if (lane == 0) {
      tc::tma_prefetch_desc(tmA);
      tc::tma_prefetch_desc(tmB);
      if constexpr (XR) tc::tma_prefetch_desc(tmX);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        const TileCoord c = decode(p, t);
        const int m0 = c.mb * 2 * BM + (int)rank * BM;
        const int n0 = c.nb * BN + (int)rank * (BN / 2);
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!tc::mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (leader) tc::mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          uint8_t* a_dst = smem + stage * C::STAGE_BYTES;
          uint8_t* b_dst = a_dst + C::A_BYTES;
          const int k0 = kb * (FP8 ? 2 * BK : BK);
          if (!p.a_mn) {
            tc::tma_load_3d_pair(a_dst, tmA, &full[stage], k0, m0, c.b);
          } else {
            tc::tma_load_3d_pair(a_dst, tmA, &full[stage], m0, k0, c.b);
            tc::tma_load_3d_pair(a_dst + 8192, tmA, &full[stage], m0 + 64, k0, c.b);
          }
          if (!p.b_mn) {
            tc::tma_load_3d_pair(b_dst, tmB, &full[stage], k0, n0, c.b);
          } else {
            tc::tma_load_3d_pair(b_dst, tmB, &full[stage], n0, k0, c.b);
            tc::tma_load_3d_pair(b_dst + 8192, tmB, &full[stage], n0 + 64, k0, c.b);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // Copies land on the leader's barriers; let this CTA's stages settle.
        for (int i = 0; i < min(issued, C::STAGES); ++i) {
          if (--stage < 0) {
            stage = C::STAGES - 1;
            phase ^= 1;
          }
          drain_wait(&empty[stage], phase);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = FP8 ? tc::idesc_e4m3_f32(2 * BM, BN) : tc::idesc_bf16_f32(2 * BM, BN, p.a_mn, p.b_mn);
      const uint32_t s0 = tc::smem_u32(smem);
      const uint64_t adesc0 = p.a_mn ? tc::smem_desc_sw128(s0, 8192, 1024) : tc::smem_desc_sw128(s0, 16, 1024);
      const uint64_t bdesc0 = p.b_mn ? tc::smem_desc_sw128(s0 + C::A_BYTES, 8192, 1024)
                                     : tc::smem_desc_sw128(s0 + C::A_BYTES, 16, 1024);
      const uint32_t a_step = p.a_mn ? 2048 : 32, b_step = p.b_mn ? 2048 : 32;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        const TileCoord c = decode(p, t);
        if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!tc::mbar_wait(&full[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint64_t ad = adesc0 + (uint64_t)((stage * C::STAGE_BYTES) >> 4);
          const uint64_t bd = bdesc0 + (uint64_t)((stage * C::STAGE_BYTES) >> 4);
          // Four MMAs per stage: K = 16 bf16 or K = 32 E4M3 elements, 32 bytes each.
          if constexpr (FP8) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc::umma_f8_ss_pair(d_tmem, tc::desc_add(ad, kk * a_step), tc::desc_add(bd, kk * b_step),
                                  idesc, (kb > c.kb0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc::umma_bf16_ss_pair(d_tmem, tc::desc_add(ad, kk * a_step), tc::desc_add(bd, kk * b_step),
                                    idesc, (kb > c.kb0 || kk > 0) ? 1u : 0u);
          }
          tc::umma_commit_pair(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc::umma_commit_pair(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      tc::umma_commit_pair(drained);
      drain_wait(drained, 0);
    }
  } else {
    // The epilogue, on the kernel's arguments or (FP8) on a copy whose alpha
    // is the product of the operands' dequantisation factors.
    auto epilogue = [&](const Args& pe) {
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int CH = BN / 32 / 2;
    const int row_in_tile = q * 32 + lane;
    const uint32_t tempty_leader = tc::mapa_shared(tc::smem_u32(tempty), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    // XR: this warp's aux ring; chunk g (counted over this warp's tiles)
    // lives in slot g % slots.  Chunks [g_use, g_use + slots) are in flight.
    const bool xf32 = pe.epi == NC_EPI_RESID_F32;
    const int slot_bytes = xf32 ? 4096 : 2048;
    const int slots = XR ? Cfg2X::X_WARP_BYTES / slot_bytes : 1;
    const int slot_shift = slots == 4 ? 2 : 1;
    uint8_t* ring = xring_all + (warp - 2) * C::X_WARP_BYTES;  // XR: aux ring; else: staging slot
    uint64_t* xfull = xbar + (warp - 2) * Cfg2X::X_MAX_SLOTS;
    int g_use = 0;
    if constexpr (XR) {
      if (lane == 0)
        for (int g = 0; g < slots; ++g)
          aux_issue<BN, CH>(pe, tmX, ring, xfull, slot_bytes, slots, g, pair, npairs, total, (int)rank, q,
                            half);
    }
    bool xabort = false;
    float amx = 0.f;  // max |output| of this thread's values (fp8 kernels' amax_out)
    for (int t = pair; t < total; t += npairs) {
      const TileCoord c = decode(pe, t);
      bool ok = tc::mbar_wait(&tfull[acc], acc_phase, abort_flag, pe.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::tc_fence_after();
      const int row = c.mb * 2 * BM + (int)rank * BM + row_in_tile;
      const bool aux = epi_has_aux(pe.epi);
      const bool mirror = pe.tiles_m < 0 && c.mb != c.nb;  // symmetric output, off the diagonal
      if constexpr (ROPE) {  // separate instantiation: the other GEMMs carry no RoPE code
        rope_head_epilogue(pe, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + half * CH * 32, c.b,
                           row, c.nb * BN + half * CH * 32, ring, lane);
      } else if constexpr (XR) {
#pragma unroll
        for (int k = 0; k < CH; ++k) {
          const int ch = half * CH + k;
          uint32_t r[32];
          tc::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + ch * 32, r);
          const int col0 = c.nb * BN + ch * 32;
          const int slot = g_use & (slots - 1);
          const bool got = tc::mbar_wait(&xfull[slot], (g_use >> slot_shift) & 1, abort_flag, pe.status);
          tc::tmem_ld_wait();
          if (!__all_sync(0xffffffffu, got)) {
            xabort = true;
            break;
          }
          if (col0 < pe.N)
            aux_epilogue_chunk(pe, ring + slot * slot_bytes, lane, xf32, c.b, row - lane, col0, r, mirror, amx);
          // Every lane is done with the slot: order its accesses before the
          // TMA refill of the same slot with the chunk `slots` ahead.
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            aux_issue<BN, CH>(pe, tmX, ring, xfull, slot_bytes, slots, g_use + slots, pair, npairs, total,
                              (int)rank, q, half);
          }
          ++g_use;
        }
        if (xabort) break;
      } else if (epi_staged(pe.epi)) {
        const bool f32 = pe.epi == NC_EPI_STORE_F32;
#pragma unroll
        for (int k = 0; k < CH; ++k) {
          const int ch = half * CH + k;
          uint32_t r[32];
          tc::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + ch * 32, r);
          const int col0 = c.nb * BN + ch * 32;
          tc::tmem_ld_wait();
          if (col0 < pe.N) {
            float w[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float a = __uint_as_float(r[j]) * pe.alpha;
              w[j] = pe.epi == NC_EPI_RELU2 ? fmaxf(a, 0.f) * fmaxf(a, 0.f) : a;
              amx = fmaxf(amx, fabsf(w[j]));
            }
            stage_store_chunk(pe, ring, lane, f32, c.b, row - lane, col0, w, mirror);
          }
        }
      } else {
      float xa[32], xb[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) xa[j] = xb[j] = 0.f;
      {
        const int col0 = c.nb * BN + half * CH * 32;
        if (aux && row < pe.M && col0 < pe.N) load_aux(pe, c.b, row, col0, xa);
      }
#pragma unroll
      for (int k = 0; k < CH; ++k) {
        const int ch = half * CH + k;
        uint32_t r[32];
        tc::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + ch * 32, r);
        const int col0 = c.nb * BN + ch * 32;
        float(&cur)[32] = (k & 1) ? xb : xa;
        float(&nxt)[32] = (k & 1) ? xa : xb;
        if (aux && k + 1 < CH && row < pe.M && col0 + 32 < pe.N) load_aux(pe, c.b, row, col0 + 32, nxt);
        tc::tmem_ld_wait();
        if (row < pe.M && col0 < pe.N) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          store_row_chunk(pe, c.b, row, col0, v, cur);
        }
      }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_cluster(tempty_leader + acc * 8);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    if constexpr (XR) {
      // After an abort, let the aux copies still in flight land before the
      // CTA exits (chunks past the last tile were never requested).
      for (int g = g_use; g < g_use + slots; ++g)
        if (pair + (g / CH) * npairs < total) drain_wait(&xfull[g & (slots - 1)], (g >> slot_shift) & 1);
    }
    if constexpr (FP8 && !ROPE) {
      // The output's amax as the bf16 values stored (rounding is monotonic).
      if (pe.batch == 1 && pe.amax_out && pe.epi != NC_EPI_STORE_F32 && pe.epi != NC_EPI_RESID_F32 &&
          pe.epi != NC_EPI_ACC_F32) {
        amx = warp_max(amx);
        if (lane == 0) atomicMax(pe.amax_out, __float_as_uint(__bfloat162float(__float2bfloat16_rn(amx))));
      }
    }
      };
    if constexpr (FP8) {
      Args pe = p;
      pe.alpha = 1.f / (p.ab_scale[0] * p.ab_scale[1]);
      epilogue(pe);
    } else {
      epilogue(p);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc2(tmem_base, C::TMEM_COLS);
  }
}


template <bool ROPE, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Args p) {
  gemm_tc2_body<ROPE, false, FP8>(&tmA, &tmB, nullptr, p);
}

template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc2_aux_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmX, const Args p) {
  gemm_tc2_body<false, true, FP8>(&tmA, &tmB, &tmX, p);
}

// ------------------------------------------------------------------ host
template <int BN, bool ROPE>
nc_status launch_bn(const nc_gemm_desc& d, int split, int* status, const char* tag,
                    cudaStream_t s, Profiler* prof) {
  using C = Cfg<BN>;
  static DeviceOnce smem_attr;
  NC_TRY(once_per_device(smem_attr, []() -> nc_status {
    NC_CUDA_TRY(cudaFuncSetAttribute(gemm_tc_kernel<BN, ROPE>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    return NC_OK;
  }));
  CUtensorMap ta, tb;
  const bool ok_a = d.a_kmajor ? make_tmap_bf16_3d(&ta, d.A, d.K, d.M, d.batch, d.lda, d.stride_a, BM)
                               : make_tmap_bf16_3d(&ta, d.A, d.M, d.K, d.batch, d.lda, d.stride_a, 64);
  const bool ok_b = d.b_kmajor ? make_tmap_bf16_3d(&tb, d.B, d.K, d.N, d.batch, d.ldb, d.stride_b, BN)
                               : make_tmap_bf16_3d(&tb, d.B, d.N, d.K, d.batch, d.ldb, d.stride_b, 64);
  if (!ok_a || !ok_b) return fail(NC_ERR_INVALID_ARG, "gemm: cuTensorMapEncodeTiled rejected an operand");

  Args a;
  a.M = d.M;
  a.N = d.N;
  a.K = d.K;
  a.batch = d.batch;
  a.tiles_m = (d.M + BM - 1) / BM;
  a.tiles_n = (d.N + BN - 1) / BN;
  a.num_kb = (d.K + BK - 1) / BK;
  a.kb_per_split = (a.num_kb + split - 1) / split;
  a.split_k = (a.num_kb + a.kb_per_split - 1) / a.kb_per_split;
  a.a_mn = d.a_kmajor ? 0 : 1;
  a.b_mn = d.b_kmajor ? 0 : 1;
  a.epi = d.epi;
  a.alpha = d.alpha;
  a.beta = d.beta;
  a.D = d.D;
  a.ldd = d.ldd;
  a.stride_d = d.stride_d;
  a.aux = d.aux;
  a.ldaux = d.ldaux;
  a.stride_aux = d.stride_aux;
  if (d.epi == NC_EPI_ROPE_QKNORM) {  // shares storage with stride_d and the aux fields
    a.rope_T = d.rope_T;
    a.rope_H = (int16_t)d.rope_H;
    a.rope_Hkv = (int16_t)(d.rope_Hkv > 0 ? d.rope_Hkv : d.rope_H);
    a.rope_tab = static_cast<const float2*>(d.rope_tab);
    a.rstd_q = d.rstd_q;
    a.rstd_k = d.rstd_k;
  }
  a.status = status;
  const int64_t total = (int64_t)a.tiles_m * a.tiles_n * a.split_k * a.batch;
  if (total >= (1ll << 31)) return fail(NC_ERR_INVALID_ARG, "gemm: too many tiles");
  const int grid = (int)std::min<int64_t>(total, num_sms());
  const double flops = 2.0 * d.M * (double)d.N * d.K * d.batch;
  Probe probe(prof, s, tag, flops, 0.0);
  gemm_tc_kernel<BN, ROPE><<<grid, kThreads, C::SMEM_BYTES, s>>>(ta, tb, a);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

template <bool ROPE, bool XR>
nc_status launch_pair(const nc_gemm_desc& d, int split, int* status, const char* tag,
                      cudaStream_t s, Profiler* prof, bool symmetric = false) {
  using C = std::conditional_t<XR, Cfg2X, Cfg2>;
  static DeviceOnce smem_attr;
  NC_TRY(once_per_device(smem_attr, []() -> nc_status {
    if constexpr (XR) {
      NC_CUDA_TRY(cudaFuncSetAttribute(gemm_tc2_aux_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES));
      NC_CUDA_TRY(cudaFuncSetAttribute(gemm_tc2_aux_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES));
    } else {
      NC_CUDA_TRY(cudaFuncSetAttribute(gemm_tc2_kernel<ROPE, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
      NC_CUDA_TRY(cudaFuncSetAttribute(gemm_tc2_kernel<ROPE, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    }
    return NC_OK;
  }));
  CUtensorMap ta, tb, tx;
  if constexpr (XR) {
    // aux chunks of 32 columns x 32 rows: 128-byte rows (fp32) or 64-byte rows (bf16)
    const bool f32 = d.epi == NC_EPI_RESID_F32;
    if (!make_tmap_3d(&tx, d.aux, f32, d.N, d.M, d.batch, d.ldaux, d.stride_aux, 32, 32, f32 ? 128 : 64))
      return fail(NC_ERR_INVALID_ARG, "gemm: cuTensorMapEncodeTiled rejected the aux operand");
  }
  const bool fp8 = d.ab_type == 1;  // E4M3, both operands K-major (checked by the caller)
  bool ok_a, ok_b;
  if (fp8) {
    ok_a = make_tmap_u8_3d(&ta, d.A, d.K, d.M, d.batch, d.lda, d.stride_a, BM);
    ok_b = make_tmap_u8_3d(&tb, d.B, d.K, d.N, d.batch, d.ldb, d.stride_b, C::BN / 2);
  } else {
    ok_a = d.a_kmajor ? make_tmap_bf16_3d(&ta, d.A, d.K, d.M, d.batch, d.lda, d.stride_a, BM)
                      : make_tmap_bf16_3d(&ta, d.A, d.M, d.K, d.batch, d.lda, d.stride_a, 64);
    ok_b = d.b_kmajor ? make_tmap_bf16_3d(&tb, d.B, d.K, d.N, d.batch, d.ldb, d.stride_b, C::BN / 2)
                      : make_tmap_bf16_3d(&tb, d.B, d.N, d.K, d.batch, d.ldb, d.stride_b, 64);
  }
  if (!ok_a || !ok_b) return fail(NC_ERR_INVALID_ARG, "gemm: cuTensorMapEncodeTiled rejected an operand");
  const int bk = fp8 ? 2 * BK : BK;  // K elements per 128-byte stage row
  Args a;
  a.M = d.M;
  a.N = d.N;
  a.K = d.K;
  a.batch = d.batch;
  a.tiles_m = (d.M + 2 * BM - 1) / (2 * BM);
  a.tiles_n = (d.N + C::BN - 1) / C::BN;
  a.num_kb = (d.K + bk - 1) / bk;
  a.kb_per_split = (a.num_kb + split - 1) / split;
  a.split_k = (a.num_kb + a.kb_per_split - 1) / a.kb_per_split;
  a.a_mn = d.a_kmajor ? 0 : 1;
  a.b_mn = d.b_kmajor ? 0 : 1;
  a.epi = d.epi;
  if (fp8) {  // the operand type itself is the kernel's FP8 template argument
    a.ab_scale = d.ab_scale;
  } else {
    a.alpha = d.alpha;
    a.beta = d.beta;
  }
  a.D = d.D;
  a.ldd = d.ldd;
  a.stride_d = d.batch > 1 ? d.stride_d : 0;
  if (fp8 && d.amax_out) a.amax_out = d.amax_out;  // batch 1 (checked by the caller)
  a.aux = d.aux;
  a.ldaux = d.ldaux;
  a.stride_aux = d.stride_aux;
  if (d.epi == NC_EPI_ROPE_QKNORM) {  // shares storage with stride_d and the aux fields
    a.rope_T = d.rope_T;
    a.rope_H = (int16_t)d.rope_H;
    a.rope_Hkv = (int16_t)(d.rope_Hkv > 0 ? d.rope_Hkv : d.rope_H);
    a.rope_tab = static_cast<const float2*>(d.rope_tab);
    a.rstd_q = d.rstd_q;
    a.rstd_k = d.rstd_k;
  }
  a.status = status;
  int64_t plane = (int64_t)a.tiles_m * a.tiles_n;
  if (symmetric) {  // tiles_m < 0 marks it; the kernel walks the upper triangle
    plane = (int64_t)a.tiles_n * (a.tiles_n + 1) / 2;
    a.tiles_m = -a.tiles_n;
  }
  const int64_t total = plane * a.split_k * a.batch;
  if (total >= (1ll << 31)) return fail(NC_ERR_INVALID_ARG, "gemm: too many tiles");
  const int pairs = (int)std::min<int64_t>(total, num_sms() / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Algorithmic FLOPs: a symmetric output counts the tiles it computes.
  const double flops = symmetric ? 2.0 * d.K * d.batch * (double)plane * 256.0 * 256.0
                                 : 2.0 * d.M * (double)d.N * d.K * d.batch;
  (void)bk;
  Probe probe(prof, s, tag, flops, 0.0);
  if constexpr (XR) {
    if (fp8)
      NC_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_tc2_aux_kernel<true>, ta, tb, tx, a));
    else
      NC_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_tc2_aux_kernel<false>, ta, tb, tx, a));
  } else {
    if (fp8)
      NC_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<ROPE, true>, ta, tb, a));
    else
      NC_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<ROPE, false>, ta, tb, a));
  }
  return NC_OK;
}

// K-split of the weight-gradient GEMMs (automatic split): each split's
// slice of A and B should fit in L2 with room to spare, so that the CTAs
// working on the same slice at the same time share it (a 5120 x 1280 x 65536
// weight gradient ran 1194 TFLOP/s at 2 splits, 210 MB per slice, against
// 1357 at 8, 52 MB).
constexpr double kSplitSliceBytes = 112e6;

// Smallest split, at least the L2 minimum, that keeps the last wave at least
// 85% full (or the best below 16).  operand_bytes: A and B over the whole K.
int auto_split(int64_t tiles, int num_kb, double operand_bytes) {
  const int sms = num_sms();
  // (Planes with several waves of tiles of their own keep the plain rule:
  // their concurrent tiles already share A rows, and every split adds a
  // full fp32 pass of reductions over D.)
  const int smin = tiles >= 4 * sms ? 1
                                    : std::max(1, std::min(16, (int)std::ceil(operand_bytes / kSplitSliceBytes)));
  int best = 1;
  double best_eff = 0;
  for (int s = smin; s <= 16; ++s) {
    if (s > smin && num_kb / s < 8) break;
    const int64_t t = tiles * s;
    const double eff = (double)t / (double)(((t + sms - 1) / sms) * sms);
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = s;
    }
    if (eff >= 0.85) break;
  }
  return best;
}

}  // namespace

nc_status gemm_launch(const GemmLaunch& g, cudaStream_t s, Profiler* prof) {
  const nc_gemm_desc& d = g.d;
  if (d.M < 1 || d.N < 1 || d.K < 1 || d.batch < 1 || !d.A || !d.B || !d.D)
    return fail(NC_ERR_INVALID_ARG, "gemm: empty shape or null operand");
  auto aligned = [](int64_t v) { return v % 8 == 0; };
  if (d.ab_type != 0 && d.ab_type != 1) return fail(NC_ERR_INVALID_ARG, "gemm: unknown operand type");
  const bool fp8 = d.ab_type == 1;
  if (d.amax_out && (!fp8 || d.batch != 1 || d.epi == NC_EPI_ROPE_QKNORM || d.epi == NC_EPI_STORE_F32 ||
                     d.epi == NC_EPI_RESID_F32 || d.epi == NC_EPI_ACC_F32))
    return fail(NC_ERR_INVALID_ARG, "gemm: amax_out needs E4M3 operands, one batch and a bf16 epilogue");
  if (fp8 && (!d.a_kmajor || !d.b_kmajor || d.lda % 16 || d.ldb % 16 ||
              (d.batch > 1 && (d.stride_a % 16 || d.stride_b % 16)) || !d.ab_scale || d.alpha != 1.f ||
              d.epi == NC_EPI_AXPBY_BF16 || g.symmetric))
    return fail(NC_ERR_INVALID_ARG,
                "gemm: E4M3 operands must be K-major with leading dimensions and batch strides of "
                "16-byte multiples, scales given, alpha 1 and no alpha*acc + beta*aux epilogue");
  if (!aligned(d.lda) || !aligned(d.ldb) || (d.batch > 1 && (!aligned(d.stride_a) || !aligned(d.stride_b))))
    return fail(NC_ERR_INVALID_ARG, "gemm: leading dimensions and batch strides must be multiples of 8");
  if ((reinterpret_cast<uintptr_t>(d.A) | reinterpret_cast<uintptr_t>(d.B)) & 15)
    return fail(NC_ERR_INVALID_ARG, "gemm: operands must be 16-byte aligned");
  const bool needs_aux = d.epi == NC_EPI_RESID_F32 || d.epi == NC_EPI_RELU2_BWD ||
                         d.epi == NC_EPI_AXPBY_BF16;
  if (needs_aux && (!d.aux || !aligned(d.ldaux)))
    return fail(NC_ERR_INVALID_ARG, "gemm: epilogue needs an aux operand with ld multiple of 8");
  if (!aligned(d.ldd) || (reinterpret_cast<uintptr_t>(d.D) & 15) ||
      (needs_aux && (reinterpret_cast<uintptr_t>(d.aux) & 15)))
    return fail(NC_ERR_INVALID_ARG, "gemm: output / aux must be 16-byte aligned rows");
  if (d.epi < NC_EPI_STORE_BF16 || d.epi > NC_EPI_ROPE_QKNORM)
    return fail(NC_ERR_INVALID_ARG, "gemm: unknown epilogue");
  const bool rope = d.epi == NC_EPI_ROPE_QKNORM;
  const int rope_kv = d.rope_Hkv > 0 ? d.rope_Hkv : d.rope_H;
  if (rope && (d.rope_T < 1 || d.rope_H < 1 || d.rope_H > 4096 || rope_kv > d.rope_H ||
               d.N != 128 * (d.rope_H + 2 * rope_kv) || !d.rope_tab || !d.rstd_q || !d.rstd_k ||
               d.alpha != 1.f || d.batch != 1))
    return fail(NC_ERR_INVALID_ARG, "gemm: the RoPE/QK-norm epilogue needs N = 128*(H + 2*Hkv), Hkv <= H, T, a table and rstd outputs");
  int split = d.split_k;
  if (split != 1 && d.epi != NC_EPI_ACC_F32)
    return fail(NC_ERR_INVALID_ARG, "gemm: split_k > 1 needs the accumulate epilogue");
  // N tile: 256 unless 128 wastes less of the last column tile (but see below).
  const int waste256 = ((d.N + 255) / 256) * 256 - d.N;
  const int waste128 = ((d.N + 127) / 128) * 128 - d.N;
  // (the RoPE/QK-norm epilogue needs 256-wide tiles: each warp-half is a head)
  // (a symmetric output walks square 256 x 256 tiles whatever the edge waste)
  // The 256-wide pair kernel also when its last column tile is ragged, as
  // long as the padding stays within an eighth of the columns computed
  // (d = 1664 at depth 26: 128 of 1792): it outruns 128-wide single-CTA
  // tiles by more than that.  E4M3 operands run only on the pair kernel.
  const int n256 = ((d.N + 255) / 256) * 256;
  const bool bn256 = rope || g.symmetric ||
                     (d.N > 128 && (waste256 <= waste128 || 8 * waste256 <= n256 || fp8));
  const int bn = bn256 ? 256 : 128;
  const int num_kb = (d.K + (fp8 ? 2 * BK : BK) - 1) / (fp8 ? 2 * BK : BK);
  const double operand_bytes = (fp8 ? 1.0 : 2.0) * ((double)d.M + d.N) * d.K * d.batch;
  if (split <= 0) {
    const int64_t tiles = (int64_t)((d.M + BM - 1) / BM) * ((d.N + bn - 1) / bn) * d.batch;
    split = auto_split(tiles, num_kb, operand_bytes);
  }
  if (split > num_kb) split = num_kb;
  // 256 x 256 tiles on a CTA pair whenever M spans more than one 128-row
  // tile and 256-wide column tiles fit N; 128 x BN on one CTA otherwise.
  if (g.symmetric &&
      (d.M != d.N || !bn256 || d.M <= BM || split != 1 ||
       (d.epi != NC_EPI_STORE_BF16 && d.epi != NC_EPI_AXPBY_BF16)))
    return fail(NC_ERR_INVALID_ARG, "gemm: a symmetric output needs M == N > 128, one split and a bf16 epilogue");
  if (bn256 && d.M > BM) {
    if (d.split_k <= 0) {
      const int64_t tiles = (int64_t)((d.M + 2 * BM - 1) / (2 * BM)) * ((d.N + 255) / 256) * d.batch;
      split = std::min(auto_split(tiles * 2, num_kb, operand_bytes), num_kb);
    }
    if (rope) return launch_pair<true, false>(d, split, g.status, g.tag, s, prof);
    // Aux epilogues read the aux operand by TMA (rows and batch strides of
    // 16-byte multiples, which the checks above already imply).
    if (needs_aux && (d.batch == 1 || aligned(d.stride_aux)))
      return launch_pair<false, true>(d, split, g.status, g.tag, s, prof, g.symmetric);
    return launch_pair<false, false>(d, split, g.status, g.tag, s, prof, g.symmetric);
  }
  if (fp8)
    return fail(NC_ERR_INVALID_ARG, "gemm: E4M3 operands need M > 128 and N > 128");
  if (rope) return launch_bn<256, true>(d, split, g.status, g.tag, s, prof);
  return bn256 ? launch_bn<256, false>(d, split, g.status, g.tag, s, prof)
               : launch_bn<128, false>(d, split, g.status, g.tag, s, prof);
}

}  // namespace nc
