// elementwise.cu -- the memory-bound kernels of the step: embedding gather
// and scatter-add, RMSNorm forward/backward, the RoPE table,
// fused softmax cross-entropy (loss and logits gradient in one pass),
// parameter init, bf16 refresh, the Muon momentum / normalise / apply
// passes and the AdamW step of the embedding and lm_head.  One warp per row where a row reduction is needed (warp-shuffle
// sums, fp32 statistics), 16-byte vector accesses where rows allow.

#include "common.cuh"
#include "internal.h"
#include "kernels.h"
#include "exp2_poly.cuh"

#include <cuda_fp8.h>

namespace nc {
namespace {

// ------------------------------------------------------------------ embedding
__global__ void embed_gather_kernel(const int32_t* __restrict__ tok, int64_t n, const float* __restrict__ E,
                                    int V, int d, float* __restrict__ x, int* status) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= n) return;
  int id = tok[w];
  if (id < 0 || id >= V) {
    if (lane == 0) atomicExch(status, kDevTokenRange);
    id = id < 0 ? 0 : V - 1;
  }
  const float4* src = reinterpret_cast<const float4*>(E + (int64_t)id * d);
  float4* dst = reinterpret_cast<float4*>(x + w * d);
  for (int i = lane; i < d / 4; i += 32) dst[i] = src[i];
}

__global__ void embed_scatter_kernel(const int32_t* __restrict__ tok, int64_t n, const float* __restrict__ dx,
                                     int V, int d, float* __restrict__ dE) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= n) return;
  int id = tok[w];
  id = id < 0 ? 0 : (id >= V ? V - 1 : id);
  const float4* src = reinterpret_cast<const float4*>(dx + w * d);
  float* dst = dE + (int64_t)id * d;
  for (int i = lane; i < d / 4; i += 32) {
    const float4 g = src[i];
    // One 16-byte vector reduction per float4 (rows are 16-byte aligned).
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 4 * i), "f"(g.x),
                 "f"(g.y), "f"(g.z), "f"(g.w)
                 : "memory");
  }
}

// ------------------------------------------------------------------ RMSNorm
// max |v| of a block's values (one per thread) into *amax as bf16 bits of a
// non-negative float (the output's rounding is monotonic, so this is the max
// of the stored bf16 values); one atomic per block.
__device__ __forceinline__ void block_amax_bf16(float v, unsigned* amax) {
  __shared__ float red[32];
  v = warp_max(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) v = fmaxf(v, red[i]);
    atomicMax(amax, __float_as_uint(__bfloat162float(__float2bfloat16_rn(v))));
  }
}

// y = x / sqrt(mean(x^2) + eps) as bf16, rstd saved; one warp per row.
// amax (fp8 mode): max |y| folded in, for the quantisation of y.
__global__ void rmsnorm_fwd_kernel(const float* __restrict__ x, int64_t rows, int d,
                                   __nv_bfloat16* __restrict__ y, float* __restrict__ rstd,
                                   unsigned* amax) {
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) {
    if (amax) block_amax_bf16(0.f, amax);
    return;
  }
  const float4* xr = reinterpret_cast<const float4*>(x + r * d);
  float ss = 0.f;
  for (int i = lane; i < d / 4; i += 32) {
    const float4 v = xr[i];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  const float rs = rsqrtf(ss / d + kNormEps);
  uint2* yr = reinterpret_cast<uint2*>(y + r * d);
  float am = 0.f;
  for (int i = lane; i < d / 4; i += 32) {
    const float4 v = xr[i];
    uint2 u;
    u.x = pack_bf16x2(v.x * rs, v.y * rs);
    u.y = pack_bf16x2(v.z * rs, v.w * rs);
    yr[i] = u;
    if (amax) am = fmaxf(am, fmaxf(fmaxf(fabsf(v.x * rs), fabsf(v.y * rs)), fmaxf(fabsf(v.z * rs), fabsf(v.w * rs))));
  }
  if (lane == 0 && rstd) rstd[r] = rs;
  if (amax) block_amax_bf16(am, amax);
}

// dx = dres + r * (dh - y * mean(dh * y)) with y = x * r the norm's output,
// read as the bf16 activation the forward saved (the operand the next GEMM
// consumed); fp32 out and a bf16 copy.  One warp per row, two passes over
// dh and y (the second from L1/L2), 16-byte fp32 and 8-byte bf16 accesses.
__global__ void __launch_bounds__(256) rmsnorm_bwd_kernel(
    const __nv_bfloat16* __restrict__ dh, const __nv_bfloat16* __restrict__ y,
    const float* __restrict__ rstd, const float* __restrict__ dres, int64_t rows, int d,
    float* __restrict__ dx, __nv_bfloat16* __restrict__ dx_bf16, unsigned* amax) {
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) {
    if (amax) block_amax_bf16(0.f, amax);
    return;
  }
  const int n4 = d / 4;
  const uint2* gr = reinterpret_cast<const uint2*>(dh + r * d);
  const uint2* yr = reinterpret_cast<const uint2*>(y + r * d);
  float dot = 0.f;
  for (int i = lane; i < n4; i += 32) {
    const uint2 g = gr[i], v = yr[i];
    const float2 g0 = unpack_bf16x2(g.x), g1 = unpack_bf16x2(g.y);
    const float2 y0 = unpack_bf16x2(v.x), y1 = unpack_bf16x2(v.y);
    dot += g0.x * y0.x + g0.y * y0.y + g1.x * y1.x + g1.y * y1.y;
  }
  const float m = warp_sum(dot) / d;
  const float rs = rstd[r];
  const float4* rr = dres ? reinterpret_cast<const float4*>(dres + r * d) : nullptr;
  float4* o = reinterpret_cast<float4*>(dx + r * d);
  uint2* ob = dx_bf16 ? reinterpret_cast<uint2*>(dx_bf16 + r * d) : nullptr;
  float am = 0.f;
  for (int i = lane; i < n4; i += 32) {
    const uint2 g = gr[i], v = yr[i];
    const float2 g0 = unpack_bf16x2(g.x), g1 = unpack_bf16x2(g.y);
    const float2 y0 = unpack_bf16x2(v.x), y1 = unpack_bf16x2(v.y);
    float4 res = rr ? rr[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    res.x += rs * (g0.x - y0.x * m);
    res.y += rs * (g0.y - y0.y * m);
    res.z += rs * (g1.x - y1.x * m);
    res.w += rs * (g1.y - y1.y * m);
    o[i] = res;
    if (ob) ob[i] = make_uint2(pack_bf16x2(res.x, res.y), pack_bf16x2(res.z, res.w));
    if (amax) am = fmaxf(am, fmaxf(fmaxf(fabsf(res.x), fabsf(res.y)), fmaxf(fabsf(res.z), fabsf(res.w))));
  }
  if (amax) block_amax_bf16(am, amax);
}

// ------------------------------------------------------------------ RoPE + QK-norm
// cos/sin table [T][hd/2]: theta_i(pos) = pos * 10000^(-2i/hd), in double;
// the same values again, grouped four pairs at a time per position
// ([hd/8][T][4]), after it.
__global__ void rope_table_kernel(float2* tab, int T, int hd) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int half = hd / 2;
  if (i >= (int64_t)T * half) return;
  const int pos = (int)(i / half), j = (int)(i % half);
  const double th = (double)pos * pow(10000.0, -2.0 * j / hd);
  const float2 v = make_float2((float)cos(th), (float)sin(th));
  tab[i] = v;
  tab[(int64_t)T * half + ((int64_t)(j >> 2) * T + pos) * 4 + (j & 3)] = v;
}

// ------------------------------------------------------------------ cross-entropy
// One CTA (512 threads) per row of logits z[n, V] (bf16, V <= 32768, V % 8 == 0):
// loss_row = lse(z) - z[target];  z <- (softmax(z) - onehot(target)) * inv_n
// in place.  The row stays in registers between the two reductions.
constexpr int kCeThreads = 512;
constexpr int kCeChunks = 8;  // 8 x 8 bf16 per thread -> V <= 32768

__global__ void __launch_bounds__(kCeThreads, 2) ce_fwd_bwd_kernel(__nv_bfloat16* __restrict__ z,
                                                                const int32_t* __restrict__ tgt,
                                                                int V, float inv_n,
                                                                float* __restrict__ loss_rows,
                                                                int* status) {
  __shared__ float red[kCeThreads / 32];
  __shared__ float s_bcast;
  __shared__ float s_zt;
  const int64_t row = blockIdx.x;
  uint4* zr = reinterpret_cast<uint4*>(z + row * (int64_t)V);
  const int nchunk = V / 8;
  int t = tgt[row];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) atomicExch(status, kDevTokenRange);
    t = t < 0 ? 0 : V - 1;
  }
  if (threadIdx.x == 0) s_zt = bf2f(z[row * (int64_t)V + t]);
  uint4 buf[kCeChunks];
  float mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < kCeChunks; ++c) {
    const int idx = threadIdx.x + c * kCeThreads;
    buf[c] = make_uint4(0u, 0u, 0u, 0u);
    if (idx < nchunk) {
      buf[c] = zr[idx];
      const uint32_t u[4] = {buf[c].x, buf[c].y, buf[c].z, buf[c].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = unpack_bf16x2(u[j]);
        mx = fmaxf(mx, fmaxf(f.x, f.y));
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  mx = warp_max(mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int i = 1; i < kCeThreads / 32; ++i) m = fmaxf(m, red[i]);
    s_bcast = m;
  }
  __syncthreads();
  mx = s_bcast;
  // e = exp(z - max), summed in fp32 and kept (as bf16) in place of z, so the
  // gradient pass scales by 1 / sum instead of exponentiating again.
  float se = 0.f;
#pragma unroll
  for (int c = 0; c < kCeChunks; ++c) {
    const int idx = threadIdx.x + c * kCeThreads;
    if (idx < nchunk) {
      const uint32_t u[4] = {buf[c].x, buf[c].y, buf[c].z, buf[c].w};
      uint32_t e[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = unpack_bf16x2(u[j]);
        const float e0 = __expf(f.x - mx), e1 = __expf(f.y - mx);
        se += e0 + e1;
        e[j] = pack_bf16x2(e0, e1);
      }
      buf[c] = make_uint4(e[0], e[1], e[2], e[3]);
    }
  }
  se = warp_sum(se);
  __syncthreads();
  if (lane == 0) red[warp] = se;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < kCeThreads / 32; ++i) s += red[i];
    loss_rows[row] = mx + logf(s) - s_zt;
    s_bcast = 1.f / s;
  }
  __syncthreads();
  const float scale = s_bcast * inv_n;  // softmax = e / sum, then times 1/n
#pragma unroll
  for (int c = 0; c < kCeChunks; ++c) {
    const int idx = threadIdx.x + c * kCeThreads;
    if (idx < nchunk) {
      const uint32_t u[4] = {buf[c].x, buf[c].y, buf[c].z, buf[c].w};
      uint32_t ou[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = unpack_bf16x2(u[j]);
        const int col = idx * 8 + 2 * j;
        const float p0 = f.x * scale - (col == t ? inv_n : 0.f);
        const float p1 = f.y * scale - (col + 1 == t ? inv_n : 0.f);
        ou[j] = pack_bf16x2(p0, p1);
      }
      zr[idx] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
    }
  }
}

// Deterministic mean of per-row losses (one CTA).
__global__ void mean_kernel(const float* __restrict__ v, int64_t n, float* out) {
  __shared__ double red[256];
  double s = 0;
  for (int64_t i = threadIdx.x; i < n; i += 256) s += v[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = (float)(red[0] / (double)n);
}

// ------------------------------------------------------------------ init
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Normal draws by Box-Muller from a counter-based SplitMix64 stream.
__global__ void init_normal_kernel(float* __restrict__ out, int64_t n, uint64_t key, float stdv) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t w1 = splitmix64(key + 2 * (uint64_t)i);
    const uint64_t w2 = splitmix64(key + 2 * (uint64_t)i + 1);
    const double u1 = (double)(w1 >> 11) * 0x1.0p-53;
    const double u2 = (double)(w2 >> 11) * 0x1.0p-53;
    const double z = sqrt(-2.0 * log(1.0 - u1)) * cos(6.283185307179586476925286766559 * u2);
    out[i] = (float)(z * stdv);
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                   int64_t n) {
  const int64_t i4 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  const int64_t base = i4 * 4;
  if (base + 3 < n) {
    const float4 v = reinterpret_cast<const float4*>(in)[i4];
    uint2 u;
    u.x = pack_bf16x2(v.x, v.y);
    u.y = pack_bf16x2(v.z, v.w);
    reinterpret_cast<uint2*>(out)[i4] = u;
  } else {
    for (int64_t i = base; i < n; ++i) out[i] = f2bf(in[i]);
  }
}

// ------------------------------------------------------------------ Muon
// Block matrices of layer l live at l * (10 d^2 + 2 dkv d), in the order
// wq (d x d), wk and wv (dkv x d each; dkv = d with one KV head per query
// head), wo (d x d), wup (4d x d), wdown (d x 4d).
__device__ __forceinline__ void mat_of(int64_t d, int64_t dkv, int j, int64_t* off,
                                       int64_t* size) {
  const int64_t d2 = d * d, kv = dkv * d;
  *off = j == 0 ? 0 : j == 1 ? d2 : j == 2 ? d2 + kv : j == 3 ? d2 + 2 * kv
       : j == 4 ? 2 * d2 + 2 * kv : 6 * d2 + 2 * kv;
  *size = (j == 1 || j == 2) ? kv : (j >= 4 ? 4 * d2 : d2);
}

// M <- mu*M + G over matrix (blockIdx.y = l*6 + j); sumsq[l*6 + j] += ||M||^2.
__global__ void muon_momentum_kernel(float* __restrict__ M, const float* __restrict__ G, int d,
                                     int dkv, float mu, float* __restrict__ sumsq) {
  const int mat = blockIdx.y;
  const int l = mat / 6, j = mat % 6;
  int64_t off, size;
  mat_of(d, dkv, j, &off, &size);
  off += (int64_t)l * (10ll * d * d + 2ll * dkv * d);
  float4* m4 = reinterpret_cast<float4*>(M + off);
  const float4* g4 = reinterpret_cast<const float4*>(G + off);
  float ss = 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < size / 4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 m = m4[i];
    const float4 g = g4[i];
    m.x = mu * m.x + g.x;
    m.y = mu * m.y + g.y;
    m.z = mu * m.z + g.z;
    m.w = mu * m.w + g.w;
    m4[i] = m;
    ss += m.x * m.x + m.y * m.y + m.z * m.z + m.w * m.w;
  }
  __shared__ float red[8];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
    atomicAdd(sumsq + mat, s);
  }
}

// X = bf16(M / (||M|| + eps)) for matrix j of layer blockIdx.y (src at
// src + y*src_stride, dst at dst + y*dst_stride, norm index y*6 + j), same
// orientation: 16-byte fp32 loads, 8-byte bf16 stores, grid-stride.
__global__ void muon_prep_kernel(const float* __restrict__ src, int64_t src_stride, int64_t n4,
                                 __nv_bfloat16* __restrict__ dst, int64_t dst_stride,
                                 const float* __restrict__ sumsq, int j, float eps) {
  const int z = blockIdx.y;
  const float inv = 1.f / (sqrtf(sumsq[z * 6 + j]) + eps);
  const float4* s4 = reinterpret_cast<const float4*>(src + z * src_stride);
  uint2* d2 = reinterpret_cast<uint2*>(dst + z * dst_stride);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = s4[i];
    d2[i] = make_uint2(pack_bf16x2(v.x * inv, v.y * inv), pack_bf16x2(v.z * inv, v.w * inv));
  }
}

// The same, transposed (dst is cols x rows), through 64 x 64 shared tiles:
// each thread reads 16-byte rows of the fp32 source and writes 8-byte runs
// of the bf16 destination (256 threads, 4 passes of 16 rows each way).
__global__ void __launch_bounds__(256) muon_prep_t_kernel(
    const float* __restrict__ src, int64_t src_stride, int rows, int cols,
    __nv_bfloat16* __restrict__ dst, int64_t dst_stride, const float* __restrict__ sumsq, int j,
    float eps) {
  __shared__ float tile[64][65];
  const int z = blockIdx.z;
  const float inv = 1.f / (sqrtf(sumsq[z * 6 + j]) + eps);
  const float* s = src + z * src_stride;
  __nv_bfloat16* dd = dst + z * dst_stride;
  const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int i = ty + 16 * p, r = r0 + i, c = c0 + 4 * tx;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rows && c < cols) v = *reinterpret_cast<const float4*>(s + (int64_t)r * cols + c);
    tile[i][4 * tx] = v.x;
    tile[i][4 * tx + 1] = v.y;
    tile[i][4 * tx + 2] = v.z;
    tile[i][4 * tx + 3] = v.w;
  }
  __syncthreads();
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int i = ty + 16 * p;  // destination row c0 + i, columns r0 + 4 tx ..
    const int r = c0 + i, c = r0 + 4 * tx;
    if (r < cols && c < rows)
      *reinterpret_cast<uint2*>(dd + (int64_t)r * rows + c) =
          make_uint2(pack_bf16x2(tile[4 * tx][i] * inv, tile[4 * tx + 1][i] * inv),
                     pack_bf16x2(tile[4 * tx + 2][i] * inv, tile[4 * tx + 3][i] * inv));
  }
}

// W <- W - lr * X and its bf16 copy refreshed, same orientation, per layer
// blockIdx.y: 16-byte fp32, 8-byte bf16 accesses, grid-stride.
__global__ void muon_apply_kernel(float* __restrict__ W, __nv_bfloat16* __restrict__ Wb,
                                  int64_t w_stride, int64_t n4, const __nv_bfloat16* __restrict__ X,
                                  int64_t x_stride, float lr) {
  const int z = blockIdx.y;
  float4* w4 = reinterpret_cast<float4*>(W + z * w_stride);
  uint2* wb2 = reinterpret_cast<uint2*>(Wb + z * w_stride);
  const uint2* x2 = reinterpret_cast<const uint2*>(X + z * x_stride);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 w = w4[i];
    const uint2 x = x2[i];
    const float2 x01 = unpack_bf16x2(x.x), x23 = unpack_bf16x2(x.y);
    w.x -= lr * x01.x;
    w.y -= lr * x01.y;
    w.z -= lr * x23.x;
    w.w -= lr * x23.y;
    w4[i] = w;
    wb2[i] = make_uint2(pack_bf16x2(w.x, w.y), pack_bf16x2(w.z, w.w));
  }
}

// The same with X stored transposed (cols x rows): X staged through a 64 x 64
// shared tile, W (rows x cols) updated in 16-byte runs.
__global__ void __launch_bounds__(256) muon_apply_t_kernel(
    float* __restrict__ W, __nv_bfloat16* __restrict__ Wb, int64_t w_stride, int rows, int cols,
    const __nv_bfloat16* __restrict__ X, int64_t x_stride, float lr) {
  __shared__ float tile[64][65];
  const int z = blockIdx.z;
  float* w = W + z * w_stride;
  __nv_bfloat16* wb = Wb + z * w_stride;
  const __nv_bfloat16* x = X + z * x_stride;
  const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  // X rows c0 .. c0 + 63 (W's columns), X columns r0 .. r0 + 63 (W's rows).
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int i = ty + 16 * p, xr = c0 + i, xc = r0 + 4 * tx;
    uint2 u = make_uint2(0u, 0u);
    if (xr < cols && xc < rows) u = *reinterpret_cast<const uint2*>(x + (int64_t)xr * rows + xc);
    const float2 a0 = unpack_bf16x2(u.x), a1 = unpack_bf16x2(u.y);
    tile[i][4 * tx] = a0.x;
    tile[i][4 * tx + 1] = a0.y;
    tile[i][4 * tx + 2] = a1.x;
    tile[i][4 * tx + 3] = a1.y;
  }
  __syncthreads();
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int i = ty + 16 * p, r = r0 + i, c = c0 + 4 * tx;
    if (r < rows && c < cols) {
      float4 v = *reinterpret_cast<float4*>(w + (int64_t)r * cols + c);
      v.x -= lr * tile[4 * tx][i];
      v.y -= lr * tile[4 * tx + 1][i];
      v.z -= lr * tile[4 * tx + 2][i];
      v.w -= lr * tile[4 * tx + 3][i];
      *reinterpret_cast<float4*>(w + (int64_t)r * cols + c) = v;
      *reinterpret_cast<uint2*>(wb + (int64_t)r * cols + c) =
          make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
  }
}

// Frobenius norms of a bf16 stack (count matrices of n elements) for the
// standalone Newton-Schulz op.
__global__ void sumsq_bf16_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, float* out) {
  const __nv_bfloat16* p = x + (int64_t)blockIdx.y * n;
  float ss = 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = bf2f(p[i]);
    ss += v * v;
  }
  __shared__ float red[8];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
    atomicAdd(out + blockIdx.y, s);
  }
}

// y = bf16(x * inv_norm) (optionally transposed), per matrix blockIdx.z.
__global__ void scale_bf16_kernel(const __nv_bfloat16* __restrict__ x, int rows, int cols,
                                  int transpose, const float* __restrict__ sumsq, float eps,
                                  __nv_bfloat16* __restrict__ y) {
  __shared__ float tile[32][33];
  const int z = blockIdx.z;
  const int64_t n = (int64_t)rows * cols;
  const float inv = sumsq ? 1.f / (sqrtf(sumsq[z]) + eps) : 1.f;
  const __nv_bfloat16* s = x + z * n;
  __nv_bfloat16* dd = y + z * n;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < rows && c < cols) ? bf2f(s[(int64_t)r * cols + c]) * inv : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    if (!transpose) {
      const int r = r0 + i, c = c0 + threadIdx.x;
      if (r < rows && c < cols) dd[(int64_t)r * cols + c] = f2bf(tile[i][threadIdx.x]);
    } else {
      const int r = c0 + i, c = r0 + threadIdx.x;
      if (r < cols && c < rows) dd[(int64_t)r * rows + c] = f2bf(tile[threadIdx.x][i]);
    }
  }
}

inline unsigned blocks_for(int64_t threads, int per_block) {
  return (unsigned)((threads + per_block - 1) / per_block);
}

}  // namespace

// ------------------------------------------------------------------ launchers
nc_status embed_gather(const int32_t* tok, int64_t n, const float* E, int V, int d, float* x,
                       int* status, cudaStream_t s, Profiler* prof) {
  Probe probe(prof, s, "embed_gather", 0.0, n * (8.0 * d + 4.0));
  embed_gather_kernel<<<blocks_for(n * 32, 256), 256, 0, s>>>(tok, n, E, V, d, x, status);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status embed_scatter(const int32_t* tok, int64_t n, const float* dx, int V, int d, float* dE,
                        cudaStream_t s, Profiler* prof) {
  Probe probe(prof, s, "embed_scatter", 0.0, n * (8.0 * d + 4.0));
  embed_scatter_kernel<<<blocks_for(n * 32, 256), 256, 0, s>>>(tok, n, dx, V, d, dE);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status rmsnorm_fwd(const float* x, int64_t rows, int d, void* y, float* rstd, cudaStream_t s,
                      Profiler* prof, unsigned* amax) {
  if (d % 4) return fail(NC_ERR_INVALID_ARG, "rmsnorm: width must be a multiple of 4");
  Probe probe(prof, s, "rmsnorm_fwd", 0.0, rows * (6.0 * d + 4.0));
  rmsnorm_fwd_kernel<<<blocks_for(rows * 32, 256), 256, 0, s>>>(x, rows, d, (__nv_bfloat16*)y,
                                                                 rstd, amax);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status rmsnorm_bwd(const void* dh, const void* y, const float* rstd, const float* dres,
                      int64_t rows, int d, float* dx, void* dx_bf16, cudaStream_t s,
                      Profiler* prof, unsigned* amax) {
  if (d % 4) return fail(NC_ERR_UNSUPPORTED, "rmsnorm_bwd: width must be a multiple of 4");
  if (amax && !dx_bf16) return fail(NC_ERR_INVALID_ARG, "rmsnorm_bwd: amax is of the bf16 copy");
  Probe probe(prof, s, "rmsnorm_bwd", 0.0,
              rows * ((2.0 + 2.0 + (dres ? 4.0 : 0.0) + 4.0 + (dx_bf16 ? 2.0 : 0.0)) * d + 4.0));
  rmsnorm_bwd_kernel<<<blocks_for(rows * 32, 256), 256, 0, s>>>(
      (const __nv_bfloat16*)dh, (const __nv_bfloat16*)y, rstd, dres, rows, d, dx,
      (__nv_bfloat16*)dx_bf16, amax);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status rope_table(float2* tab, int T, int hd, cudaStream_t s) {
  rope_table_kernel<<<blocks_for((int64_t)T * hd / 2, 256), 256, 0, s>>>(tab, T, hd);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status ce_fwd_bwd(void* z, const int32_t* tgt, int64_t n, int V, float inv_n, float* loss_rows,
                     int* status, cudaStream_t s, Profiler* prof) {
  if (V % 8 || V > kCeThreads * kCeChunks * 8)
    return fail(NC_ERR_UNSUPPORTED, "cross-entropy: vocab must be a multiple of 8 and <= 32768");
  if (n >= (1ll << 31)) return fail(NC_ERR_INVALID_ARG, "cross-entropy: too many rows");
  Probe probe(prof, s, "ce_fwd_bwd", 0.0, n * (4.0 * V + 8.0));
  ce_fwd_bwd_kernel<<<(unsigned)n, kCeThreads, 0, s>>>((__nv_bfloat16*)z, tgt, V, inv_n, loss_rows, status);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status loss_mean(const float* loss_rows, int64_t n, float* loss_out, cudaStream_t s) {
  mean_kernel<<<1, 256, 0, s>>>(loss_rows, n, loss_out);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status init_normal(float* out, int64_t n, uint64_t key, float stdv, cudaStream_t s) {
  const unsigned grid = (unsigned)std::min<int64_t>(blocks_for(n, 256), 148 * 16);
  init_normal_kernel<<<grid, 256, 0, s>>>(out, n, key, stdv);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

// 2^x through exp2_fma2, two elements per thread (the softmax's FMA-pipe
// exponential, run on a plain array so that its error can be measured).
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_fma2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_fma2(make_float2(x[i], 0.f)).x;
  }
}

nc_status exp2_poly(const float* x, float* y, int64_t n, cudaStream_t s) {
  exp2_poly_kernel<<<blocks_for((n + 1) / 2, 256), 256, 0, s>>>(x, y, n);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

// ------------------------------------------------------------------ fp8 (E4M3)
// One dynamic scale per tensor: s = 448 / amax(|x|) (1 when x is all zero),
// q = E4M3(x * s) rounded to nearest even and saturated to +-448.  x is a
// rows x cols matrix of bf16 (activations, gradients) or fp32 (weights) with
// row stride ld; cols a multiple of 8.

__device__ __forceinline__ float fp8_src(const void* x, bool bf16, int64_t i) {
  return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(x)[i]) : static_cast<const float*>(x)[i];
}

// Eight consecutive elements of one row as floats (16- or 32-byte loads).
__device__ __forceinline__ void fp8_load8(const void* x, bool bf16, int64_t i, float (&v)[8]) {
  if (bf16) {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf16x2(w[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(x) + i);
    const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(x) + i + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// amax over the matrix into *amax_bits (the bits of a non-negative float, so
// integer max orders them; zeroed by the caller).  NaN elements are skipped,
// as fmaxf does.
__global__ void __launch_bounds__(256) fp8_amax_kernel(const void* __restrict__ x, int bf16, int64_t rows,
                                                       int cols, int64_t ld, unsigned* amax_bits) {
  const int cv = cols / 8;
  const int64_t total = rows * cv;
  float m = 0.f;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = u / cv;
    float v[8];
    fp8_load8(x, bf16 != 0, r * ld + (u - r * cv) * 8, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
  }
  m = warp_max(m);
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
    atomicMax(amax_bits, __float_as_uint(m));
  }
}

__device__ __forceinline__ float fp8_scale_of(const unsigned* amax_bits) {
  const float amax = __uint_as_float(*amax_bits);
  return amax > 0.f ? 448.f / amax : 1.f;
}

// Two floats to two E4M3 bytes (the first in the low byte).
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// q[r * ldq + c] = E4M3(x[r, c] * s), eight elements per thread.
__global__ void __launch_bounds__(256) fp8_quant_kernel(const void* __restrict__ x, int bf16, int64_t rows,
                                                        int cols, int64_t ld, const unsigned* amax_bits,
                                                        uint8_t* __restrict__ q, int64_t ldq, float* scale) {
  const float s = fp8_scale_of(amax_bits);
  if (blockIdx.x == 0 && threadIdx.x == 0 && scale) *scale = s;
  const int cv = cols / 8;
  const int64_t total = rows * cv;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = u / cv;
    const int64_t c = (u - r * cv) * 8;
    float v[8];
    fp8_load8(x, bf16 != 0, r * ld + c, v);
    uint2 o;
    o.x = e4m3x2(v[0] * s, v[1] * s) | (e4m3x2(v[2] * s, v[3] * s) << 16);
    o.y = e4m3x2(v[4] * s, v[5] * s) | (e4m3x2(v[6] * s, v[7] * s) << 16);
    *reinterpret_cast<uint2*>(q + r * ldq + c) = o;
  }
}

// The transpose: q[c * ldq + r] = E4M3(x[r, c] * s), through 64 x 64 tiles in
// shared memory (rows a multiple of 8 as well).
__global__ void __launch_bounds__(256) fp8_quant_t_kernel(const void* __restrict__ x, int bf16, int64_t rows,
                                                          int cols, int64_t ld, const unsigned* amax_bits,
                                                          uint8_t* __restrict__ q, int64_t ldq, float* scale) {
  __shared__ uint8_t tile[64][64 + 8];
  const float s = fp8_scale_of(amax_bits);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && scale) *scale = s;
  const int64_t r0 = (int64_t)blockIdx.y * 64;
  const int c0 = blockIdx.x * 64;
  // Load: 64 rows x 8 groups of 8 columns, one group per thread per pass.
  for (int u = threadIdx.x; u < 64 * 8; u += blockDim.x) {
    const int rr = u >> 3, cg = (u & 7) * 8;
    const int64_t r = r0 + rr;
    const int c = c0 + cg;
    float v[8];
    if (r < rows && c < cols) {
      fp8_load8(x, bf16 != 0, r * ld + c, v);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const uint32_t b = e4m3x2(v[j] * s, v[j + 1] * s);
      tile[cg + j][rr] = (uint8_t)(b & 0xffu);
      tile[cg + j + 1][rr] = (uint8_t)(b >> 8);
    }
  }
  __syncthreads();
  // Store: 64 output rows (columns of x) x 8 groups of 8 bytes.
  for (int u = threadIdx.x; u < 64 * 8; u += blockDim.x) {
    const int cc = u >> 3, rg = (u & 7) * 8;
    const int c = c0 + cc;
    const int64_t r = r0 + rg;
    if (c < cols && r < rows) {
      uint2 o;
      o.x = (uint32_t)tile[cc][rg] | ((uint32_t)tile[cc][rg + 1] << 8) | ((uint32_t)tile[cc][rg + 2] << 16) |
            ((uint32_t)tile[cc][rg + 3] << 24);
      o.y = (uint32_t)tile[cc][rg + 4] | ((uint32_t)tile[cc][rg + 5] << 8) | ((uint32_t)tile[cc][rg + 6] << 16) |
            ((uint32_t)tile[cc][rg + 7] << 24);
      *reinterpret_cast<uint2*>(q + (int64_t)c * ldq + r) = o;
    }
  }
}

// Both layouts of a bf16 matrix in one pass: q[r * cols + c] and
// qT[c * rows + r] (either may be null), through 64 x 128 tiles; rows and
// cols multiples of 8.  The scale goes to s0 and, when given, s1.
__global__ void __launch_bounds__(256) fp8_quant2_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                         int cols, int64_t ld, const unsigned* amax_bits,
                                                         uint8_t* __restrict__ q, uint8_t* __restrict__ qT,
                                                         float* s0, float* s1) {
  __shared__ uint8_t tile[128][65];  // [column][row]; the odd row length spreads the byte writes over banks
  const float s = fp8_scale_of(amax_bits);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    if (s0) *s0 = s;
    if (s1) *s1 = s;
  }
  const int64_t r0 = (int64_t)blockIdx.y * 64;
  const int c0 = blockIdx.x * 128;
  for (int u = threadIdx.x; u < 64 * 16; u += blockDim.x) {
    const int rr = u >> 4, cg = (u & 15) * 8;
    const int64_t r = r0 + rr;
    const int c = c0 + cg;
    uint32_t w0 = 0, w1 = 0;
    if (r < rows && c < cols) {
      float v[8];
      fp8_load8(x, true, r * ld + c, v);
      w0 = e4m3x2(v[0] * s, v[1] * s) | (e4m3x2(v[2] * s, v[3] * s) << 16);
      w1 = e4m3x2(v[4] * s, v[5] * s) | (e4m3x2(v[6] * s, v[7] * s) << 16);
      if (q) *reinterpret_cast<uint2*>(q + r * cols + c) = make_uint2(w0, w1);
    }
    if (qT) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        tile[cg + j][rr] = (uint8_t)(w0 >> (8 * j));
        tile[cg + 4 + j][rr] = (uint8_t)(w1 >> (8 * j));
      }
    }
  }
  if (!qT) return;
  __syncthreads();
  for (int u = threadIdx.x; u < 128 * 8; u += blockDim.x) {
    const int cc = u >> 3, rg = (u & 7) * 8;
    const int c = c0 + cc;
    const int64_t r = r0 + rg;
    if (c < cols && r < rows) {
      uint32_t o0 = 0, o1 = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        o0 |= (uint32_t)tile[cc][rg + j] << (8 * j);
        o1 |= (uint32_t)tile[cc][rg + 4 + j] << (8 * j);
      }
      *reinterpret_cast<uint2*>(qT + (int64_t)c * rows + r) = make_uint2(o0, o1);
    }
  }
}

nc_status fp8_quantize2(const void* x, int64_t rows, int cols, int64_t ld, uint8_t* q, uint8_t* qT, float* s0,
                        float* s1, unsigned* amax_scratch, bool amax_ready, cudaStream_t s, Profiler* prof) {
  Probe probe(prof, s, "fp8_quantize", 0.0,
              (double)rows * cols * ((amax_ready ? 1.0 : 2.0) * 2 + (q ? 1.0 : 0.0) + (qT ? 1.0 : 0.0)));
  if (!amax_ready) {
    NC_CUDA_TRY(cudaMemsetAsync(amax_scratch, 0, sizeof(unsigned), s));
    const int64_t units = rows * (cols / 8);
    const unsigned g = (unsigned)std::min<int64_t>((units + 255) / 256, 8LL * num_sms());
    fp8_amax_kernel<<<g, 256, 0, s>>>(x, 1, rows, cols, ld, amax_scratch);
    NC_CUDA_TRY(cudaGetLastError());
  }
  dim3 grid((unsigned)((cols + 127) / 128), (unsigned)((rows + 63) / 64));
  fp8_quant2_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), rows, cols, ld, amax_scratch, q,
                                         qT, s0, s1);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status fp8_quantize(const void* x, bool bf16, int64_t rows, int cols, int64_t ld, bool transpose,
                       uint8_t* q, int64_t ldq, float* scale, unsigned* amax_scratch, cudaStream_t s,
                       Profiler* prof) {
  Probe probe(prof, s, "fp8_quantize", 0.0, (double)rows * cols * (2.0 * (bf16 ? 2 : 4) + 1.0));
  NC_CUDA_TRY(cudaMemsetAsync(amax_scratch, 0, sizeof(unsigned), s));
  const int64_t units = rows * (cols / 8);
  const unsigned g = (unsigned)std::min<int64_t>((units + 255) / 256, 8LL * num_sms());
  fp8_amax_kernel<<<g, 256, 0, s>>>(x, bf16 ? 1 : 0, rows, cols, ld, amax_scratch);
  NC_CUDA_TRY(cudaGetLastError());
  if (transpose) {
    dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64));
    fp8_quant_t_kernel<<<grid, 256, 0, s>>>(x, bf16 ? 1 : 0, rows, cols, ld, amax_scratch, q, ldq, scale);
  } else {
    fp8_quant_kernel<<<g, 256, 0, s>>>(x, bf16 ? 1 : 0, rows, cols, ld, amax_scratch, q, ldq, scale);
  }
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status f32_to_bf16(const float* in, void* out, int64_t n, cudaStream_t s, Profiler* prof) {
  Probe probe(prof, s, "f32_to_bf16", 0.0, n * 6.0);
  f32_to_bf16_kernel<<<blocks_for((n + 3) / 4, 256), 256, 0, s>>>(in, (__nv_bfloat16*)out, n);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status muon_momentum(float* M, const float* G, int L, int d, int dkv, float mu, float* sumsq,
                        cudaStream_t s, Profiler* prof) {
  Probe probe(prof, s, "muon_momentum", 0.0,
              12.0 * L * (10.0 * d * d + 2.0 * dkv * (double)d));
  dim3 grid(64, 6 * L);
  muon_momentum_kernel<<<grid, 256, 0, s>>>(M, G, d, dkv, mu, sumsq);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status muon_prep(const float* src, int64_t src_stride, int rows, int cols, int transpose,
                    void* dst, int64_t dst_stride, const float* sumsq, int j, int L,
                    cudaStream_t s, Profiler* prof) {
  if (rows % 4 || cols % 4 || src_stride % 4 || dst_stride % 4)
    return fail(NC_ERR_INVALID_ARG, "muon_prep: dims and strides must be multiples of 4");
  Probe probe(prof, s, "muon_prep", 0.0, (double)L * rows * cols * 6.0);
  if (transpose) {
    dim3 grid((cols + 63) / 64, (rows + 63) / 64, L);
    muon_prep_t_kernel<<<grid, 256, 0, s>>>(src, src_stride, rows, cols, (__nv_bfloat16*)dst,
                                            dst_stride, sumsq, j, 1e-7f);
  } else {
    const int64_t n4 = (int64_t)rows * cols / 4;
    dim3 grid((unsigned)std::min<int64_t>(blocks_for(n4, 256), 4 * num_sms() / std::max(L, 1) + 1), L);
    muon_prep_kernel<<<grid, 256, 0, s>>>(src, src_stride, n4, (__nv_bfloat16*)dst, dst_stride,
                                          sumsq, j, 1e-7f);
  }
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status muon_apply(float* W, void* Wb, int64_t w_stride, int rows, int cols, int transpose,
                     const void* X, int64_t x_stride, float lr, int L, cudaStream_t s,
                     Profiler* prof) {
  if (rows % 4 || cols % 4 || w_stride % 4 || x_stride % 4)
    return fail(NC_ERR_INVALID_ARG, "muon_apply: dims and strides must be multiples of 4");
  Probe probe(prof, s, "muon_apply", 0.0, (double)L * rows * cols * 12.0);
  if (transpose) {
    dim3 grid((cols + 63) / 64, (rows + 63) / 64, L);
    muon_apply_t_kernel<<<grid, 256, 0, s>>>(W, (__nv_bfloat16*)Wb, w_stride, rows, cols,
                                             (const __nv_bfloat16*)X, x_stride, lr);
  } else {
    const int64_t n4 = (int64_t)rows * cols / 4;
    dim3 grid((unsigned)std::min<int64_t>(blocks_for(n4, 256), 4 * num_sms() / std::max(L, 1) + 1), L);
    muon_apply_kernel<<<grid, 256, 0, s>>>(W, (__nv_bfloat16*)Wb, w_stride, n4,
                                           (const __nv_bfloat16*)X, x_stride, lr);
  }
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status sumsq_bf16(const void* x, int64_t n, int count, float* out, cudaStream_t s,
                     Profiler* prof) {
  Probe probe(prof, s, "ns_sumsq", 0.0, (double)count * n * 2.0);
  dim3 grid((unsigned)std::min<int64_t>(blocks_for(n, 256), 64), count);
  sumsq_bf16_kernel<<<grid, 256, 0, s>>>((const __nv_bfloat16*)x, n, out);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

nc_status scale_bf16(const void* x, int rows, int cols, int transpose, const float* sumsq,
                     float eps, void* y, int count, cudaStream_t s, Profiler* prof) {
  Probe probe(prof, s, "ns_scale", 0.0, (double)count * rows * cols * 4.0);
  dim3 grid((cols + 31) / 32, (rows + 31) / 32, count);
  scale_bf16_kernel<<<grid, dim3(32, 8), 0, s>>>((const __nv_bfloat16*)x, rows, cols, transpose,
                                                 sumsq, eps, (__nv_bfloat16*)y);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

// ------------------------------------------------------------------ AdamW
namespace {

// One AdamW step on n contiguous fp32 elements (guide, section "2. Otimizador
// Muon": the embeddings and lm_head take AdamW), decoupled weight decay and
// bias correction ic1 = 1/(1 - b1^t), ic2 = 1/(1 - b2^t):
//   m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
//   W <- W - lr ((m ic1) / (sqrt(v ic2) + eps) + wd W);  Wb <- bf16(W) if given.
// Four elements per thread (16-byte accesses), grid-stride.
__device__ __forceinline__ float adamw_elem(float& w, float& m, float& v, float g, float lr, float b1,
                                            float b2, float eps, float wd, float ic1, float ic2) {
  m = b1 * m + (1.f - b1) * g;
  v = b2 * v + (1.f - b2) * g * g;
  w -= lr * ((m * ic1) / (sqrtf(v * ic2) + eps) + wd * w);
  return w;
}

__global__ void adamw_kernel(float* __restrict__ W, __nv_bfloat16* __restrict__ Wb,
                             float* __restrict__ M, float* __restrict__ Vs,
                             const float* __restrict__ G, int64_t n, float lr, float b1, float b2,
                             float eps, float wd, float ic1, float ic2) {
  const int64_t n4 = n / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 w = reinterpret_cast<float4*>(W)[i];
    float4 m = reinterpret_cast<float4*>(M)[i];
    float4 v = reinterpret_cast<float4*>(Vs)[i];
    const float4 g = reinterpret_cast<const float4*>(G)[i];
    adamw_elem(w.x, m.x, v.x, g.x, lr, b1, b2, eps, wd, ic1, ic2);
    adamw_elem(w.y, m.y, v.y, g.y, lr, b1, b2, eps, wd, ic1, ic2);
    adamw_elem(w.z, m.z, v.z, g.z, lr, b1, b2, eps, wd, ic1, ic2);
    adamw_elem(w.w, m.w, v.w, g.w, lr, b1, b2, eps, wd, ic1, ic2);
    reinterpret_cast<float4*>(W)[i] = w;
    reinterpret_cast<float4*>(M)[i] = m;
    reinterpret_cast<float4*>(Vs)[i] = v;
    if (Wb) reinterpret_cast<uint2*>(Wb)[i] = make_uint2(pack_bf16x2(w.x, w.y), pack_bf16x2(w.z, w.w));
  }
  for (int64_t i = n4 * 4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float w = adamw_elem(W[i], M[i], Vs[i], G[i], lr, b1, b2, eps, wd, ic1, ic2);
    if (Wb) Wb[i] = f2bf(w);
  }
}

}  // namespace

nc_status adamw(float* W, void* Wb, float* m, float* v, const float* g, int64_t n, float lr,
                float b1, float b2, float eps, float wd, int t, cudaStream_t s, Profiler* prof) {
  if (n < 1 || t < 1 || !W || !m || !v || !g) return fail(NC_ERR_INVALID_ARG, "adamw: bad arguments");
  if ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(m) | reinterpret_cast<uintptr_t>(v) |
       reinterpret_cast<uintptr_t>(g) | reinterpret_cast<uintptr_t>(Wb)) & 15)
    return fail(NC_ERR_INVALID_ARG, "adamw: buffers must be 16-byte aligned");
  const double ic1 = 1.0 / (1.0 - std::pow((double)b1, t)), ic2 = 1.0 / (1.0 - std::pow((double)b2, t));
  Probe probe(prof, s, "adamw", 0.0, (double)n * (16.0 + 12.0 + (Wb ? 2.0 : 0.0)));
  const unsigned grid = (unsigned)std::min<int64_t>(blocks_for((n + 3) / 4, 256), 148 * 8);
  adamw_kernel<<<grid, 256, 0, s>>>(W, static_cast<__nv_bfloat16*>(Wb), m, v, g, n, lr, b1, b2, eps, wd,
                                    (float)ic1, (float)ic2);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

}  // namespace nc
