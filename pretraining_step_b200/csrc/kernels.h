// kernels.h -- launchers of the device kernels (host side).  Pointers are
// device pointers; bf16 tensors are passed as void*.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace nc {

// 3-D bf16 TMA tensor map {inner, outer, batch} (element strides ld and
// bstride), box {64, box_outer, 1}, 128-byte swizzle, zero fill out of range.
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t batch, int64_t ld, int64_t bstride, uint32_t box_outer);

// The same for 8-bit elements (fp8 operands): box {128, box_outer, 1}, one
// 128-byte swizzled row of 128 elements per outer index.
bool make_tmap_u8_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t batch, int64_t ld, int64_t bstride, uint32_t box_outer);

// 3-D TMA tensor map of fp32 (f32) or bf16 elements with an explicit box
// {box_inner, box_outer, 1} and swizzle span (0, 32, 64 or 128 bytes).
bool make_tmap_3d(CUtensorMap* m, const void* base, bool f32, uint64_t inner, uint64_t outer,
                  uint64_t batch, int64_t ld, int64_t bstride, uint32_t box_inner, uint32_t box_outer,
                  int swizzle_bytes);

struct GemmLaunch {
  nc_gemm_desc d;
  int* status;             // device status word (may be null)
  const char* tag = "gemm_tc";  // profiler class
  // The output is symmetric (M == N, e.g. X X^T): only the 256 x 256 tiles on
  // or above the diagonal are computed, each off-diagonal one also stored
  // transposed (bf16 store or a*acc + b*aux epilogues, one split, CTA pairs).
  bool symmetric = false;
};
// d.split_k == 0 selects the split automatically (NC_EPI_ACC_F32 only).
nc_status gemm_launch(const GemmLaunch& g, cudaStream_t s, Profiler* prof);

nc_status attention_fwd(const void* q, const void* k, const void* v, int64_t ld, void* o,
                        int64_t ldo, float* lse, int B, int T, int H, int* status, cudaStream_t s,
                        Profiler* prof);
nc_status attention_bwd(const void* q, const void* k, const void* v, int64_t ld, const void* o,
                        const void* dout, int64_t ldo, const float* lse, float* dq, void* dk,
                        void* dv, int64_t ldg, float* delta, int B, int T, int H, int* status,
                        cudaStream_t s, Profiler* prof);
// The tcgen05 backward proper (delta = rowsum(dO * O) precomputed, dq zeroed).
nc_status attention_bwd_tc(const void* q, const void* k, const void* v, int64_t ld,
                           const void* dout, int64_t ldo, const float* lse, const float* delta,
                           float* dq, void* dk, void* dv, int64_t ldg, int B, int T, int H,
                           int* status, cudaStream_t s, Profiler* prof);
// Grouped KV heads (Hkv divides H; q / o / dO / dq rows hold H heads, k / v /
// dk / dv rows Hkv heads) and a left window (query t sees keys
// [t - window, t]; < 0: every key up to t).  The calls above are these with
// Hkv = H, one row stride for q, k and v, and no window.
nc_status attention_fwd_ex(const void* q, int64_t ldq, const void* k, const void* v, int64_t ldkv,
                           void* o, int64_t ldo, float* lse, int B, int T, int H, int Hkv,
                           int window, int* status, cudaStream_t s, Profiler* prof);
nc_status attention_bwd_ex(const void* q, int64_t ldq, const void* k, const void* v, int64_t ldkv,
                           const void* o, const void* dout, int64_t ldo, const float* lse,
                           float* dq, void* dk, void* dv, int64_t ldg, float* delta, int B, int T,
                           int H, int Hkv, int window, int* status, cudaStream_t s, Profiler* prof);
// ds non-null: the persistent key-side kernel stores every dS^T tile (bf16
// [B*H][T keys][T queries], row stride ld_ds, a multiple of 8 >= T) instead
// of computing dQ, dq is not touched, and dK leaves through the k-side RoPE
// + QK-norm backward (rope_tab: rope_table()'s buffer for rope_T >= T
// positions; rstd_k non-null; dk, dv 32-byte aligned with ldg a multiple of
// 16); attention_dq_ex then contracts dS^T with K.
nc_status attention_bwd_tc_ex(const void* q, int64_t ldq, const void* k, const void* v, int64_t ldkv,
                              const void* dout, int64_t ldo, const float* lse, const float* delta,
                              float* dq, void* dk, void* dv, int64_t ldg, int B, int T, int H,
                              int Hkv, int window, const float2* rope_tab, int rope_T,
                              const float* rstd_k, void* ds, int64_t ld_ds, int* status,
                              cudaStream_t s, Profiler* prof);
// dQ = dS K / sqrt(128) from the stored dS^T tiles, through the backward of
// the q-side RoPE + QK-norm (yhat: the saved normalised q, row stride ldy;
// rstd_q [B*T, H]), written as bf16 rows of stride ldo (the q slice of the
// q|k|v gradient; yhat and out 32-byte aligned, ldy and ldo multiples of 16).
// rope_tab: rope_table()'s buffer for rope_T >= T positions.
nc_status attention_dq_ex(const void* ds, int64_t ld_ds, const void* k, int64_t ldkv, int B, int T,
                          int H, int Hkv, int window, const void* yhat, int64_t ldy,
                          const float* rstd_q, const float2* rope_tab, int rope_T, void* out,
                          int64_t ldo, int* status, cudaStream_t s, Profiler* prof);
// The model's attention backward: the row sums D, the key-side kernel with
// the k-side RoPE + QK-norm backward in its dK epilogue and dS^T stored to
// ds, then the query-side kernel with the q-side backward in its epilogue.
// dq_out, dk, dv: the q, k, v slices of the bf16 q|k|v gradient.
nc_status attention_bwd_model(const void* q, int64_t ldq, const void* k, const void* v,
                              int64_t ldkv, const void* o, const void* dout, int64_t ldo,
                              const float* lse, float* delta, void* ds, int64_t ld_ds,
                              void* dq_out, void* dk, void* dv, int64_t ldg, int B, int T, int H,
                              int Hkv, int window, const float2* rope_tab, int rope_T,
                              const float* rstd_q, const float* rstd_k, int* status, cudaStream_t s,
                              Profiler* prof);

nc_status embed_gather(const int32_t* tok, int64_t n, const float* E, int V, int d, float* x,
                       int* status, cudaStream_t s, Profiler* prof);
nc_status embed_scatter(const int32_t* tok, int64_t n, const float* dx, int V, int d, float* dE,
                        cudaStream_t s, Profiler* prof);
// amax (fp8 mode; zeroed by the caller): max |y| of the bf16 output folded in.
nc_status rmsnorm_fwd(const float* x, int64_t rows, int d, void* y, float* rstd, cudaStream_t s,
                      Profiler* prof, unsigned* amax = nullptr);
// y: the norm's saved bf16 output (x * rstd as the forward stored it).
nc_status rmsnorm_bwd(const void* dh, const void* y, const float* rstd, const float* dres,
                      int64_t rows, int d, float* dx, void* dx_bf16, cudaStream_t s,
                      Profiler* prof, unsigned* amax = nullptr);
// RoPE cos/sin for positions [0, T): tab[pos * hd/2 + i] = (cos, sin) of
// pos * 10000^(-2i/hd); then, from tab + T * hd/2, the same values grouped
// for 32-byte loads of four consecutive pairs of one position:
// [(i / 4) * T + pos] * 4 + i % 4.  tab holds T * hd floats (two float2 per pair).
nc_status rope_table(float2* tab, int T, int hd, cudaStream_t s);
// Softmax cross-entropy of n rows of bf16 logits z [n, V]: loss_rows[i] =
// lse(z_i) - z_i[tgt_i]; z is overwritten by its gradient (softmax - onehot)
// * inv_n (inv_n: 1 / the rows of the whole batch when z is one chunk of it).
nc_status ce_fwd_bwd(void* z, const int32_t* tgt, int64_t n, int V, float inv_n, float* loss_rows,
                     int* status, cudaStream_t s, Profiler* prof);
// *loss_out = mean of loss_rows[0, n).
nc_status loss_mean(const float* loss_rows, int64_t n, float* loss_out, cudaStream_t s);
nc_status init_normal(float* out, int64_t n, uint64_t key, float stdv, cudaStream_t s);
nc_status f32_to_bf16(const float* in, void* out, int64_t n, cudaStream_t s, Profiler* prof);
// E4M3 quantisation of a rows x cols matrix (bf16, or fp32 when !bf16; row
// stride ld, cols a multiple of 8, rows too when transposing) with one
// dynamic scale s = 448 / amax, written to *scale: q[r * ldq + c] (or the
// transpose, q[c * ldq + r]) = E4M3(x[r, c] * s).  amax_scratch: one device
// word of scratch.
nc_status fp8_quantize(const void* x, bool bf16, int64_t rows, int cols, int64_t ld, bool transpose,
                       uint8_t* q, int64_t ldq, float* scale, unsigned* amax_scratch, cudaStream_t s,
                       Profiler* prof);
// The same for a bf16 matrix in both layouts at once (q [rows, cols] and qT
// [cols, rows], either may be null; rows and cols multiples of 8), the
// scale written to s0 and, when not null, s1.  amax_ready: *amax_scratch
// already holds max |x| (its producer folded it in), so x is read once.
nc_status fp8_quantize2(const void* x, int64_t rows, int cols, int64_t ld, uint8_t* q, uint8_t* qT, float* s0,
                        float* s1, unsigned* amax_scratch, bool amax_ready, cudaStream_t s, Profiler* prof);
// y[i] = 2^x[i] by exp2_fma2 (exp2_poly.cuh), the softmax's FMA-pipe exponential.
nc_status exp2_poly(const float* x, float* y, int64_t n, cudaStream_t s);
// Momentum and per-matrix squared norms over the 6*L block matrices; dkv is
// the width of wk and wv (d with one KV head per query head).
nc_status muon_momentum(float* M, const float* G, int L, int d, int dkv, float mu, float* sumsq,
                        cudaStream_t s, Profiler* prof);
nc_status muon_prep(const float* src, int64_t src_stride, int rows, int cols, int transpose,
                    void* dst, int64_t dst_stride, const float* sumsq, int j, int L,
                    cudaStream_t s, Profiler* prof);
nc_status muon_apply(float* W, void* Wb, int64_t w_stride, int rows, int cols, int transpose,
                     const void* X, int64_t x_stride, float lr, int L, cudaStream_t s,
                     Profiler* prof);
// AdamW step t on n fp32 elements in place; Wb (bf16 copy) refreshed when
// not null.
nc_status adamw(float* W, void* Wb, float* m, float* v, const float* g, int64_t n, float lr,
                float b1, float b2, float eps, float wd, int t, cudaStream_t s, Profiler* prof);
nc_status sumsq_bf16(const void* x, int64_t n, int count, float* out, cudaStream_t s,
                     Profiler* prof);
nc_status scale_bf16(const void* x, int rows, int cols, int transpose, const float* sumsq,
                     float eps, void* y, int count, cudaStream_t s, Profiler* prof);

// Newton-Schulz on a wide bf16 stack X[count][m][n] (m <= n), in place in
// x0 (result lands back in x0); ws: 2*count*m*m + count*m*n bf16 elements.
nc_status newton_schulz_wide(void* x0, int count, int m, int n, int steps, void* ws,
                             int* status, cudaStream_t s, Profiler* prof);

}  // namespace nc
