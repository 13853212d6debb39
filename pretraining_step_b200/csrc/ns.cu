// ns.cu -- the Newton-Schulz engine of the Muon step.
//
// Five quintic steps on a stack of wide bf16 matrices X [count][m][n]
// (m <= n), every product a batched tcgen05 GEMM over the whole stack:
//   A = X X^T                        (m x m, K = n)
//   B = b A + c A A                  (A is symmetric, so A A = A A^T; the
//                                     b A term is fused into the epilogue)
//   X = a X + B X                    (X read MN-major as the B operand; the
//                                     a X term is fused into the epilogue)
// The left-hand form with the m x m Gram is the page's X = a X + X B on X^T
// (X p(X^T X) = p(X X^T) X), chosen because m <= n keeps the Gram small.

#include <utility>

#include "common.cuh"
#include "kernels.h"

namespace nc {

namespace {
constexpr float kNsA = 3.4445f, kNsB = -4.7750f, kNsC = 2.0315f;
}

nc_status newton_schulz_wide(void* x0, int count, int m, int n, int steps, void* ws, int* status,
                             cudaStream_t s, Profiler* prof) {
  if (count < 1 || m < 1 || n < m || steps < 0 || !x0 || !ws)
    return fail(NC_ERR_INVALID_ARG, "newton_schulz: expects count >= 1 and m <= n");
  __nv_bfloat16* A = static_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* Bm = A + (int64_t)count * m * m;
  __nv_bfloat16* x1 = Bm + (int64_t)count * m * m;
  __nv_bfloat16* X = static_cast<__nv_bfloat16*>(x0);
  __nv_bfloat16* Y = x1;
  const int64_t mm = (int64_t)m * m, mn = (int64_t)m * n;
  for (int it = 0; it < steps; ++it) {
    GemmLaunch g{};
    g.status = status;
    g.tag = "gemm_ns";
    // A = X X^T
    g.d = nc_gemm_desc{};
    g.d.M = m; g.d.N = m; g.d.K = n; g.d.batch = count;
    g.d.A = X; g.d.lda = n; g.d.stride_a = mn; g.d.a_kmajor = 1;
    g.d.B = X; g.d.ldb = n; g.d.stride_b = mn; g.d.b_kmajor = 1;
    g.d.D = A; g.d.ldd = m; g.d.stride_d = mm;
    g.d.epi = NC_EPI_STORE_BF16; g.d.alpha = 1.f; g.d.split_k = 1;
    g.symmetric = m > 128;  // the upper triangle of tiles, mirrored
    NC_TRY(gemm_launch(g, s, prof));
    // B = c A A + b A (symmetric too)
    g.d = nc_gemm_desc{};
    g.d.M = m; g.d.N = m; g.d.K = m; g.d.batch = count;
    g.d.A = A; g.d.lda = m; g.d.stride_a = mm; g.d.a_kmajor = 1;
    g.d.B = A; g.d.ldb = m; g.d.stride_b = mm; g.d.b_kmajor = 1;
    g.d.D = Bm; g.d.ldd = m; g.d.stride_d = mm;
    g.d.aux = A; g.d.ldaux = m; g.d.stride_aux = mm;
    g.d.epi = NC_EPI_AXPBY_BF16; g.d.alpha = kNsC; g.d.beta = kNsB; g.d.split_k = 1;
    NC_TRY(gemm_launch(g, s, prof));
    // Y = B X + a X
    g.symmetric = false;
    g.d = nc_gemm_desc{};
    g.d.M = m; g.d.N = n; g.d.K = m; g.d.batch = count;
    g.d.A = Bm; g.d.lda = m; g.d.stride_a = mm; g.d.a_kmajor = 1;
    g.d.B = X; g.d.ldb = n; g.d.stride_b = mn; g.d.b_kmajor = 0;
    g.d.D = Y; g.d.ldd = n; g.d.stride_d = mn;
    g.d.aux = X; g.d.ldaux = n; g.d.stride_aux = mn;
    g.d.epi = NC_EPI_AXPBY_BF16; g.d.alpha = 1.f; g.d.beta = kNsA; g.d.split_k = 1;
    NC_TRY(gemm_launch(g, s, prof));
    std::swap(X, Y);
  }
  if (X != x0)
    NC_CUDA_TRY(cudaMemcpyAsync(x0, X, sizeof(__nv_bfloat16) * count * mn,
                                cudaMemcpyDeviceToDevice, s));
  return NC_OK;
}

}  // namespace nc
