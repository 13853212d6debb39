// mma_throughput.cu -- throughput of tcgen05.mma by N and operand majorness.
//
// One CTA per SM (120 KB of dynamic shared memory keeps a second CTA off);
// one thread issues `iters` x 4 back-to-back tcgen05.mma.cta_group::1
// kind::f16 (M 128, K 16, bf16 in, fp32 accumulate in TMEM) from zeroed
// shared memory laid out with the 128-byte swizzle, commits, and waits (at
// most 2 s) for the commit; clock64 brackets the batch.  Prints one line per
// case: "N a_mn b_mn flop_per_clk_per_sm" (mean over the CTAs), or a
// negative rate if the wait expired.  Test infrastructure only: it uses the
// library's tcgen05 wrappers, not the library.
#include <cstdio>

#include "tc.cuh"

using namespace nc;

namespace {

constexpr int kSmem = 120 * 1024;

template <int N, int AMN, int BMN>
__global__ void __launch_bounds__(128, 1) mma_probe(unsigned long long* cycles, int iters) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t bar;
  __shared__ uint32_t slot;
  // A: 128 rows x 64 K (16 KB); B: N rows x 64 K (N * 128 bytes); zeroed.
  const int nbytes = 16384 + N * 128;
  for (int i = threadIdx.x; i < nbytes / 16; i += blockDim.x)
    tc::st_shared_v4(tc::smem_u32(smem) + 16 * i, 0, 0, 0, 0);
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tc::tmem_alloc(&slot, 512);
    tc::tmem_relinquish();
  }
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = slot;
  if (threadIdx.x == 0) {
    const uint32_t a = tc::smem_u32(smem), b = a + 16384;
    // K-major: rows of 128 bytes, K step +32 B.  MN-major: 64-wide MN
    // chunks 8 KB apart (64 K rows of 128 B), K step +2048 B.
    const uint64_t ad = AMN ? tc::smem_desc_sw128(a, 8192, 1024) : tc::smem_desc_sw128(a, 16, 1024);
    const uint64_t bd = BMN ? tc::smem_desc_sw128(b, 8192, 1024) : tc::smem_desc_sw128(b, 16, 1024);
    const uint32_t as = AMN ? 2048 : 32, bs = BMN ? 2048 : 32;
    const uint32_t id = tc::idesc_bf16_f32(128, N, AMN, BMN);
    const unsigned long long t0 = clock64();
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        tc::umma_bf16_ss(tmem, tc::desc_add(ad, kk * as), tc::desc_add(bd, kk * bs), id, 1u);
    tc::umma_commit(&bar);
    const uint64_t g0 = globaltimer();
    bool done = false;
    while (!(done = tc::mbar_try_wait(&bar, 0)))
      if (globaltimer() - g0 > kWaitTimeoutNs) break;
    cycles[blockIdx.x] = done ? clock64() - t0 : 0ull;
  }
  tc::tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int N, int AMN, int BMN>
int run(unsigned long long* d, int sms, int iters) {
  if (cudaFuncSetAttribute(mma_probe<N, AMN, BMN>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
      cudaSuccess)
    return 1;
  for (int rep = 0; rep < 2; ++rep) mma_probe<N, AMN, BMN><<<sms, 128, kSmem>>>(d, iters);
  if (cudaDeviceSynchronize() != cudaSuccess) return 1;
  unsigned long long h[1024];
  if (cudaMemcpy(h, d, sizeof(unsigned long long) * sms, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
  double mean = 0;
  bool timeout = false;
  for (int i = 0; i < sms; ++i) {
    timeout |= h[i] == 0;
    mean += (double)h[i];
  }
  mean /= sms;
  const double flop = (double)iters * 4 * 2 * 128 * N * 16;
  printf("%d %d %d %.1f\n", N, AMN, BMN, timeout ? -1.0 : flop / mean);
  return 0;
}

}  // namespace

int main() {
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0) != cudaSuccess || sms < 1 ||
      sms > 1024)
    return 1;
  unsigned long long* d = nullptr;
  if (cudaMalloc(&d, sizeof(unsigned long long) * sms) != cudaSuccess) return 1;
  const int iters = 4000;
  int rc = 0;
  rc |= run<256, 0, 0>(d, sms, iters);
  rc |= run<128, 0, 0>(d, sms, iters);
  rc |= run<64, 0, 0>(d, sms, iters);
  rc |= run<256, 0, 1>(d, sms, iters);
  rc |= run<128, 0, 1>(d, sms, iters);
  rc |= run<64, 0, 1>(d, sms, iters);
  rc |= run<128, 1, 1>(d, sms, iters);
  rc |= run<64, 1, 1>(d, sms, iters);
  rc |= run<128, 1, 0>(d, sms, iters);
  cudaFree(d);
  return rc;
}
