// wait_timeout.cu -- the bounded mbarrier wait of the library's kernels,
// made to run out.
//
// One CTA waits on an mbarrier that nothing ever arrives on, with the
// library's tc::mbar_wait (a wall-clock limit of kWaitTimeoutNs).  When the
// limit passes the wait sets the abort flag and writes kDevTimeout to the
// device status word, and the kernel returns normally.  The host then reads
// the status, the wait's result and the elapsed time, and launches a second
// kernel to show the context is still usable.  Prints one line:
// "status waited_ok elapsed_ms after".  Test infrastructure only.
#include <cstdio>

#include "tc.cuh"

using namespace nc;

namespace {

__global__ void wait_on_nothing(int* status, int* result) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);  // expects one arrival; none comes
    tc::fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  const bool ok = tc::mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), status);
  if (threadIdx.x == 0) result[0] = ok ? 1 : 0;
}

__global__ void add_one(int* x) {
  if (threadIdx.x == 0 && blockIdx.x == 0) x[0] += 1;
}

}  // namespace

int main() {
  int* d = nullptr;
  if (cudaMalloc(&d, 3 * sizeof(int)) != cudaSuccess) return 1;
  if (cudaMemset(d, 0, 3 * sizeof(int)) != cudaSuccess) return 1;
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  cudaEventRecord(e0);
  wait_on_nothing<<<1, 32>>>(d, d + 1);
  cudaEventRecord(e1);
  if (cudaDeviceSynchronize() != cudaSuccess) return 2;
  float ms = 0.f;
  cudaEventElapsedTime(&ms, e0, e1);
  add_one<<<1, 32>>>(d + 2);
  if (cudaDeviceSynchronize() != cudaSuccess) return 3;
  int h[3] = {-1, -1, -1};
  if (cudaMemcpy(h, d, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return 4;
  printf("%d %d %.1f %d\n", h[0], h[1], ms, h[2]);
  cudaFree(d);
  return 0;
}
