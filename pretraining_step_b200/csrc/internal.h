// internal.h -- host-side interfaces between the translation units of the
// step library (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string>

#include "../../include/nc.h"

namespace nc {

// Thread-local error message behind nc_last_error().
void set_error(const std::string& msg);
nc_status fail(nc_status s, const std::string& msg);
nc_status cuda_fail(cudaError_t e, const char* what);

#define NC_CUDA_TRY(expr)                                     \
  do {                                                        \
    cudaError_t _e = (expr);                                  \
    if (_e != cudaSuccess) return ::nc::cuda_fail(_e, #expr); \
  } while (0)

#define NC_TRY(expr)                   \
  do {                                 \
    nc_status _s = (expr);             \
    if (_s != NC_OK) return _s;        \
  } while (0)

int num_sms();

// Setup that holds per device, such as a kernel's shared-memory limit
// (cudaFuncSetAttribute): once_per_device(o, f) runs f the first time each
// device (0..63; beyond that, every time) reaches it, and again after a
// failure.  Thread-safe.
struct DeviceOnce {
  std::mutex m;
  uint64_t done = 0;
};
template <class F>
nc_status once_per_device(DeviceOnce& o, F&& f) {
  int dev = 0;
  NC_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return f();
  const uint64_t bit = 1ull << dev;
  std::lock_guard<std::mutex> lock(o.m);
  if (o.done & bit) return NC_OK;
  const nc_status st = f();
  if (st == NC_OK) o.done |= bit;
  return st;
}

// Device address of the library's op status word on the current device (a
// file-scope __device__ int, looked up once per device): the single-kernel
// entry points (nc_op_*) hand it to their kernels as the status word, and
// nc_op_sync reads and clears it.
nc_status op_status_word(int** out);

// Per-kernel-class timing (profile.cpp).  Every launch site wraps its launch
// in a Probe; with profiling off it only counts the launch.
struct Profiler;
struct Probe {
  Probe(Profiler* prof, cudaStream_t s, const char* name, double flops, double bytes);
  ~Probe();
  Profiler* prof;
  cudaStream_t stream;
  int slot;
};
Profiler* profiler_create();
void profiler_destroy(Profiler*);
void profiler_enable(Profiler*, bool on);
nc_status profiler_read(Profiler*, nc_kernel_stat* out, int max, int* n);
int64_t profiler_launches(const Profiler*);
bool profiler_enabled(const Profiler*);
// Adds n to the launch count (graph replays; a capture takes back the
// launches it recorded but did not run).
void profiler_add_launches(Profiler*, int64_t n);

}  // namespace nc
