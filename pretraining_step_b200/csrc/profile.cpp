// profile.cpp -- per-kernel-class device timing with CUDA events.
//
// Each launch site constructs a Probe around its launch.  While profiling is
// enabled the probe records an event pair on the launch stream; reading the
// profile synchronises, sums the elapsed times per class together with the
// algorithmic FLOPs / bytes the launch sites declared, and resets.  Launches
// are counted whether or not timing is enabled.

#include <cuda_runtime.h>

#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "internal.h"

namespace nc {

struct Profiler {
  bool on = false;
  int64_t launches = 0;
  struct Pending {
    cudaEvent_t a, b;
    std::string name;
    double flops, bytes;
  };
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;
  struct Acc {
    int launches = 0;
    double ms = 0, flops = 0, bytes = 0;
  };
  std::map<std::string, Acc> acc;

  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};

Profiler* profiler_create() { return new Profiler(); }

void profiler_destroy(Profiler* p) {
  if (!p) return;
  for (auto& q : p->pending) {
    cudaEventDestroy(q.a);
    cudaEventDestroy(q.b);
  }
  for (auto e : p->pool) cudaEventDestroy(e);
  delete p;
}

void profiler_enable(Profiler* p, bool on) {
  if (p) p->on = on;
}

int64_t profiler_launches(const Profiler* p) { return p ? p->launches : 0; }

bool profiler_enabled(const Profiler* p) { return p && p->on; }

void profiler_add_launches(Profiler* p, int64_t n) {
  if (p) p->launches += n;
}

Probe::Probe(Profiler* prof_, cudaStream_t s, const char* name, double flops, double bytes)
    : prof(prof_), stream(s), slot(-1) {
  if (!prof) return;
  prof->launches++;
  if (!prof->on) return;
  Profiler::Pending q;
  q.a = prof->get();
  q.b = prof->get();
  q.name = name;
  q.flops = flops;
  q.bytes = bytes;
  cudaEventRecord(q.a, s);
  prof->pending.push_back(q);
  slot = (int)prof->pending.size() - 1;
}

Probe::~Probe() {
  if (prof && slot >= 0) cudaEventRecord(prof->pending[slot].b, stream);
}

nc_status profiler_read(Profiler* p, nc_kernel_stat* out, int max, int* n) {
  if (!p) return fail(NC_ERR_INVALID_ARG, "profile: no profiler");
  for (auto& q : p->pending) {
    cudaError_t e = cudaEventSynchronize(q.b);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float ms = 0;
    cudaEventElapsedTime(&ms, q.a, q.b);
    Profiler::Acc& a = p->acc[q.name];
    a.launches++;
    a.ms += ms;
    a.flops += q.flops;
    a.bytes += q.bytes;
    p->pool.push_back(q.a);
    p->pool.push_back(q.b);
  }
  p->pending.clear();
  int k = 0;
  for (auto& kv : p->acc) {
    if (k >= max) break;
    nc_kernel_stat& s = out[k++];
    std::memset(&s, 0, sizeof(s));
    std::strncpy(s.name, kv.first.c_str(), sizeof(s.name) - 1);
    s.launches = kv.second.launches;
    s.total_ms = kv.second.ms;
    s.flops = kv.second.flops;
    s.bytes = kv.second.bytes;
  }
  if (n) *n = k;
  p->acc.clear();
  return NC_OK;
}

}  // namespace nc
