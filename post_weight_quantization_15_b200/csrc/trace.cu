// Kernel timing trace: CUDA events recorded around the library's own launches, on
// the stream each kernel is launched on (the caller's stream or one of the
// library's), aggregated per kernel with the launch's algorithmic work.  Off by
// default; when off, a trace scope costs one relaxed atomic load.  Benchmarks use
// it to time each kernel inside a whole step, where several library streams run
// at once and events on the caller's stream alone cannot separate the kernels.
// Also the FP32 peak probe: the denominator of the CUDA-core kernels' roofline.
#include <cuda_runtime.h>

#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace {

struct Rec {
  const char* kernel;
  const char* unit;
  double work;
  cudaEvent_t a, b;
  int dev;            // the device the events were created on
  cudaStream_t s;     // the stream the launch went to
};

std::atomic<int> g_on{0};
std::mutex g_mu;
std::vector<Rec> g_recs;
// Events already created, by device, reused by later scopes (creating one per
// launch would cost more host time than recording it).
std::map<int, std::vector<cudaEvent_t>> g_pool;

cudaEvent_t take_event() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    std::vector<cudaEvent_t>& v = g_pool[dev];
    if (!v.empty()) {
      cudaEvent_t e = v.back();
      v.pop_back();
      return e;
    }
  }
  cudaEvent_t e = nullptr;
  return cudaEventCreate(&e) == cudaSuccess ? e : nullptr;
}

// FP32 peak probe: every thread runs 8 independent FMA chains.
__global__ void __launch_bounds__(256) ffma_probe_kernel(float* out, int iters, float b, float c) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = (float)(threadIdx.x + i);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = fmaf(a[i], b, c);
    }
  }
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) t += a[i];
  if (t == 1234.5f) out[blockIdx.x * blockDim.x + threadIdx.x] = t;   // keeps the chains live
}

struct Agg {
  const char* unit = "";
  uint64_t launches = 0;
  double ms = 0.0, work = 0.0;
};

}  // namespace

bool trace_enabled() { return g_on.load(std::memory_order_relaxed) != 0; }

TraceScope::TraceScope(const char* kernel, const char* unit, double work, cudaStream_t s)
    : kernel_(kernel), unit_(unit), work_(work), s_(s), a_(nullptr) {
  if (g_on.load(std::memory_order_relaxed) == 0) return;
  cudaEvent_t a = take_event();
  if (a == nullptr) return;
  if (cudaEventRecord(a, s_) != cudaSuccess) {
    cudaEventDestroy(a);
    return;
  }
  a_ = a;
}

TraceScope::~TraceScope() {
  if (a_ == nullptr) return;
  cudaEvent_t b = take_event();
  if (b == nullptr || cudaEventRecord(b, s_) != cudaSuccess) {
    if (b) cudaEventDestroy(b);
    cudaEventDestroy(static_cast<cudaEvent_t>(a_));
    return;
  }
  int dev = -1;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_mu);
  g_recs.push_back(Rec{kernel_, unit_, work_, static_cast<cudaEvent_t>(a_), b, dev, s_});
}

}  // namespace gptq

using namespace gptq;

extern "C" {

int gptq_trace_enable(int on) {
  g_on.store(on ? 1 : 0, std::memory_order_relaxed);
  return GPTQ_OK;
}

int gptq_trace_read(gptq_trace_row* rows, int max_rows, int* n_rows) {
  if (n_rows == nullptr || max_rows < 0 || (max_rows > 0 && rows == nullptr)) return GPTQ_ERR_INVALID_ARG;
  std::vector<Rec> recs;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    recs.swap(g_recs);
  }
  std::map<std::string, Agg> agg;
  std::vector<std::string> order;
  int rc = GPTQ_OK;
  for (const Rec& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      rc = GPTQ_ERR_CUDA;
    {   // the events go back to the pool of the device they belong to
      std::lock_guard<std::mutex> lock(g_mu);
      g_pool[r.dev].push_back(r.a);
      g_pool[r.dev].push_back(r.b);
    }
    auto it = agg.find(r.kernel);
    if (it == agg.end()) {
      order.push_back(r.kernel);
      it = agg.emplace(r.kernel, Agg{}).first;
      it->second.unit = r.unit;
    }
    it->second.launches += 1;
    it->second.ms += ms;
    it->second.work += r.work;
  }
  // kernel names are string literals of the library: their pointers stay valid
  std::map<std::string, const char*> names;
  for (const Rec& r : recs) names.emplace(r.kernel, r.kernel);
  int k = 0;
  for (const std::string& name : order) {
    if (k >= max_rows) break;
    const Agg& a = agg[name];
    rows[k] = gptq_trace_row{names[name], a.unit, a.launches, a.ms, a.work};
    ++k;
  }
  *n_rows = k;
  return rc;
}

int gptq_trace_read_timeline(gptq_trace_event* events, int max_events, int* n_events) {
  if (n_events == nullptr || max_events < 0 || (max_events > 0 && events == nullptr)) return GPTQ_ERR_INVALID_ARG;
  std::vector<Rec> recs;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    recs.swap(g_recs);
  }
  int rc = GPTQ_OK;
  for (const Rec& r : recs)
    if (cudaEventSynchronize(r.b) != cudaSuccess) rc = GPTQ_ERR_CUDA;
  // the origin: the earliest start among the records of the first record's device
  size_t origin = 0;
  for (size_t i = 1; i < recs.size(); ++i) {
    if (recs[i].dev != recs[0].dev) continue;
    float d = 0.f;
    if (cudaEventElapsedTime(&d, recs[origin].a, recs[i].a) == cudaSuccess && d < 0.f) origin = i;
  }
  int k = 0;
  for (const Rec& r : recs) {
    float t0 = 0.f, t1 = 0.f;
    if (r.dev == recs[origin].dev && k < max_events &&
        cudaEventElapsedTime(&t0, recs[origin].a, r.a) == cudaSuccess &&
        cudaEventElapsedTime(&t1, recs[origin].a, r.b) == cudaSuccess) {
      events[k++] = gptq_trace_event{r.kernel, reinterpret_cast<uint64_t>(r.s), t0, t1};
    }
  }
  for (const Rec& r : recs) {   // the events go back to their device's pool
    std::lock_guard<std::mutex> lock(g_mu);
    g_pool[r.dev].push_back(r.a);
    g_pool[r.dev].push_back(r.b);
  }
  *n_events = k;
  return rc;
}

}  // extern "C"

extern "C" int gptq_probe_fp32_peak(float* out, int blocks, int iters, void* stream) {
  if (out == nullptr || blocks <= 0 || iters <= 0) return GPTQ_ERR_INVALID_ARG;
  ffma_probe_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(out, iters, 0.999f, 1e-3f);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}
