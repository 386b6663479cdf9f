// Graph replay of a whole stage.  The preparation and the quantizer each enqueue a
// chain of small dependent launches on several streams; every link of such a chain
// that crosses streams costs an event wait on the device.  Captured once as a CUDA
// graph and replayed, the same launches run with their dependencies as graph edges.
//
// A graph holds the launches' arguments by value, so it is only valid for calls with
// the same arguments (pointers, sizes, settings) on the same device: the key.  The
// data behind the pointers is read when the graph runs, as by a direct call.  A key is
// captured the second time it comes (a one-off call never pays for a capture) and at
// most kMaxGraphs graphs are kept per process; a graph is never destroyed while the
// library is loaded (one could still be running), so the cache does not evict.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace {

struct Entry {
  GraphKey key;
  int dev;
  cudaGraphExec_t exec;
  int64_t launches;   // the kernels the graph holds (counted again at each replay)
};

constexpr size_t kMaxGraphs = 32;
constexpr size_t kMaxSeen = 64;

thread_local int g_replay = 1;   // per host thread: the calls a thread makes
std::mutex g_mu;
std::vector<Entry> g_graphs;
std::vector<std::pair<GraphKey, int>> g_seen;   // keys seen once, oldest first

// A stream and two events per host thread and device: graphs are captured and
// launched there (never on the legacy default stream, which cannot be captured).
struct GraphStream {
  cudaStream_t s = nullptr;
  cudaEvent_t in = nullptr, out = nullptr;
};

int graph_stream(int dev, GraphStream** out) {
  thread_local GraphStream per_dev[64];
  if (dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
  GraphStream& g = per_dev[dev];
  if (g.s == nullptr) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&g.s, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaEventCreateWithFlags(&g.in, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&g.out, cudaEventDisableTiming) != cudaSuccess)
      return GPTQ_ERR_CUDA;
  }
  *out = &g;
  return GPTQ_OK;
}

}  // namespace

int run_graph_cached(const GraphKey& key, cudaStream_t s, const std::function<int(cudaStream_t)>& enqueue) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (!key.ok || g_replay == 0 || trace_enabled() ||
      cudaStreamIsCapturing(s, &cap) != cudaSuccess ||
      cap != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return enqueue(s);
  }
  int dev = -1;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  cudaGraphExec_t exec = nullptr;
  int64_t nl = 0;
  bool capture = false;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (const Entry& e : g_graphs)
      if (e.dev == dev && e.key == key) {
        exec = e.exec;
        nl = e.launches;
      }
    if (exec == nullptr && g_graphs.size() < kMaxGraphs) {
      auto it = std::find_if(g_seen.begin(), g_seen.end(),
                             [&](const std::pair<GraphKey, int>& p) { return p.second == dev && p.first == key; });
      if (it != g_seen.end()) {
        g_seen.erase(it);
        capture = true;
      } else {
        if (g_seen.size() >= kMaxSeen) g_seen.erase(g_seen.begin());
        g_seen.emplace_back(key, dev);
      }
    }
  }
  if (exec == nullptr && !capture) return enqueue(s);
  GraphStream* gs = nullptr;
  int rc = graph_stream(dev, &gs);
  if (rc != GPTQ_OK) return rc;
  if (exec == nullptr) {
    const uint64_t before = gptq_kernel_launches();
    if (cudaStreamBeginCapture(gs->s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
      cudaGetLastError();
      return enqueue(s);
    }
    rc = enqueue(gs->s);
    cudaGraph_t graph = nullptr;
    const cudaError_t ec = cudaStreamEndCapture(gs->s, &graph);
    nl = (int64_t)(gptq_kernel_launches() - before);
    count_launches(-nl);                                   // captured, not run
    cudaError_t ei = cudaErrorUnknown;
    if (rc == GPTQ_OK && ec == cudaSuccess && graph != nullptr) ei = cudaGraphInstantiate(&exec, graph, 0);
    if (graph != nullptr) cudaGraphDestroy(graph);
    if (rc != GPTQ_OK || ec != cudaSuccess || ei != cudaSuccess) {
      cudaGetLastError();
      return enqueue(s);                                   // the stage runs launch by launch
    }
    std::lock_guard<std::mutex> lock(g_mu);
    g_graphs.push_back(Entry{key, dev, exec, nl});
  }
  // the graph runs after the work already on s, and s continues after it
  GPTQ_CUDA_TRY(cudaEventRecord(gs->in, s));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(gs->s, gs->in, 0));
  GPTQ_CUDA_TRY(cudaGraphLaunch(exec, gs->s));
  GPTQ_CUDA_TRY(cudaEventRecord(gs->out, gs->s));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, gs->out, 0));
  count_launches(nl);
  return GPTQ_OK;
}

}  // namespace gptq

extern "C" int gptq_set_graph_replay(int on) {
  const int prev = gptq::g_replay;
  if (on >= 0) gptq::g_replay = on ? 1 : 0;
  return prev;
}
