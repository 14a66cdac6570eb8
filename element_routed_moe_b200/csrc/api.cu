// Library-wide entry points: status strings, version, janus_check, the debug
// build's fault word (janus_debug_build, janus_debug_check), the launch trace
// (janus_trace_*), and the host-side launch-failure injection used by the
// tests.
#include <atomic>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "common.cuh"

namespace janus {

static std::atomic<int32_t> g_inject{0};

bool consume_injected_failure() {
  int32_t v = g_inject.load();
  while (v > 0) {
    if (g_inject.compare_exchange_weak(v, v - 1)) return true;
  }
  return false;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

#ifdef JANUS_DEBUG
// The debug build's fault word for calls without a workspace (one per GPU that
// loads the library).  Host code takes its address with cudaGetSymbolAddress.
static __device__ __align__(256) int32_t g_debug_fault[64];

static std::mutex g_debug_mu;
static std::unordered_map<int, int32_t*> g_debug_addr;   // device ordinal -> address

int32_t* debug_fault_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_debug_mu);
  auto it = g_debug_addr.find(dev);
  if (it != g_debug_addr.end()) return it->second;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_debug_fault) != cudaSuccess) return nullptr;
  g_debug_addr[dev] = (int32_t*)p;
  return (int32_t*)p;
}
#else
int32_t* debug_fault_word() { return nullptr; }
#endif

// ---- launch trace -------------------------------------------------------
// Records of (kernel name, start event, end event), events created when the
// trace starts (never inside a traced region); a launch past the capacity is
// not recorded.
namespace {
struct TraceRec {
  const char* name;
  cudaEvent_t beg, end;
};
std::mutex g_trace_mu;
std::vector<TraceRec> g_trace;
int g_trace_used = 0;
std::atomic<bool> g_trace_on{false};

void trace_release() {
  for (TraceRec& r : g_trace) {
    cudaEventDestroy(r.beg);
    cudaEventDestroy(r.end);
  }
  g_trace.clear();
  g_trace_used = 0;
}
}  // namespace

bool trace_on() { return g_trace_on.load(std::memory_order_relaxed); }

int trace_begin(const char* name, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  if (!g_trace_on.load() || g_trace_used >= (int)g_trace.size()) return -1;
  const int slot = g_trace_used++;
  g_trace[slot].name = name;
  cudaEventRecord(g_trace[slot].beg, stream);
  return slot;
}

void trace_end(int slot, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  if (slot >= 0 && slot < (int)g_trace.size()) cudaEventRecord(g_trace[slot].end, stream);
}

}  // namespace janus

extern "C" {

janus_status janus_trace_start(int32_t capacity) {
  JANUS_CHECK_ARG(capacity >= 1 && capacity <= (1 << 20));
  std::lock_guard<std::mutex> lock(janus::g_trace_mu);
  janus::g_trace_on.store(false);
  janus::trace_release();
  janus::g_trace.reserve((size_t)capacity);
  for (int i = 0; i < capacity; ++i) {
    janus::TraceRec r{nullptr, nullptr, nullptr};
    if (cudaEventCreate(&r.beg) != cudaSuccess) return JANUS_ERR_CUDA;
    if (cudaEventCreate(&r.end) != cudaSuccess) {
      cudaEventDestroy(r.beg);
      return JANUS_ERR_CUDA;
    }
    janus::g_trace.push_back(r);
  }
  janus::g_trace_on.store(true);
  return JANUS_OK;
}

janus_status janus_trace_stop(void) {
  janus::g_trace_on.store(false);
  return JANUS_OK;
}

janus_status janus_trace_count(int32_t* n) {
  JANUS_CHECK_ARG(n);
  std::lock_guard<std::mutex> lock(janus::g_trace_mu);
  *n = janus::g_trace_used;
  return JANUS_OK;
}

janus_status janus_trace_get(int32_t i, const char** name, float* ms) {
  JANUS_CHECK_ARG(name && ms);
  std::lock_guard<std::mutex> lock(janus::g_trace_mu);
  JANUS_CHECK_ARG(i >= 0 && i < janus::g_trace_used);
  const janus::TraceRec& r = janus::g_trace[i];
  if (cudaEventSynchronize(r.end) != cudaSuccess) return JANUS_ERR_CUDA;
  if (cudaEventElapsedTime(ms, r.beg, r.end) != cudaSuccess) return JANUS_ERR_CUDA;
  *name = r.name;
  return JANUS_OK;
}

janus_status janus_trace_release(void) {
  std::lock_guard<std::mutex> lock(janus::g_trace_mu);
  janus::g_trace_on.store(false);
  janus::trace_release();
  return JANUS_OK;
}

const char* janus_status_string(janus_status s) {
  switch (s) {
    case JANUS_OK: return "JANUS_OK";
    case JANUS_ERR_INVALID_ARG: return "JANUS_ERR_INVALID_ARG: null pointer, size/limit violation or workspace too small";
    case JANUS_ERR_MISALIGNED: return "JANUS_ERR_MISALIGNED: feature pointer not 16/8-byte aligned or d % 4 != 0";
    case JANUS_ERR_CUDA: return "JANUS_ERR_CUDA: a CUDA launch or runtime call failed";
    case JANUS_ERR_DATA:
      return "JANUS_ERR_DATA: a kernel recorded a data fault (bad type id, non-finite feature, a bounded "
             "tensor-core wait that ran out, or rows that break JANUS_FFN_X_DEQUANTIZED)";
  }
  return "JANUS_ERR_UNKNOWN";
}

int32_t janus_version(void) { return 10000; }

janus_status janus_check(const void* workspace, janus_stream_t stream) {
  if (!workspace) return JANUS_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return JANUS_ERR_CUDA;
  int32_t err = 0;
  if (cudaMemcpy(&err, workspace, sizeof(err), cudaMemcpyDeviceToHost) != cudaSuccess)
    return JANUS_ERR_CUDA;
  return err == 0 ? JANUS_OK : JANUS_ERR_DATA;
}

int32_t janus_debug_build(void) { return janus::kDebug ? 1 : 0; }

janus_status janus_debug_check(janus_stream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return JANUS_ERR_CUDA;
  int32_t* w = janus::debug_fault_word();
  if (!w) return JANUS_OK;   // release build: nothing is recorded here
  int32_t err = 0;
  if (cudaMemcpy(&err, w, sizeof(err), cudaMemcpyDeviceToHost) != cudaSuccess) return JANUS_ERR_CUDA;
  if (err != 0 && cudaMemset(w, 0, sizeof(int32_t)) != cudaSuccess) return JANUS_ERR_CUDA;
  return err == 0 ? JANUS_OK : JANUS_ERR_DATA;
}

void janus_debug_inject_launch_failures(int32_t n_calls) {
  janus::g_inject.store(n_calls > 0 ? n_calls : 0);
}

}  // extern "C"
