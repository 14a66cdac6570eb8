// Library-wide entry points: status strings, version, janus_check, and the
// host-side launch-failure injection used by the tests.
#include <atomic>

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

}  // namespace janus

extern "C" {

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

void janus_debug_inject_launch_failures(int32_t n_calls) {
  janus::g_inject.store(n_calls > 0 ? n_calls : 0);
}

}  // extern "C"
