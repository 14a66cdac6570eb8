// Internal helpers shared by the libjanus CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "janus.h"

namespace janus {

// Every workspace starts with this header; janus_check reads `error`.
struct WsHeader {
  int32_t error;      // 0 = ok, else a data-fault code written by a kernel
  uint32_t done;      // "last block" counter for single-pass reductions
  int32_t pad[62];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

// Data-fault codes written to a workspace's error word (first fault wins).
enum DataFault : int32_t {
  kFaultBadType = 1,     // element type id outside [0, T)
  kFaultNonFinite = 2,   // non-finite feature to pack, or non-finite gate logit
  kFaultTimeout = 3,     // a bounded tensor-core pipeline wait ran out
  kFaultNotTf32 = 4,     // JANUS_FFN_X_DEQUANTIZED rows with bits below TF32 precision
  kFaultIndex = 5,       // debug builds: a caller-supplied index outside its range
  kFaultCapacity = 6,    // expert-parallel receive buffer too small for the routed rows
};

// Debug builds (compiled with -DJANUS_DEBUG) check every caller-supplied index
// (slot_of, perm, offsets, row_ptr, senders, exchange tables) on the device
// before using it, record kFaultIndex and skip the access instead.
#ifdef JANUS_DEBUG
constexpr bool kDebug = true;
#else
constexpr bool kDebug = false;
#endif

// Debug builds: device address, on the current device, of the library's fault
// word for calls that take no workspace; release builds: nullptr.
int32_t* debug_fault_word();

constexpr int kMaxExperts = 256;
constexpr int kMaxTypes = 4096;
constexpr int kMaxDim = 1 << 20;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// Host-side failure injection (tests only).
bool consume_injected_failure();

// Number of SMs of the current device.
int num_sms();

// Launch trace (janus_trace_*): while it records, a traced launch is
// bracketed by two CUDA events on its stream.  trace_begin returns the record's
// slot, or -1 when the trace is off or full.
bool trace_on();
int trace_begin(const char* name, cudaStream_t stream);
void trace_end(int slot, cudaStream_t stream);
struct TraceScope {
  int slot;
  cudaStream_t stream;
  TraceScope(const char* name, cudaStream_t s) : slot(trace_on() ? trace_begin(name, s) : -1), stream(s) {}
  ~TraceScope() {
    if (slot >= 0) trace_end(slot, stream);
  }
};

inline janus_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? JANUS_OK : JANUS_ERR_CUDA;
}

__device__ __forceinline__ void record_fault(WsHeader* ws, int32_t code) {
  atomicCAS(&ws->error, 0, code);
}

// Debug builds: record an index fault in `word` (the library's debug fault
// word or a workspace's error word); a no-op in release builds.
__device__ __forceinline__ void debug_fault(int32_t* word) {
  if (kDebug && word) atomicCAS(word, 0, (int32_t)kFaultIndex);
}

// 0 <= v < n
__device__ __forceinline__ bool in_range(int64_t v, int64_t n) { return (uint64_t)v < (uint64_t)n; }

}  // namespace janus

#define JANUS_CHECK_ARG(cond)                         \
  do {                                                \
    if (!(cond)) return JANUS_ERR_INVALID_ARG;        \
  } while (0)

#define JANUS_CHECK_ALIGN(cond)                       \
  do {                                                \
    if (!(cond)) return JANUS_ERR_MISALIGNED;         \
  } while (0)

#define JANUS_CUDA_TRY(expr)                          \
  do {                                                \
    if ((expr) != cudaSuccess) return JANUS_ERR_CUDA; \
  } while (0)
