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

enum DataFault : int32_t { kFaultBadType = 1, kFaultNonFinite = 2 };

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

inline janus_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? JANUS_OK : JANUS_ERR_CUDA;
}

__device__ __forceinline__ void record_fault(WsHeader* ws, int32_t code) {
  atomicCAS(&ws->error, 0, code);
}

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
