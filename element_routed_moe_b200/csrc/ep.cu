// Expert-parallel exchange of the MoE layer: the dispatch rows travel to the
// rank that owns their expert, the expert outputs travel back.
//
// Sources: paper review "Breaking the Training Barrier of Billion-Parameter
// Universal Machine Learning Interatomic Potentials" section 3.4 (FSEP: the
// experts are sharded over ranks) and section 3.5 (the MoE all-to-all moves
// atom-type-aware FP16-packed rows, half the FP32 volume).
//
// B200 design: one process per GPU; every rank maps the other ranks' receive
// buffers (CUDA IPC over NVLink / NVSwitch), so the packing kernel stores each
// packed row straight into its owner's buffer (peer stores, no staging copy,
// no library collective on the data path, no multicast).  The exchange is
// stream-ordered: a kernel's peer stores are complete when it finishes, and
// the caller orders the phases with a collective barrier.  No kernel here
// waits on another rank.
//
// Layout (rank o owns experts [o*E/P, (o+1)*E/P)):
//   src_off[s][e]  = sum_{e' < e} counts_all[s][e']       (the sender's local order)
//   recv_off[o][j] = rows of o's local experts j' < j, summed over senders
//   dst_off[s][e]  = recv_off[owner(e)][local(e)] + sum_{s' < s} counts_all[s'][e]
// Row i of (s, e) goes from sender row src_off[s][e] + i to owner row
// dst_off[s][e] + i; the owner's rows are grouped by local expert, then sender,
// so its expert MLP runs on recv_off[o] unchanged.
//
// Capacity: every receive buffer holds `cap` rows (a capacity factor times a
// rank's fair share, chosen by the caller).  recv_off is clamped to cap, so the
// owner's kernels never touch a row past it; a send whose owner row would be
// at or past cap is skipped and recorded as kFaultCapacity in the send's
// workspace error word (the layer's result is then incomplete, never an
// out-of-bounds store).
#include <cuda.h>
#include <cuda_fp16.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "rows.cuh"

namespace janus {
namespace {

constexpr int kMaxRanks = JANUS_EP_MAX_RANKS;

struct PeerRows {          // one device pointer per rank (local or peer-mapped)
  void* ptr[kMaxRanks];
  float* scale[kMaxRanks];
};

// One CTA: the whole layout is at most kMaxRanks x kMaxExperts entries.
// recv_off is clamped to cap; dst_off keeps the unclamped positions (a send
// compares them with cap).
__global__ void ep_layout_kernel(const int32_t* __restrict__ counts_all, int P, int E, int64_t cap,
                                 int32_t* __restrict__ src_off, int32_t* __restrict__ dst_off,
                                 int32_t* __restrict__ recv_off) {
  const int El = E / P;
  for (int s = threadIdx.x; s < P; s += blockDim.x) {
    int32_t acc = 0;
    for (int e = 0; e < E; ++e) {
      src_off[s * (E + 1) + e] = acc;
      acc += counts_all[s * E + e];
    }
    src_off[s * (E + 1) + E] = acc;
  }
  for (int o = threadIdx.x; o < P; o += blockDim.x) {
    int64_t acc = 0;
    for (int j = 0; j < El; ++j) {
      recv_off[o * (El + 1) + j] = (int32_t)min(acc, cap);
      for (int s = 0; s < P; ++s) acc += counts_all[s * E + o * El + j];
    }
    recv_off[o * (El + 1) + El] = (int32_t)min(acc, cap);
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int o = e / El, j = e - o * El;
    int32_t acc = 0;        // rows of the owner's local experts before j
    for (int jj = 0; jj < j; ++jj)
      for (int s = 0; s < P; ++s) acc += counts_all[s * E + o * El + jj];
    for (int s = 0; s < P; ++s) {
      dst_off[s * E + e] = acc;
      acc += counts_all[s * E + e];
    }
  }
}

// Destination of flat slot s (atom i's k-th expert): (owner, owner row), or
// row -1 when the owner's receive buffer has no room for it (recorded as
// kFaultCapacity) or, in debug builds, when slot_of / topk_expert hold an
// index outside its range (recorded as kFaultIndex).  p = slot_of[s] is the
// slot's row in this rank's local dispatch order, e = topk_expert[s].
__device__ __forceinline__ void ep_dest(int64_t s, int64_t R, int E, int El, const int32_t* __restrict__ slot_of,
                                        const int32_t* __restrict__ topk_expert,
                                        const int32_t* __restrict__ src_off_r, const int32_t* __restrict__ dst_off_r,
                                        int64_t cap, WsHeader* ws, int* owner, int64_t* row) {
  const int32_t p = slot_of[s], e = topk_expert[s];
  *owner = 0;
  *row = -1;
  if (kDebug && !(in_range(p, R) && in_range(e, E) && p >= src_off_r[e] && p < src_off_r[e + 1])) {
    if (ws) debug_fault(&ws->error);
    return;
  }
  const int64_t r = (int64_t)dst_off_r[e] + (p - src_off_r[e]);
  if (r < 0 || r >= cap) {
    if (ws) record_fault(ws, kFaultCapacity);
    return;
  }
  *owner = e / El;
  *row = r;
}

// Pack-and-send: quant_pack_kernel's scatter form with the K destinations in
// the owners' receive buffers; the row's scale goes along (one float per row).
__global__ void __launch_bounds__(kThreads)
ep_pack_send_kernel(const float4* __restrict__ x, int64_t n_atoms, int d4, int K,
                    const int32_t* __restrict__ types, int T, const int32_t* __restrict__ slot_of,
                    const int32_t* __restrict__ topk_expert, const uint32_t* __restrict__ amax_bits,
                    const int32_t* __restrict__ src_off_r, const int32_t* __restrict__ dst_off_r, int E, int El,
                    int64_t cap, PeerRows peers, float* __restrict__ scale, WsHeader* ws) {
  const int64_t R = n_atoms * K;
  extern __shared__ float s_tab[];            // [T] inverse scales, [T] scales
  float* s_inv = s_tab;
  float* s_scale = s_tab + T;
  for (int t = threadIdx.x; t < T; t += kThreads) {
    const uint32_t a = amax_bits[t];
    const int e = scale_exponent_from_bits(a);
    s_inv[t] = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23) : 0.0f;
    s_scale[t] = __uint_as_float((uint32_t)(127 + e) << 23);
    if (blockIdx.x == 0) {
      scale[t] = s_scale[t];
      if (a >= 0x7f800000u) record_fault(ws, kFaultNonFinite);
    }
  }
  __syncthreads();
  const int lane = threadIdx.x % 32;
  for (int64_t i = global_warp(); i < n_atoms; i += total_warps()) {
    int t = types[i];
    if (t < 0 || t >= T) t = 0;                // recorded by the amax pass
    const float inv = s_inv[t];
    int my_owner = 0;
    int64_t my_row = -1;
    if (lane < K)
      ep_dest(i * K + lane, R, E, El, slot_of, topk_expert, src_off_r, dst_off_r, cap, ws, &my_owner, &my_row);
    if (lane < K && my_row >= 0) peers.scale[my_owner][my_row] = s_scale[t];
    const float4* src = x + i * d4;
    for (int c0 = 0; c0 < d4; c0 += 32 * kU) {
      uint2 q[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) {
          const float4 v = __ldcs(src + c);
          const __half2 lo = __floats2half2_rn(v.x * inv, v.y * inv);
          const __half2 hi = __floats2half2_rn(v.z * inv, v.w * inv);
          q[u].x = *reinterpret_cast<const uint32_t*>(&lo);
          q[u].y = *reinterpret_cast<const uint32_t*>(&hi);
        }
      }
      for (int k = 0; k < K; ++k) {
        const int o = __shfl_sync(0xffffffffu, my_owner, k);
        const int64_t row = __shfl_sync(0xffffffffu, (long long)my_row, k);
        if (row < 0) continue;                 // no room at the owner (same in every lane)
        uint2* dst = reinterpret_cast<uint2*>(peers.ptr[o]) + row * d4;
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < d4) dst[c] = q[u];
        }
      }
    }
  }
  // the peer stores are visible system-wide before this kernel completes
  __threadfence_system();
}

// FP32 send (the gradient direction): row x[i] (times the gate weight when
// kWeighted) to the owners of the atom's K experts.
template <bool kWeighted>
__global__ void __launch_bounds__(kThreads)
ep_send_kernel(const float4* __restrict__ x, int64_t n_atoms, int d4, int K, const int32_t* __restrict__ slot_of,
               const int32_t* __restrict__ topk_expert, const float* __restrict__ w,
               const int32_t* __restrict__ src_off_r, const int32_t* __restrict__ dst_off_r, int E, int El,
               int64_t cap, PeerRows peers, WsHeader* ws) {
  const int lane = threadIdx.x % 32;
  const int64_t R = n_atoms * K;
  for (int64_t i = global_warp(); i < n_atoms; i += total_warps()) {
    int my_owner = 0;
    int64_t my_row = -1;
    float my_w = 1.0f;
    if (lane < K) {
      ep_dest(i * K + lane, R, E, El, slot_of, topk_expert, src_off_r, dst_off_r, cap, ws, &my_owner, &my_row);
      if (kWeighted) my_w = w[i * K + lane];
    }
    const float4* src = x + i * d4;
    for (int c0 = 0; c0 < d4; c0 += 32 * kU) {
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) v[u] = __ldcs(src + c);
      }
      for (int k = 0; k < K; ++k) {
        const int o = __shfl_sync(0xffffffffu, my_owner, k);
        const int64_t row = __shfl_sync(0xffffffffu, (long long)my_row, k);
        const float wk = kWeighted ? __shfl_sync(0xffffffffu, my_w, k) : 1.0f;
        if (row < 0) continue;                 // no room at the owner (same in every lane)
        float4* dst = reinterpret_cast<float4*>(peers.ptr[o]) + row * d4;
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < d4) dst[c] = kWeighted ? make_float4(v[u].x * wk, v[u].y * wk, v[u].z * wk, v[u].w * wk) : v[u];
        }
      }
    }
  }
  // the peer stores are visible system-wide before this kernel completes
  __threadfence_system();
}

// Owner side: received FP16 rows times their own scale (exact: powers of two).
// The row count is the last recv_off entry, read on the device.
__global__ void __launch_bounds__(kThreads)
ep_dequant_rows_kernel(const uint2* __restrict__ payload, const float* __restrict__ row_scale,
                       const int32_t* __restrict__ recv_off_r, int El, int64_t max_rows, int d4,
                       float4* __restrict__ xd) {
  const int64_t n = min((int64_t)recv_off_r[El], max_rows);
  const int lane = threadIdx.x % 32;
  for (int64_t p = global_warp(); p < n; p += total_warps()) {
    const float s = row_scale[p];
    const uint2* src = payload + p * d4;
    float4* dst = xd + p * d4;
    for (int c0 = 0; c0 < d4; c0 += 32 * kU) {
      uint2 q[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) q[u] = __ldcs(src + c);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) {
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&q[u].x));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&q[u].y));
          dst[c] = make_float4(a.x * s, a.y * s, b.x * s, b.y * s);
        }
      }
    }
  }
}

// Where owner row j (j < the received count) came from: its sender s and
// the row in the sender's local expert order.
__device__ __forceinline__ int64_t sender_row(const int32_t* __restrict__ src_off,
                                              const int32_t* __restrict__ dst_off,
                                              const int32_t* __restrict__ recv_off_r, int rank, int P, int E,
                                              int64_t j, int* sender) {
  const int El = E / P;
  int lo = 0, hi = El;                         // recv_off_r[lo] <= j < recv_off_r[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (recv_off_r[mid] <= j) lo = mid; else hi = mid;
  }
  const int e = rank * El + lo;
  int s = 0;                                   // the last sender whose block starts at or before j
  while (s + 1 < P && dst_off[(s + 1) * E + e] <= j) ++s;
  *sender = s;
  return (int64_t)src_off[s * (E + 1) + e] + (j - dst_off[s * E + e]);
}

// Owner side: each received row's result back to its sender's local row.
__global__ void __launch_bounds__(kThreads)
ep_return_kernel(const float4* __restrict__ yd, const int32_t* __restrict__ src_off,
                 const int32_t* __restrict__ dst_off, const int32_t* __restrict__ recv_off_r, int rank,
                 int P, int E, int64_t max_rows, int d4, PeerRows peers, int32_t* dbg) {
  const int64_t n = min((int64_t)recv_off_r[E / P], max_rows);
  const int lane = threadIdx.x % 32;
  for (int64_t j = global_warp(); j < n; j += total_warps()) {
    int s;
    const int64_t row = sender_row(src_off, dst_off, recv_off_r, rank, P, E, j, &s);
    if (kDebug && !in_range(row, src_off[s * (E + 1) + E])) {   // past the sender's routed rows
      if (lane == 0) debug_fault(dbg);
      continue;
    }
    const float4* src = yd + j * d4;
    float4* dst = reinterpret_cast<float4*>(peers.ptr[s]) + row * d4;
    for (int c0 = 0; c0 < d4; c0 += 32 * kU) {
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) v[u] = __ldcs(src + c);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) dst[c] = v[u];
      }
    }
  }
  // the peer stores are visible system-wide before this kernel completes
  __threadfence_system();
}

// Owner side of the fused return: the address in its sender's return buffer
// of every received row, for a GEMM epilogue that stores through the table.
__global__ void __launch_bounds__(kThreads)
ep_return_rows_kernel(const int32_t* __restrict__ src_off, const int32_t* __restrict__ dst_off,
                      const int32_t* __restrict__ recv_off_r, int rank, int P, int E, int64_t max_rows, int d,
                      PeerRows peers, float** __restrict__ rows, int32_t* dbg) {
  const int64_t n = min((int64_t)recv_off_r[E / P], max_rows);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += stride) {
    int s;
    const int64_t row = sender_row(src_off, dst_off, recv_off_r, rank, P, E, j, &s);
    if (kDebug && !in_range(row, src_off[s * (E + 1) + E])) {
      debug_fault(dbg);
      continue;
    }
    rows[j] = reinterpret_cast<float*>(peers.ptr[s]) + row * d;
  }
}

janus_status check_ep(int32_t rank, int32_t world, int32_t n_experts) {
  JANUS_CHECK_ARG(world >= 1 && world <= kMaxRanks && rank >= 0 && rank < world);
  JANUS_CHECK_ARG(n_experts >= world && n_experts <= kMaxExperts && n_experts % world == 0);
  return JANUS_OK;
}

janus_status peer_table(void* const* ptrs, float* const* scales, int32_t world, size_t align, PeerRows* t) {
  JANUS_CHECK_ARG(ptrs);
  for (int r = 0; r < kMaxRanks; ++r) {
    t->ptr[r] = nullptr;
    t->scale[r] = nullptr;
  }
  for (int r = 0; r < world; ++r) {
    JANUS_CHECK_ARG(ptrs[r]);
    JANUS_CHECK_ALIGN(aligned(ptrs[r], align));
    t->ptr[r] = ptrs[r];
    if (scales) {
      JANUS_CHECK_ARG(scales[r]);
      t->scale[r] = scales[r];
    }
  }
  return JANUS_OK;
}

}  // namespace
}  // namespace janus

using namespace janus;

extern "C" janus_status janus_ep_layout(const int32_t* counts_all, int32_t world, int32_t n_experts,
                                        int64_t recv_cap, int32_t* src_off, int32_t* dst_off, int32_t* recv_off,
                                        janus_stream_t stream) {
  janus_status st = check_ep(0, world, n_experts);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(recv_cap >= 0 && recv_cap < (int64_t)INT32_MAX);
  JANUS_CHECK_ARG(counts_all && src_off && dst_off && recv_off);
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  ep_layout_kernel<<<1, 256, 0, (cudaStream_t)stream>>>(counts_all, world, n_experts, recv_cap, src_off, dst_off,
                                                        recv_off);
  return launch_status();
}

extern "C" janus_status janus_ep_dispatch_quant(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                                                const int32_t* types, int32_t n_types, const int32_t* slot_of,
                                                const int32_t* topk_expert, const int32_t* src_off,
                                                const int32_t* dst_off, int32_t rank, int32_t world,
                                                int32_t n_experts, int64_t recv_cap, uint16_t* const* recv_payload,
                                                float* const* recv_scale, float* scale, void* workspace,
                                                size_t workspace_bytes, janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  janus_status st = check_ep(rank, world, n_experts);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(recv_cap >= 0 && recv_cap < (int64_t)INT32_MAX);
  JANUS_CHECK_ARG(n_atoms >= 0 && top_k >= 1 && top_k <= 32 && top_k <= n_experts);
  JANUS_CHECK_ARG(d >= 1 && d <= kMaxDim && n_types >= 1 && n_types <= kMaxTypes);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  JANUS_CHECK_ARG(n_atoms * (int64_t)top_k < (int64_t)INT32_MAX);
  size_t need = 0;
  st = janus_quant_by_type_workspace_size(n_types, &need);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(scale && workspace && workspace_bytes >= need && recv_scale);
  JANUS_CHECK_ARG(n_atoms == 0 || (x && types && slot_of && topk_expert && src_off && dst_off));
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  JANUS_CHECK_ALIGN(n_atoms == 0 || aligned(x, 16));
  PeerRows peers;
  st = peer_table(reinterpret_cast<void* const*>(recv_payload), recv_scale, world, 8, &peers);
  if (st != JANUS_OK) return st;
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  WsHeader* hdr = (WsHeader*)workspace;
  uint32_t* amax_bits = (uint32_t*)((char*)workspace + sizeof(WsHeader));
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, need, stream));
  const unsigned grid = rows_grid(n_atoms, 8);
  if (n_atoms > 0)
    quant_amax_kernel<<<rows_grid(row_items(n_atoms, d / 4), 8), kThreads, sizeof(uint32_t) * n_types, stream>>>(
        (const float4*)x, n_atoms, d / 4, types, n_types, amax_bits, hdr);
  ep_pack_send_kernel<<<grid, kThreads, 2 * sizeof(float) * n_types, stream>>>(
      (const float4*)x, n_atoms, d / 4, top_k, types, n_types, slot_of, topk_expert, amax_bits,
      src_off + (size_t)rank * (n_experts + 1), dst_off + (size_t)rank * n_experts, n_experts, n_experts / world,
      recv_cap, peers, scale, hdr);
  return launch_status();
}

extern "C" janus_status janus_ep_dispatch(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                                          const int32_t* slot_of, const int32_t* topk_expert,
                                          const float* topk_weight, const int32_t* src_off, const int32_t* dst_off,
                                          int32_t rank, int32_t world, int32_t n_experts, int64_t recv_cap,
                                          float* const* recv_rows, void* workspace, janus_stream_t stream) {
  janus_status st = check_ep(rank, world, n_experts);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(recv_cap >= 0 && recv_cap < (int64_t)INT32_MAX);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  JANUS_CHECK_ARG(n_atoms >= 0 && top_k >= 1 && top_k <= 32 && top_k <= n_experts);
  JANUS_CHECK_ARG(d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  JANUS_CHECK_ARG(n_atoms * (int64_t)top_k < (int64_t)INT32_MAX);
  PeerRows peers;
  st = peer_table(reinterpret_cast<void* const*>(recv_rows), nullptr, world, 16, &peers);
  if (st != JANUS_OK) return st;
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(x && slot_of && topk_expert && src_off && dst_off);
  JANUS_CHECK_ALIGN(aligned(x, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const unsigned grid = rows_grid(n_atoms, 8);
  const int32_t* so = src_off + (size_t)rank * (n_experts + 1);
  const int32_t* dof = dst_off + (size_t)rank * n_experts;
  WsHeader* hdr = (WsHeader*)workspace;   // may be NULL: faults are then not recorded
  if (topk_weight)
    ep_send_kernel<true><<<grid, kThreads, 0, (cudaStream_t)stream>>>(
        (const float4*)x, n_atoms, d / 4, top_k, slot_of, topk_expert, topk_weight, so, dof, n_experts,
        n_experts / world, recv_cap, peers, hdr);
  else
    ep_send_kernel<false><<<grid, kThreads, 0, (cudaStream_t)stream>>>(
        (const float4*)x, n_atoms, d / 4, top_k, slot_of, topk_expert, nullptr, so, dof, n_experts,
        n_experts / world, recv_cap, peers, hdr);
  return launch_status();
}

extern "C" janus_status janus_ep_dequant_rows(const uint16_t* payload, const float* row_scale,
                                              const int32_t* recv_off, int32_t rank, int32_t world,
                                              int32_t n_experts, int64_t max_rows, int32_t d, float* xd,
                                              janus_stream_t stream) {
  janus_status st = check_ep(rank, world, n_experts);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(max_rows >= 0 && d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  if (max_rows == 0) return JANUS_OK;
  JANUS_CHECK_ARG(payload && row_scale && recv_off && xd);
  JANUS_CHECK_ALIGN(aligned(payload, 8) && aligned(xd, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int El = n_experts / world;
  ep_dequant_rows_kernel<<<rows_grid(max_rows, 8), kThreads, 0, (cudaStream_t)stream>>>(
      (const uint2*)payload, row_scale, recv_off + (size_t)rank * (El + 1), El, max_rows, d / 4, (float4*)xd);
  return launch_status();
}

extern "C" janus_status janus_ep_return(const float* yd, const int32_t* counts_all, const int32_t* src_off,
                                        const int32_t* dst_off, const int32_t* recv_off, int32_t rank,
                                        int32_t world, int32_t n_experts, int64_t max_rows, int32_t d,
                                        float* const* ret_rows, janus_stream_t stream) {
  janus_status st = check_ep(rank, world, n_experts);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(max_rows >= 0 && d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  PeerRows peers;
  st = peer_table(reinterpret_cast<void* const*>(ret_rows), nullptr, world, 16, &peers);
  if (st != JANUS_OK) return st;
  if (max_rows == 0) return JANUS_OK;
  JANUS_CHECK_ARG(yd && counts_all && src_off && dst_off && recv_off);
  JANUS_CHECK_ALIGN(aligned(yd, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int El = n_experts / world;
  ep_return_kernel<<<rows_grid(max_rows, 8), kThreads, 0, (cudaStream_t)stream>>>(
      (const float4*)yd, src_off, dst_off, recv_off + (size_t)rank * (El + 1), rank, world, n_experts,
      max_rows, d / 4, peers, debug_fault_word());
  return launch_status();
}

extern "C" janus_status janus_ep_return_rows(const int32_t* src_off, const int32_t* dst_off,
                                             const int32_t* recv_off, int32_t rank, int32_t world,
                                             int32_t n_experts, int64_t max_rows, int32_t d,
                                             float* const* ret_rows, float** rows, janus_stream_t stream) {
  janus_status st = check_ep(rank, world, n_experts);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(max_rows >= 0 && d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  PeerRows peers;
  st = peer_table(reinterpret_cast<void* const*>(ret_rows), nullptr, world, 16, &peers);
  if (st != JANUS_OK) return st;
  if (max_rows == 0) return JANUS_OK;
  JANUS_CHECK_ARG(rows && src_off && dst_off && recv_off);
  JANUS_CHECK_ALIGN(aligned(rows, 8));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int El = n_experts / world;
  const int64_t blocks = std::min<int64_t>((max_rows + kThreads - 1) / kThreads, (int64_t)num_sms() * 8);
  ep_return_rows_kernel<<<(unsigned)blocks, kThreads, 0, (cudaStream_t)stream>>>(
      src_off, dst_off, recv_off + (size_t)rank * (El + 1), rank, world, n_experts, max_rows, d, peers, rows,
      debug_fault_word());
  return launch_status();
}

// ---- CUDA IPC: map another process's buffer (same node) ---------------------
// A handle names the whole allocation that holds the pointer (PyTorch
// sub-allocates), so the byte offset of the pointer inside it travels along.
namespace {
typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (AddressRangeFn)p;
  });
  return fn;
}
}  // namespace

extern "C" janus_status janus_ipc_get_handle(const void* dev_ptr, janus_ipc_handle* out) {
  JANUS_CHECK_ARG(dev_ptr && out);
  AddressRangeFn range = address_range_fn();
  if (!range) return JANUS_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, (CUdeviceptr)dev_ptr) != CUDA_SUCCESS) return JANUS_ERR_CUDA;
  cudaIpcMemHandle_t h;
  JANUS_CUDA_TRY(cudaIpcGetMemHandle(&h, (void*)base));
  static_assert(sizeof(h) <= sizeof(out->bytes), "IPC handle size");
  memcpy(out->bytes, &h, sizeof(h));
  out->offset = (uint64_t)((CUdeviceptr)dev_ptr - base);
  return JANUS_OK;
}

extern "C" janus_status janus_ipc_open_handle(const janus_ipc_handle* handle, void** dev_ptr) {
  JANUS_CHECK_ARG(handle && dev_ptr);
  cudaIpcMemHandle_t h;
  memcpy(&h, handle->bytes, sizeof(h));
  void* base = nullptr;
  JANUS_CUDA_TRY(cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess));
  *dev_ptr = (char*)base + handle->offset;
  return JANUS_OK;
}

extern "C" janus_status janus_ipc_close_handle(void* dev_ptr, uint64_t offset) {
  JANUS_CHECK_ARG(dev_ptr);
  JANUS_CUDA_TRY(cudaIpcCloseMemHandle((char*)dev_ptr - offset));
  return JANUS_OK;
}
