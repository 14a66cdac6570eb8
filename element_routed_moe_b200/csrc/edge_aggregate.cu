// janus_edge_aggregate: segment sum of receiver-sorted edge messages into
// their receiver atoms.
//
// Source: paper review "Breaking the Training Barrier of Billion-Parameter
// Universal Machine Learning Interatomic Potentials" section 3.5 (CNIS
// high-performance kernels: neighbour aggregation with fused indexing for
// coalesced access; edge aggregation recast as a GEMM-based reduction).
// Those kernels were written for another machine; here the reduction is a
// pure HBM stream (one pass over Ed*d*4 bytes, ~0.25 flop/byte), so it is
// neither a GEMM nor a scatter with atomics:
//   * receiver-sorted CSR: atom i's messages are one contiguous block
//     msg[row_ptr[i] : row_ptr[i+1], :], so every load is a coalesced 128-bit
//     streaming load (evict-first, the messages are read exactly once);
//   * one warp per work item (receiver, chunk of 128 float4 columns), so a
//     layer with fewer receivers than the grid has warps still fills them;
//     U = 4 column float4s per lane and the edge loop unrolled by 4 -> up to
//     16 independent 16-byte loads per lane in flight;
//   * FP32 accumulation: each group of 4 edges is summed pairwise and then
//     added to the running sum (edge order otherwise); each output row is
//     written once;
//   * 64-bit element offsets (Ed*d exceeds 2^31 at production sizes);
//   * message row 0 is edge row_ptr[0], so a receiver range of a larger CSR
//     runs as it stands (the pinned-host pipeline streams the messages in
//     such chunks);
//   * every edge range is clamped to [0, n_edges), so a malformed row_ptr
//     cannot make a kernel read or write outside the message buffer (debug
//     builds also record the fault).
#include "common.cuh"

namespace janus {
namespace {

constexpr int kThreads = 256;
constexpr int kU = 4;
constexpr int kChunk4 = 32 * kU;   // float4 columns of one work item (receiver, column chunk)

// Warp w takes column chunk w % nch of receivers w / nch, w / nch + W / nch,
// ... (W warps, nch chunks per row; the last W % nch warps stay idle): the
// chunks of one receiver go to neighbouring warps, and no warp divides per item.
struct ChunkWalk {
  int64_t row0, stride;
  int c0;
};
__device__ __forceinline__ ChunkWalk chunk_walk(int d4) {
  const int nch = (d4 + kChunk4 - 1) / kChunk4;
  const int64_t w = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / 32;
  const int64_t W = (int64_t)gridDim.x * kThreads / 32;
  ChunkWalk cw;
  cw.stride = W / nch;
  cw.row0 = w < cw.stride * nch ? w / nch : INT64_MAX;
  cw.c0 = (int)(w % nch) * kChunk4;
  return cw;
}
constexpr int kEdgeUnroll = 4;
static_assert(kEdgeUnroll == 4, "the pairwise group sum below is written for 4 edges");

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// Receiver i's rows of the message buffer, [*e0, *e1): msg row 0 is edge
// row_ptr[0], so a receiver range of a larger CSR (row_ptr + i0 with the
// messages of edges [row_ptr[i0], row_ptr[i1])) is processed as it stands.
// The range is clamped to [0, n_edges]: a row_ptr that decreases or runs past
// the edge count gives a shorter (possibly empty) range instead of an
// out-of-bounds access; debug builds record it.
__device__ __forceinline__ void edge_range(const int64_t* __restrict__ row_ptr, int64_t i, int64_t n_edges,
                                           int32_t* dbg, int64_t* e0, int64_t* e1) {
  const int64_t base = row_ptr[0];
  const int64_t a = row_ptr[i] - base, b = row_ptr[i + 1] - base;
  if (kDebug && (a < 0 || b < a || b > n_edges) && (threadIdx.x % 32) == 0) debug_fault(dbg);
  *e0 = min(max(a, (int64_t)0), n_edges);
  *e1 = min(max(b, *e0), n_edges);
}

__global__ void __launch_bounds__(kThreads)
edge_aggregate_kernel(const float4* __restrict__ msg, const int64_t* __restrict__ row_ptr,
                      int64_t n_atoms, int64_t n_edges, int d4, float4* __restrict__ out, int32_t* dbg) {
  const int lane = threadIdx.x % 32;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  // float4 columns of this lane inside the chunk (kU except in a ragged last chunk)
  const int nu = min(kU, max(0, (d4 - c0 - lane + 31) / 32));
  for (int64_t i = cw.row0; i < n_atoms; i += cw.stride) {
    int64_t e0, e1;
    edge_range(row_ptr, i, n_edges, dbg, &e0, &e1);
    float4 acc[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* p = msg + e0 * d4 + c0 + lane;     // edge e0, this lane's first column
    int n = (int)(e1 - e0);
    for (; n >= kEdgeUnroll; n -= kEdgeUnroll, p += (int64_t)kEdgeUnroll * d4) {
      float4 v[kEdgeUnroll][kU];
#pragma unroll
      for (int r = 0; r < kEdgeUnroll; ++r)
#pragma unroll
        for (int u = 0; u < kU; ++u)
          v[r][u] = u < nu ? __ldcs(p + r * d4 + u * 32) : make_float4(0.f, 0.f, 0.f, 0.f);
      // pairwise within the group of 4, then one add into the running sum
      // (a 4x shorter rounding chain for high-degree receivers)
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const float4 a = f4add(v[0][u], v[1][u]), b = f4add(v[2][u], v[3][u]);
        acc[u] = f4add(acc[u], f4add(a, b));
      }
    }
    for (; n > 0; --n, p += d4) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if (u < nu) {
          const float4 v = __ldcs(p + u * 32);
          acc[u].x += v.x; acc[u].y += v.y; acc[u].z += v.z; acc[u].w += v.w;
        }
      }
    }
    float4* dst = out + i * d4 + c0 + lane;
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (u < nu) dst[u * 32] = acc[u];
  }
}

// Gradient of the edge aggregation: every edge of receiver i gets dX[i,:].
// One warp per receiver: the dX row chunk is loaded once and written to the
// receiver's contiguous block of edge rows with streaming stores.
__global__ void __launch_bounds__(kThreads)
edge_broadcast_kernel(const float4* __restrict__ dx, const int64_t* __restrict__ row_ptr, int64_t n_atoms,
                      int64_t n_edges, int d4, float4* __restrict__ dmsg, int32_t* dbg) {
  const int lane = threadIdx.x % 32;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  for (int64_t i = cw.row0; i < n_atoms; i += cw.stride) {
    int64_t e0, e1;
    edge_range(row_ptr, i, n_edges, dbg, &e0, &e1);
    if (e1 <= e0) continue;
    float4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + u * 32 + lane;
      v[u] = c < d4 ? __ldg(dx + i * d4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int64_t e = e0; e < e1; ++e) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) __stcs(dmsg + e * d4 + c, v[u]);
      }
    }
  }
}

// Neighbour aggregation through the sender index: out[i,:] = sum over the
// receiver's edges of x[senders[e],:].  One warp per receiver; the sender ids
// of 32 edges are read with one coalesced load and broadcast by shuffles;
// rows are gathered 4 edges at a time (U float4s each) for memory-level
// parallelism; FP32 accumulation as in edge_aggregate_kernel.  Senders outside [0, N) are
// skipped (they contribute nothing; debug builds record them), so a bad index
// cannot read out of bounds.
__global__ void __launch_bounds__(kThreads)
neighbor_aggregate_kernel(const float4* __restrict__ x, const int64_t* __restrict__ row_ptr,
                          const int32_t* __restrict__ senders, int64_t n_atoms, int64_t n_edges, int d4,
                          float4* __restrict__ out, int32_t* dbg) {
  const int lane = threadIdx.x % 32;
  const int64_t nwarps = (int64_t)gridDim.x * kThreads / 32;
  for (int64_t i = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / 32; i < n_atoms; i += nwarps) {
    int64_t e0, e1;
    edge_range(row_ptr, i, n_edges, dbg, &e0, &e1);
    for (int c0 = 0; c0 < d4; c0 += 32 * kU) {
      float4 acc[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int64_t eb = e0; eb < e1; eb += 32) {
        const int64_t my_e = eb + lane;
        int32_t my_s = my_e < e1 ? senders[my_e] : -1;
        if (my_e < e1 && !in_range(my_s, n_atoms)) {
          debug_fault(dbg);
          my_s = -1;
        }
        const int n_here = (int)min((int64_t)32, e1 - eb);
        for (int t = 0; t < n_here; t += 4) {
          int32_t s4[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) s4[r] = __shfl_sync(0xffffffffu, my_s, (t + r) & 31);
          float4 v[4][kU];
#pragma unroll
          for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int u = 0; u < kU; ++u) {
              const int c = c0 + u * 32 + lane;
              const bool ok = (t + r < n_here) && s4[r] >= 0 && c < d4;
              v[r][u] = ok ? __ldg(x + (int64_t)s4[r] * d4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const float4 a = f4add(v[0][u], v[1][u]), b = f4add(v[2][u], v[3][u]);
            acc[u] = f4add(acc[u], f4add(a, b));
          }
        }
      }
      float4* dst = out + i * d4;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) dst[c] = acc[u];
      }
    }
  }
}

}  // namespace
}  // namespace janus

using namespace janus;

extern "C" janus_status janus_edge_aggregate(const float* msg, int64_t n_edges, const int64_t* row_ptr,
                                             int64_t n_atoms, int32_t d, float* out,
                                             janus_stream_t stream) {
  JANUS_CHECK_ARG(n_atoms >= 0 && n_edges >= 0 && d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(row_ptr && out && (msg || n_edges == 0));
  JANUS_CHECK_ALIGN(aligned(msg, 16) && aligned(out, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int64_t need = (n_atoms * ((d / 4 + kChunk4 - 1) / kChunk4) + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  const unsigned grid = (unsigned)(need < cap ? need : cap);
  edge_aggregate_kernel<<<grid, kThreads, 0, (cudaStream_t)stream>>>(
      (const float4*)msg, row_ptr, n_atoms, n_edges, d / 4, (float4*)out, debug_fault_word());
  return launch_status();
}

extern "C" janus_status janus_edge_broadcast(const float* dx, const int64_t* row_ptr, int64_t n_atoms,
                                             int32_t d, float* dmsg, int64_t n_edges, janus_stream_t stream) {
  JANUS_CHECK_ARG(n_atoms >= 0 && n_edges >= 0 && d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(dx && row_ptr && (dmsg || n_edges == 0));
  JANUS_CHECK_ALIGN(aligned(dx, 16) && aligned(dmsg, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int64_t need = (n_atoms * ((d / 4 + kChunk4 - 1) / kChunk4) + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  edge_broadcast_kernel<<<(unsigned)(need < cap ? need : cap), kThreads, 0, (cudaStream_t)stream>>>(
      (const float4*)dx, row_ptr, n_atoms, n_edges, d / 4, (float4*)dmsg, debug_fault_word());
  return launch_status();
}

extern "C" janus_status janus_neighbor_aggregate(const float* x, const int64_t* row_ptr,
                                                 const int32_t* senders, int64_t n_edges, int64_t n_atoms,
                                                 int32_t d, float* out, janus_stream_t stream) {
  JANUS_CHECK_ARG(n_atoms >= 0 && n_atoms < (int64_t)INT32_MAX && n_edges >= 0 && d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(x && row_ptr && out && (senders || n_edges == 0));
  JANUS_CHECK_ALIGN(aligned(x, 16) && aligned(out, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int64_t need = (n_atoms + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  neighbor_aggregate_kernel<<<(unsigned)(need < cap ? need : cap), kThreads, 0, (cudaStream_t)stream>>>(
      (const float4*)x, row_ptr, senders, n_atoms, n_edges, d / 4, (float4*)out, debug_fault_word());
  return launch_status();
}
