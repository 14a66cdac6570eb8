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
//   * one warp per atom, U = 4 column float4s per lane and the edge loop
//     unrolled by 4 -> up to 16 independent 16-byte loads per lane in flight;
//   * FP32 accumulation in edge order, each output row written once;
//   * 64-bit element offsets (Ed*d exceeds 2^31 at production sizes).
#include "common.cuh"

namespace janus {
namespace {

constexpr int kThreads = 256;
constexpr int kU = 4;
constexpr int kEdgeUnroll = 4;

__global__ void __launch_bounds__(kThreads)
edge_aggregate_kernel(const float4* __restrict__ msg, const int64_t* __restrict__ row_ptr,
                      int64_t n_atoms, int d4, float4* __restrict__ out) {
  const int lane = threadIdx.x % 32;
  const int64_t nwarps = (int64_t)gridDim.x * kThreads / 32;
  for (int64_t i = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / 32; i < n_atoms; i += nwarps) {
    const int64_t e0 = row_ptr[i], e1 = row_ptr[i + 1];
    for (int c0 = 0; c0 < d4; c0 += 32 * kU) {
      float4 acc[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      int64_t e = e0;
      for (; e + kEdgeUnroll <= e1; e += kEdgeUnroll) {
        float4 v[kEdgeUnroll][kU];
#pragma unroll
        for (int r = 0; r < kEdgeUnroll; ++r)
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int c = c0 + u * 32 + lane;
            v[r][u] = c < d4 ? __ldcs(msg + (e + r) * d4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
        for (int r = 0; r < kEdgeUnroll; ++r)
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            acc[u].x += v[r][u].x; acc[u].y += v[r][u].y;
            acc[u].z += v[r][u].z; acc[u].w += v[r][u].w;
          }
      }
      for (; e < e1; ++e) {
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < d4) {
            const float4 v = __ldcs(msg + e * d4 + c);
            acc[u].x += v.x; acc[u].y += v.y; acc[u].z += v.z; acc[u].w += v.w;
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

extern "C" janus_status janus_edge_aggregate(const float* msg, const int64_t* row_ptr,
                                             int64_t n_atoms, int32_t d, float* out,
                                             janus_stream_t stream) {
  JANUS_CHECK_ARG(n_atoms >= 0 && d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  if (n_atoms == 0) return JANUS_OK;
  // msg may be NULL only for a CSR without edges: it is read at
  // [row_ptr[i], row_ptr[i+1]) only.
  JANUS_CHECK_ARG(row_ptr && out);
  JANUS_CHECK_ALIGN(aligned(msg, 16) && aligned(out, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int64_t need = (n_atoms + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  const unsigned grid = (unsigned)(need < cap ? need : cap);
  edge_aggregate_kernel<<<grid, kThreads, 0, (cudaStream_t)stream>>>(
      (const float4*)msg, row_ptr, n_atoms, d / 4, (float4*)out);
  return launch_status();
}
