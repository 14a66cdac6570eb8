// Row-streaming helpers and the per-type absmax pass of the FP16 packing,
// shared by the local token movement (moe_io.cu) and the expert-parallel
// exchange (ep.cu).  Internal header; everything has internal linkage.
//
// Source: paper review "Breaking the Training Barrier of Billion-Parameter
// Universal Machine Learning Interatomic Potentials" section 3.5 (atom-type-
// aware FP16 compression of the dispatch volume).
#pragma once

#include "common.cuh"

namespace janus {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerBlock = kThreads / 32;
constexpr int kU = 4;

inline unsigned rows_grid(int64_t rows, int blocks_per_sm) {
  int64_t need = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  int64_t cap = (int64_t)num_sms() * blocks_per_sm;
  return (unsigned)(need < cap ? (need > 0 ? need : 1) : cap);
}

__device__ __forceinline__ int64_t global_warp() {
  return ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
}
__device__ __forceinline__ int64_t total_warps() {
  return (int64_t)gridDim.x * blockDim.x / 32;
}

// Work items of the row-streaming kernels: (row, chunk of 32 * kU float4
// columns).  Warp w of the grid always takes column chunk w % nch and strides
// over the rows w / nch, w / nch + W / nch, ... (W warps, nch chunks per row),
// so a layer with fewer rows than the grid has warps (the S layer's 8,192
// atoms, the L layer's 16,384 receivers) still fills every warp, the chunks of
// one row go to neighbouring warps at about the same time, and no warp divides
// per item.  The last W % nch warps of the grid stay idle.
constexpr int kChunk4 = 32 * kU;
inline int64_t row_items(int64_t rows, int d4) { return rows * ((d4 + kChunk4 - 1) / kChunk4); }

struct ChunkWalk {
  int64_t row0, stride;   // first row, row stride (0 rows for an idle warp)
  int c0;                 // first float4 column of the warp's chunk
};
__device__ __forceinline__ ChunkWalk chunk_walk(int d4) {
  const int nch = (d4 + kChunk4 - 1) / kChunk4;
  const int64_t w = global_warp(), W = total_warps();
  ChunkWalk cw;
  cw.stride = W / nch;
  cw.row0 = w < cw.stride * nch ? w / nch : INT64_MAX;
  cw.c0 = (int)(w % nch) * kChunk4;
  return cw;
}

// ---- atom-type-aware FP16 packing: per-type absmax and scale ------------

// |x| as ordered bits: for non-negative floats the integer order is the
// float order, and any NaN compares above +inf.
__device__ __forceinline__ uint32_t abs_bits(float v) { return __float_as_uint(v) & 0x7fffffffu; }

__global__ void __launch_bounds__(kThreads)
quant_amax_kernel(const float4* __restrict__ x, int64_t n_atoms, int d4,
                  const int32_t* __restrict__ types, int T, uint32_t* __restrict__ amax_bits,
                  WsHeader* ws) {
  extern __shared__ uint32_t s_amax[];
  for (int t = threadIdx.x; t < T; t += kThreads) s_amax[t] = 0;
  __syncthreads();
  const int lane = threadIdx.x % 32;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  for (int64_t i = cw.row0; i < n_atoms; i += cw.stride) {
    int t = types[i];
    if (t < 0 || t >= T) {
      if (lane == 0) record_fault(ws, kFaultBadType);
      t = 0;
    }
    const float4* src = x + i * d4;
    uint32_t m = 0;
    float4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + u * 32 + lane;
      v[u] = c < d4 ? __ldg(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      m = max(m, max(max(abs_bits(v[u].x), abs_bits(v[u].y)), max(abs_bits(v[u].z), abs_bits(v[u].w))));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0 && m) atomicMax(&s_amax[t], m);
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += kThreads)
    if (s_amax[t]) atomicMax(&amax_bits[t], s_amax[t]);
}

// Exponent e of the type scale 2^e: the smallest e with amax <= 65504 * 2^e,
// clamped to [-126, 127].  With amax = 1.M * 2^(Eb-127) (Eb = biased
// exponent field), 65504 = (2 - 2^-10) * 2^15, so e = Eb - 142, plus one when
// the mantissa exceeds that of 65504 (M > 0x7FE000).
__device__ __forceinline__ int scale_exponent_from_bits(uint32_t amax) {
  if (amax == 0) return 0;
  const int eb = (int)(amax >> 23);
  const uint32_t mant = amax & 0x7fffffu;
  int e = (eb == 0) ? -126 : eb - 142 + (mant > 0x7fe000u ? 1 : 0);
  return e < -126 ? -126 : (e > 127 ? 127 : e);
}

}  // namespace
}  // namespace janus
