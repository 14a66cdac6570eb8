// Token movement of the MoE layer: dispatch, combine, and the atom-type-aware
// FP16 packing of the dispatch buffer.
//
// Sources: paper review "Breaking the Training Barrier of Billion-Parameter
// Universal Machine Learning Interatomic Potentials" section 3.5 (CNIS:
// MoE dispatch/combine kernels; atom-type-aware FP16 compression), and
// "MatRIS-MoE与Janus框架" section 3.2 (gate-weighted sum of expert outputs).
//
// All four are HBM-bound streams.  Layout choices for B200:
//   * one warp per work item (row, chunk of 128 float4 columns), 128-bit
//     accesses, U = 4 independent 16-byte loads per lane in flight (2 KB per
//     warp) before any store;
//   * dispatch and pack run in scatter form: the atom row is read once and
//     written to its K dispatch rows (slot_of gives each destination; every
//     destination is distinct, so no atomics and a deterministic result);
//   * combine runs in gather form: the K expert rows of an atom are read and
//     summed in k order, one output row written;
//   * grids are a multiple of the SM count with grid-stride loops over rows.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "rows.cuh"

namespace janus {
namespace {

// slot_of / weight of the atom's k-th slot: lanes < K hold them when K <= 32
template <bool kWeighted>
__device__ __forceinline__ void slot_k(int k, int K, int64_t i, int my_slot, float my_w,
                                       const int32_t* __restrict__ slot_of,
                                       const float* __restrict__ w, int64_t* p, float* wk) {
  if (K <= 32) {
    *p = __shfl_sync(0xffffffffu, my_slot, k);
    *wk = kWeighted ? __shfl_sync(0xffffffffu, my_w, k) : 1.0f;
  } else {
    *p = slot_of[i * K + k];
    *wk = kWeighted ? w[i * K + k] : 1.0f;
  }
}

template <bool kWeighted>
__global__ void __launch_bounds__(kThreads)
dispatch_kernel(const float4* __restrict__ x, int64_t n_atoms, int d4, int K,
                const int32_t* __restrict__ slot_of, const float* __restrict__ w,
                float4* __restrict__ xd, int32_t* dbg) {
  const int64_t R = n_atoms * K;
  const int lane = threadIdx.x % 32;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  for (int64_t i = cw.row0; i < n_atoms; i += cw.stride) {
    const int my_slot = lane < K ? slot_of[i * K + lane] : 0;
    const float my_w = (kWeighted && lane < K) ? w[i * K + lane] : 1.0f;
    const float4* src = x + i * d4;
    float4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + u * 32 + lane;
      if (c < d4) v[u] = __ldcs(src + c);
    }
    for (int k = 0; k < K; ++k) {
      int64_t p;
      float wk;
      slot_k<kWeighted>(k, K, i, my_slot, my_w, slot_of, w, &p, &wk);
      if (kDebug && !in_range(p, R)) {   // p is the same in every lane
        if (lane == 0) debug_fault(dbg);
        continue;
      }
      float4* dst = xd + p * d4;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) {
          float4 o = v[u];
          if (kWeighted) { o.x *= wk; o.y *= wk; o.z *= wk; o.w *= wk; }
          dst[c] = o;
        }
      }
    }
  }
}

// acc += wk * v (or acc += v), one FMA (add) per component, in the caller's k order
template <bool kWeighted>
__device__ __forceinline__ void accumulate(float4& acc, float wk, const float4& v) {
  if (kWeighted) {
    acc.x = fmaf(wk, v.x, acc.x);
    acc.y = fmaf(wk, v.y, acc.y);
    acc.z = fmaf(wk, v.z, acc.z);
    acc.w = fmaf(wk, v.w, acc.w);
  } else {
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
}

// Gather form: the K expert rows of one (atom, column chunk) item are added
// in ascending k.
template <bool kWeighted>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const float4* __restrict__ yd, const int32_t* __restrict__ slot_of,
               const float* __restrict__ w, int64_t n_atoms, int K, int d4,
               float4* __restrict__ y, int32_t* dbg) {
  const int64_t R = n_atoms * K;
  const int lane = threadIdx.x % 32;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  const int nu = min(kU, max(0, (d4 - c0 - lane + 31) / 32));   // this lane's columns in the chunk
  const float4* yl = yd + c0 + lane;
  for (int64_t i = cw.row0; i < n_atoms; i += cw.stride) {
    const int my_slot = lane < K ? slot_of[i * K + lane] : 0;
    const float my_w = (kWeighted && lane < K) ? w[i * K + lane] : 1.0f;
    float4 acc[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < K; ++k) {
      int64_t p;
      float wk;
      slot_k<kWeighted>(k, K, i, my_slot, my_w, slot_of, w, &p, &wk);
      if (kDebug && !in_range(p, R)) {   // p is the same in every lane
        if (lane == 0) debug_fault(dbg);
        continue;
      }
      const float4* src = yl + p * d4;
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) v[u] = u < nu ? __ldcs(src + u * 32) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < kU; ++u) accumulate<kWeighted>(acc[u], wk, v[u]);
    }
    float4* dst = y + i * d4 + c0 + lane;
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (u < nu) dst[u * 32] = acc[u];
  }
}

// ---- dispatch into two FP16 terms per value (the FP16 tensor-core GEMMs) ----
//
// Each dispatch row p (slot s = i K + k) is written as hi and mid binary16
// planes with one power-of-two scale S_p per row:  v = (w_k) x[i, :] (the
// same FP32 value janus_dispatch writes), hi = fp16(v S_p), mid =
// fp16(v S_p - hi), row_scale[p] = 1 / S_p.  S_p puts the row's largest |v|,
// |w_k| max_j |x[i, j]| (rounding is monotonic), in [2^14, 2^15); a value
// within 2^18 of that maximum keeps 22 significant bits, smaller ones an
// absolute error below 2^-40 of it.  The row maxima come from a first pass.

// rowmax[i] = max_j |x[i, j]| as ordered bits (atomicMax per chunk item)
__global__ void __launch_bounds__(kThreads)
row_absmax_kernel(const float4* __restrict__ x, int64_t n_atoms, int d4, uint32_t* __restrict__ rowmax) {
  const int lane = threadIdx.x % 32;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  for (int64_t i = cw.row0; i < n_atoms; i += cw.stride) {
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + u * 32 + lane;
      if (c < d4) {
        const float4 v = __ldg(x + i * d4 + c);
        m = max(m, max(max(abs_bits(v.x), abs_bits(v.y)), max(abs_bits(v.z), abs_bits(v.w))));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0 && m) atomicMax(rowmax + i, m);
  }
}

// exponent e of S = 2^e for a row maximum m (bits): m 2^e in [2^14, 2^15),
// clamped to [-126, 126]; 0 for a zero row
__device__ __forceinline__ int split_exp(uint32_t m) {
  if (m == 0) return 0;
  const int b = max((int)(m >> 23), 1);
  return min(max(141 - b, -126), 126);
}

__device__ __forceinline__ uint2 halves(float a, float b, float c, float d) {
  const __half2 lo = __floats2half2_rn(a, b), hi = __floats2half2_rn(c, d);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}

template <bool kWeighted>
__global__ void __launch_bounds__(kThreads)
dispatch_split_kernel(const float4* __restrict__ x, int64_t n_atoms, int d4, int K, const int32_t* __restrict__ slot_of,
                      const float* __restrict__ w, const uint32_t* __restrict__ rowmax, uint2* __restrict__ rows16,
                      float* __restrict__ row_scale, int32_t* dbg) {
  const int64_t R = n_atoms * K;
  const int lane = threadIdx.x % 32;
  uint2* mid_plane = rows16 + R * d4;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  for (int64_t i = cw.row0; i < n_atoms; i += cw.stride) {
    const int my_slot = lane < K ? slot_of[i * K + lane] : 0;
    const float my_w = (kWeighted && lane < K) ? w[i * K + lane] : 1.0f;
    const float m = __uint_as_float(rowmax[i]);
    float4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + u * 32 + lane;
      v[u] = c < d4 ? __ldcs(x + i * d4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // unweighted: every destination gets the same two terms, split once
    uint2 hq0[kU], mq0[kU];
    const int e0 = split_exp(__float_as_uint(m));
    if (!kWeighted) {
      const float S = __uint_as_float((uint32_t)(127 + e0) << 23);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        float4 o = v[u];
        o.x *= S; o.y *= S; o.z *= S; o.w *= S;
        hq0[u] = halves(o.x, o.y, o.z, o.w);
        const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&hq0[u].x));
        const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&hq0[u].y));
        mq0[u] = halves(o.x - h0.x, o.y - h0.y, o.z - h1.x, o.w - h1.y);
      }
    }
    for (int k = 0; k < K; ++k) {
      int64_t p;
      float wk;
      slot_k<kWeighted>(k, K, i, my_slot, my_w, slot_of, w, &p, &wk);
      if (kDebug && !in_range(p, R)) {   // p is the same in every lane
        if (lane == 0) debug_fault(dbg);
        continue;
      }
      const int e = kWeighted ? split_exp(__float_as_uint(fabsf(wk) * m)) : e0;
      const float S = __uint_as_float((uint32_t)(127 + e) << 23);
      if (c0 == 0 && lane == 0) row_scale[p] = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) {
          if (!kWeighted) {
            rows16[p * d4 + c] = hq0[u];
            mid_plane[p * d4 + c] = mq0[u];
            continue;
          }
          float4 o = v[u];
          o.x *= wk; o.y *= wk; o.z *= wk; o.w *= wk;
          o.x *= S; o.y *= S; o.z *= S; o.w *= S;
          const uint2 hq = halves(o.x, o.y, o.z, o.w);
          const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&hq.x));
          const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&hq.y));
          rows16[p * d4 + c] = hq;
          mid_plane[p * d4 + c] = halves(o.x - h0.x, o.y - h0.y, o.z - h1.x, o.w - h1.y);
        }
      }
    }
  }
}

// ---- atom-type-aware FP16 packing ------------------------------------------

__global__ void __launch_bounds__(kThreads)
quant_pack_kernel(const float4* __restrict__ x, int64_t n_atoms, int d4, int K,
                  const int32_t* __restrict__ types, int T, const int32_t* __restrict__ slot_of,
                  const uint32_t* __restrict__ amax_bits, uint2* __restrict__ payload,
                  float* __restrict__ scale, WsHeader* ws) {
  extern __shared__ float s_inv[];
  const int64_t R = n_atoms * K;
  for (int t = threadIdx.x; t < T; t += kThreads) {
    const uint32_t a = amax_bits[t];
    const int e = scale_exponent_from_bits(a);
    // 2^-e is a normal float for every e a finite amax can produce
    s_inv[t] = (e <= 126) ? __uint_as_float((uint32_t)(127 - e) << 23) : 0.0f;
    if (blockIdx.x == 0) {
      scale[t] = __uint_as_float((uint32_t)(127 + e) << 23);
      if (a >= 0x7f800000u) record_fault(ws, kFaultNonFinite);
    }
  }
  __syncthreads();
  const int lane = threadIdx.x % 32;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  for (int64_t i = cw.row0; i < n_atoms; i += cw.stride) {
    int t = types[i];
    if (t < 0 || t >= T) t = 0;                // recorded by the amax pass
    const float inv = s_inv[t];
    const int my_slot = lane < K ? slot_of[i * K + lane] : 0;
    const float4* src = x + i * d4;
    uint2 q[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + u * 32 + lane;
      if (c < d4) {
        const float4 v = __ldcs(src + c);
        // exact power-of-two scaling, then one round-to-nearest-even
        const __half2 lo = __floats2half2_rn(v.x * inv, v.y * inv);
        const __half2 hi = __floats2half2_rn(v.z * inv, v.w * inv);
        q[u].x = *reinterpret_cast<const uint32_t*>(&lo);
        q[u].y = *reinterpret_cast<const uint32_t*>(&hi);
      }
    }
    for (int k = 0; k < K; ++k) {
      const int64_t p = K <= 32 ? __shfl_sync(0xffffffffu, my_slot, k) : slot_of[i * K + k];
      if (kDebug && !in_range(p, R)) {
        if (lane == 0) debug_fault(&ws->error);
        continue;
      }
      uint2* dst = payload + p * d4;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < d4) dst[c] = q[u];
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads)
dequant_kernel(const uint2* __restrict__ payload, int64_t n_rows, int d4, int K,
               const int32_t* __restrict__ types, int T, const int32_t* __restrict__ perm,
               const float* __restrict__ scale, float4* __restrict__ xd, int32_t* dbg) {
  const int lane = threadIdx.x % 32;
  const ChunkWalk cw = chunk_walk(d4);
  const int c0 = cw.c0;
  for (int64_t p = cw.row0; p < n_rows; p += cw.stride) {
    const int32_t slot = perm[p];
    if (kDebug && !in_range(slot, n_rows)) {
      if (lane == 0) debug_fault(dbg);
      continue;
    }
    int t = types[slot / K];
    if (t < 0 || t >= T) t = 0;
    const float s = scale[t];
    const uint2* src = payload + p * d4;
    float4* dst = xd + p * d4;
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

// row_scale[p] = scale[type of dispatch row p] (bad type ids as type 0, as in
// the dequant kernel).
__global__ void __launch_bounds__(kThreads)
row_scale_kernel(int64_t n_rows, int K, const int32_t* __restrict__ types, int T,
                 const int32_t* __restrict__ perm, const float* __restrict__ scale, float* __restrict__ row_scale,
                 int32_t* dbg) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n_rows; p += stride) {
    const int32_t slot = perm[p];
    if (kDebug && !in_range(slot, n_rows)) {
      debug_fault(dbg);
      continue;
    }
    int t = types[slot / K];
    if (t < 0 || t >= T) t = 0;
    row_scale[p] = scale[t];
  }
}

}  // namespace
}  // namespace janus

using namespace janus;

static janus_status check_rows(int64_t n_atoms, int32_t d, int32_t top_k) {
  JANUS_CHECK_ARG(n_atoms >= 0 && top_k >= 1 && top_k <= kMaxExperts);
  JANUS_CHECK_ARG(d >= 1 && d <= kMaxDim);
  JANUS_CHECK_ARG(n_atoms * (int64_t)top_k < (int64_t)INT32_MAX);
  JANUS_CHECK_ALIGN(d % 4 == 0);
  return JANUS_OK;
}

extern "C" janus_status janus_dispatch(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                                       const int32_t* slot_of, const float* topk_weight,
                                       float* xd, janus_stream_t stream) {
  janus_status st = check_rows(n_atoms, d, top_k);
  if (st != JANUS_OK) return st;
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(x && slot_of && xd);
  JANUS_CHECK_ALIGN(aligned(x, 16) && aligned(xd, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const unsigned grid = rows_grid(row_items(n_atoms, d / 4), 8);
  if (topk_weight)
    dispatch_kernel<true><<<grid, kThreads, 0, (cudaStream_t)stream>>>(
        (const float4*)x, n_atoms, d / 4, top_k, slot_of, topk_weight, (float4*)xd, debug_fault_word());
  else
    dispatch_kernel<false><<<grid, kThreads, 0, (cudaStream_t)stream>>>(
        (const float4*)x, n_atoms, d / 4, top_k, slot_of, nullptr, (float4*)xd, debug_fault_word());
  return launch_status();
}

extern "C" janus_status janus_combine(const float* yd, const int32_t* slot_of,
                                      const float* topk_weight, int64_t n_atoms, int32_t top_k,
                                      int32_t d, float* y, janus_stream_t stream) {
  janus_status st = check_rows(n_atoms, d, top_k);
  if (st != JANUS_OK) return st;
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(yd && slot_of && y);
  JANUS_CHECK_ALIGN(aligned(yd, 16) && aligned(y, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const unsigned grid = rows_grid(row_items(n_atoms, d / 4), 8);
  if (topk_weight)
    combine_kernel<true><<<grid, kThreads, 0, (cudaStream_t)stream>>>(
        (const float4*)yd, slot_of, topk_weight, n_atoms, top_k, d / 4, (float4*)y, debug_fault_word());
  else
    combine_kernel<false><<<grid, kThreads, 0, (cudaStream_t)stream>>>(
        (const float4*)yd, slot_of, nullptr, n_atoms, top_k, d / 4, (float4*)y, debug_fault_word());
  return launch_status();
}

extern "C" janus_status janus_dispatch_split_workspace_size(int64_t n_atoms, size_t* bytes) {
  JANUS_CHECK_ARG(bytes && n_atoms >= 0);
  *bytes = sizeof(WsHeader) + align_up(sizeof(uint32_t) * (size_t)(n_atoms > 0 ? n_atoms : 1), 256);
  return JANUS_OK;
}

extern "C" janus_status janus_dispatch_split(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                                             const int32_t* slot_of, const float* topk_weight, uint16_t* rows16,
                                             float* row_scale, void* workspace, size_t workspace_bytes,
                                             janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  janus_status st = check_rows(n_atoms, d, top_k);
  if (st != JANUS_OK) return st;
  size_t need = 0;
  st = janus_dispatch_split_workspace_size(n_atoms, &need);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(workspace && workspace_bytes >= need);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(x && slot_of && rows16 && row_scale);
  JANUS_CHECK_ALIGN(aligned(x, 16) && aligned(rows16, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  uint32_t* rowmax = (uint32_t*)((char*)workspace + sizeof(WsHeader));
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, need, stream));
  const unsigned grid = rows_grid(row_items(n_atoms, d / 4), 8);
  row_absmax_kernel<<<grid, kThreads, 0, stream>>>((const float4*)x, n_atoms, d / 4, rowmax);
  if (topk_weight)
    dispatch_split_kernel<true><<<grid, kThreads, 0, stream>>>((const float4*)x, n_atoms, d / 4, top_k, slot_of,
                                                               topk_weight, rowmax, (uint2*)rows16, row_scale,
                                                               debug_fault_word());
  else
    dispatch_split_kernel<false><<<grid, kThreads, 0, stream>>>((const float4*)x, n_atoms, d / 4, top_k, slot_of,
                                                                nullptr, rowmax, (uint2*)rows16, row_scale,
                                                                debug_fault_word());
  return launch_status();
}

extern "C" janus_status janus_quant_by_type_workspace_size(int32_t n_types, size_t* bytes) {
  JANUS_CHECK_ARG(bytes && n_types >= 1 && n_types <= kMaxTypes);
  *bytes = sizeof(WsHeader) + align_up(sizeof(uint32_t) * (size_t)n_types, 256);
  return JANUS_OK;
}

extern "C" janus_status janus_quant_by_type(const float* x, int64_t n_atoms, int32_t d,
                                            int32_t top_k, const int32_t* types, int32_t n_types,
                                            const int32_t* slot_of, uint16_t* payload,
                                            float* scale, void* workspace,
                                            size_t workspace_bytes, janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  janus_status st = check_rows(n_atoms, d, top_k);
  if (st != JANUS_OK) return st;
  size_t need = 0;
  st = janus_quant_by_type_workspace_size(n_types, &need);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(scale && workspace && workspace_bytes >= need);
  JANUS_CHECK_ARG(n_atoms == 0 || (x && types && slot_of && payload));
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  JANUS_CHECK_ALIGN(n_atoms == 0 || (aligned(x, 16) && aligned(payload, 8)));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  WsHeader* hdr = (WsHeader*)workspace;
  uint32_t* amax_bits = (uint32_t*)((char*)workspace + sizeof(WsHeader));
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, need, stream));
  const size_t smem = sizeof(uint32_t) * (size_t)n_types;
  const unsigned grid = rows_grid(row_items(n_atoms, d / 4), 8);
  if (n_atoms > 0)
    quant_amax_kernel<<<grid, kThreads, smem, stream>>>((const float4*)x, n_atoms, d / 4, types,
                                                        n_types, amax_bits, hdr);
  quant_pack_kernel<<<grid, kThreads, smem, stream>>>((const float4*)x, n_atoms, d / 4, top_k,
                                                      types, n_types, slot_of, amax_bits,
                                                      (uint2*)payload, scale, hdr);
  return launch_status();
}

extern "C" janus_status janus_dequant_by_type(const uint16_t* payload, int64_t n_atoms, int32_t d,
                                              int32_t top_k, const int32_t* types,
                                              int32_t n_types, const int32_t* perm,
                                              const float* scale, float* xd,
                                              janus_stream_t stream) {
  janus_status st = check_rows(n_atoms, d, top_k);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(n_types >= 1 && n_types <= kMaxTypes);
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(payload && types && perm && scale && xd);
  JANUS_CHECK_ALIGN(aligned(payload, 8) && aligned(xd, 16));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int64_t R = n_atoms * top_k;
  dequant_kernel<<<rows_grid(row_items(R, d / 4), 8), kThreads, 0, (cudaStream_t)stream>>>(
      (const uint2*)payload, R, d / 4, top_k, types, n_types, perm, scale, (float4*)xd, debug_fault_word());
  return launch_status();
}

extern "C" janus_status janus_dispatch_row_scales(int64_t n_atoms, int32_t top_k, const int32_t* types,
                                                  int32_t n_types, const int32_t* perm, const float* scale,
                                                  float* row_scale, janus_stream_t stream) {
  JANUS_CHECK_ARG(n_atoms >= 0 && top_k >= 1 && top_k <= kMaxExperts);
  JANUS_CHECK_ARG(n_atoms * (int64_t)top_k < (int64_t)INT32_MAX);
  JANUS_CHECK_ARG(n_types >= 1 && n_types <= kMaxTypes);
  if (n_atoms == 0) return JANUS_OK;
  JANUS_CHECK_ARG(types && perm && scale && row_scale);
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const int64_t R = n_atoms * top_k;
  const int64_t blocks = std::min<int64_t>((R + kThreads - 1) / kThreads, (int64_t)num_sms() * 8);
  row_scale_kernel<<<(unsigned)blocks, kThreads, 0, (cudaStream_t)stream>>>(R, top_k, types, n_types, perm, scale,
                                                                             row_scale, debug_fault_word());
  return launch_status();
}

// ---------------------------------------------------------------------------
// janus_quant_by_type_noalloc: per-type FP16 packing for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the
// point where they pack a dispatch buffer: code running under an allocator
// that forbids allocation during a step, plug-ins handed fixed buffers by a
// host framework, or host code that has already partitioned all device
// memory.  This entry point needs nothing from them beyond the inputs and
// outputs: its scratch (the error word and one absmax word per element type)
// is a file-scope device array owned by this library, 256 + 4 * 4096 =
// 16,640 bytes, which every GPU that loads the library keeps until the
// process exits.
// ---------------------------------------------------------------------------
#include <cuda.h>

#include <mutex>
#include <unordered_map>

constexpr int kNoAllocMaxTypes = 4096;
constexpr size_t kNoAllocScratchBytes = sizeof(janus::WsHeader) + sizeof(uint32_t) * kNoAllocMaxTypes;
static_assert(kNoAllocMaxTypes <= janus::kMaxTypes, "the scratch may not admit more types than the library");

// The scratch itself.  Host code must not use this name as an address (on the
// host it is only a stand-in); the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_quant_noalloc_scratch[kNoAllocScratchBytes];

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (CtxGetCurrentFn)p;
  });
  return fn;
}

std::mutex g_noalloc_mu;
std::unordered_map<CUcontext, void*> g_noalloc_addr;   // CUDA context -> scratch address

// Device address of the scratch in the current CUDA context, looked up once
// per context (cudaGetSymbolAddress may load the module into it).  Keying on
// the context, not the device ordinal, keeps a driver-API context from using
// the primary context's address.  A context destroyed and re-created at the
// same handle (cudaDeviceReset) is not detected.
janus_status noalloc_scratch(void** out) {
  CtxGetCurrentFn get = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (!get || get(&ctx) != CUDA_SUCCESS) return JANUS_ERR_CUDA;
  if (ctx == nullptr) {
    // no context is current yet: initialise the current device's primary
    // context (cudaSetDevice does so at once and allocates no memory)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return JANUS_ERR_CUDA;
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return JANUS_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  auto it = g_noalloc_addr.find(ctx);
  if (it != g_noalloc_addr.end()) {
    *out = it->second;
    return JANUS_OK;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_quant_noalloc_scratch) != cudaSuccess || p == nullptr)
    return JANUS_ERR_CUDA;
  g_noalloc_addr[ctx] = p;
  *out = p;
  return JANUS_OK;
}

}  // namespace

extern "C" janus_status janus_quant_by_type_noalloc(const float* x, int64_t n_atoms, int32_t d,
                                                    int32_t top_k, const int32_t* types,
                                                    int32_t n_types, const int32_t* slot_of,
                                                    uint16_t* payload, float* scale,
                                                    janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  janus_status st = check_rows(n_atoms, d, top_k);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(n_types >= 1 && n_types <= kNoAllocMaxTypes);
  JANUS_CHECK_ARG(scale != nullptr);
  JANUS_CHECK_ARG(n_atoms == 0 || (x && types && slot_of && payload));
  JANUS_CHECK_ALIGN(n_atoms == 0 || (aligned(x, 16) && aligned(payload, 8)));
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != JANUS_OK) return st;
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  WsHeader* hdr = (WsHeader*)scratch;
  uint32_t* amax_bits = (uint32_t*)((char*)scratch + sizeof(WsHeader));
  // the previous call's absmax words are still there: clear what this call uses
  JANUS_CUDA_TRY(cudaMemsetAsync(scratch, 0, sizeof(WsHeader) + sizeof(uint32_t) * (size_t)n_types, stream));
  const size_t smem = sizeof(uint32_t) * (size_t)n_types;
  const unsigned grid = rows_grid(row_items(n_atoms, d / 4), 8);
  if (n_atoms > 0)
    quant_amax_kernel<<<grid, kThreads, smem, stream>>>((const float4*)x, n_atoms, d / 4, types, n_types,
                                                        amax_bits, hdr);
  quant_pack_kernel<<<grid, kThreads, smem, stream>>>((const float4*)x, n_atoms, d / 4, top_k, types,
                                                      n_types, slot_of, amax_bits, (uint2*)payload, scale,
                                                      hdr);
  return launch_status();
}
