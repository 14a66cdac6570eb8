// janus_route: static per-element-type top-K routing, per-expert token counts
// and offsets, and the stable dispatch permutation.
//
// Source: paper review "Breaking the Training Barrier of Billion-Parameter
// Universal Machine Learning Interatomic Potentials" section 3.2 (each element
// type activates its own top-K experts); ScienceAI article (JIT planning:
// route before the step, count per-expert token load).
//
// Design (four launches, no host sync, no inter-CTA spin-wait):
//   1. route_table   one warp per element type: top-K of the gate row by K
//                    rounds of warp argmax, softmax weights in FP64.  The
//                    routing decision depends on the type only, so it is
//                    computed T times, not N times.
//   2. route_count   one CTA per chunk of atoms: expand the table to the
//                    atoms' K slots and histogram the chunk's slots per expert
//                    in shared memory -> blockcnt[e][b] (expert-major).
//   3. route_scan    one CTA per expert: exclusive scan of blockcnt[e][:]
//                    and counts[e]; the last CTA to finish (ticket counter,
//                    no waiting) scans counts into offsets.
//   4. route_scatter one CTA per chunk again: stable rank of every slot
//                    inside its expert (warp __match_any_sync + popc, then a
//                    cross-warp prefix in shared memory), position =
//                    offsets[e] + blockcnt-prefix[e][b] + rank.
#include "common.cuh"

namespace janus {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBlocks = 2048;       // route_scan handles up to 8 per thread

struct RouteLayout {
  int64_t atoms_per_block;
  int64_t n_blocks;
  size_t off_table_e, off_table_w, off_blockcnt, total;
};

RouteLayout route_layout(int64_t n_atoms, int32_t T, int32_t E, int32_t K) {
  RouteLayout L;
  int64_t apb = 64;
  if (n_atoms > apb * kMaxBlocks) apb = (n_atoms + kMaxBlocks - 1) / kMaxBlocks;
  L.atoms_per_block = apb;
  L.n_blocks = n_atoms > 0 ? (n_atoms + apb - 1) / apb : 0;
  size_t off = sizeof(WsHeader);
  L.off_table_e = off;
  off = align_up(off + sizeof(int32_t) * (size_t)T * K, 256);
  L.off_table_w = off;
  off = align_up(off + sizeof(float) * (size_t)T * K, 256);
  L.off_blockcnt = off;
  off = align_up(off + sizeof(int32_t) * (size_t)E * (L.n_blocks > 0 ? L.n_blocks : 1), 256);
  L.total = off;
  return L;
}

// true if (va, ia) ranks before (vb, ib): larger logit, ties to lower id
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(kThreads)
route_table(const float* __restrict__ gate, int32_t T, int32_t E, int32_t K,
            int32_t* __restrict__ table_e, float* __restrict__ table_w) {
  __shared__ float sel_logit[kWarps][kMaxExperts];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T) return;
  constexpr int kPer = kMaxExperts / 32;
  float v[kPer];
  uint32_t taken = 0;   // bit j: expert lane + 32 j already selected
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? gate[(int64_t)t * E + e] : 0.0f;
  }
  for (int k = 0; k < K; ++k) {
    // lane-local best among untaken experts
    float bv = 0.0f;
    int bi = INT32_MAX;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !(taken & (1u << j)) && (bi == INT32_MAX || ranks_before(v[j], e, bv, bi))) {
        bv = v[j];
        bi = e;
      }
    }
    // warp argmax
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != INT32_MAX && (bi == INT32_MAX || ranks_before(ov, oi, bv, bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi % 32 == lane) taken |= 1u << (bi / 32);
    if (lane == 0) {
      table_e[(int64_t)t * K + k] = bi;
      sel_logit[warp][k] = bv;
    }
  }
  __syncwarp();
  // softmax over the selected logits, shifted by the largest (FP64)
  const double l0 = (double)sel_logit[warp][0];
  double z = 0.0;
  for (int k = lane; k < K; k += 32) z += exp((double)sel_logit[warp][k] - l0);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  for (int k = lane; k < K; k += 32)
    table_w[(int64_t)t * K + k] = (float)(exp((double)sel_logit[warp][k] - l0) / z);
}

__global__ void __launch_bounds__(kThreads)
route_count(const int32_t* __restrict__ types, int64_t n_atoms, int32_t T, int32_t E, int32_t K,
            const int32_t* __restrict__ table_e, const float* __restrict__ table_w,
            int64_t atoms_per_block, int64_t n_blocks, int32_t* __restrict__ topk_e,
            float* __restrict__ topk_w, int32_t* __restrict__ blockcnt, WsHeader* ws) {
  __shared__ int32_t cnt[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += kThreads) cnt[e] = 0;
  __syncthreads();
  const int64_t a0 = (int64_t)blockIdx.x * atoms_per_block;
  const int64_t a1 = min(a0 + atoms_per_block, n_atoms);
  const int64_t s0 = a0 * K, s1 = a1 * K;
  for (int64_t s = s0 + threadIdx.x; s < s1; s += kThreads) {
    const int64_t i = s / K;
    const int k = (int)(s - i * K);
    int t = types[i];
    if (t < 0 || t >= T) {
      record_fault(ws, kFaultBadType);
      t = 0;
    }
    const int e = table_e[(int64_t)t * K + k];
    topk_e[s] = e;
    topk_w[s] = table_w[(int64_t)t * K + k];
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads) blockcnt[(int64_t)e * n_blocks + blockIdx.x] = cnt[e];
}

// block-wide exclusive scan of one int per thread; returns the prefix, *total = sum
__device__ __forceinline__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sum[kWarps];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int wpre = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int ws_ = warp_sum[w];
    if (w < warp) wpre += ws_;
    tot += ws_;
  }
  __syncthreads();
  *total = tot;
  return wpre + incl - v;
}

__global__ void __launch_bounds__(kThreads)
route_scan(int32_t E, int64_t n_blocks, int32_t* __restrict__ blockcnt,
           int32_t* __restrict__ counts, int32_t* __restrict__ offsets, WsHeader* ws) {
  __shared__ bool is_last;
  const int e = blockIdx.x;
  int32_t* col = blockcnt + (int64_t)e * n_blocks;
  const int per = (int)((n_blocks + kThreads - 1) / kThreads);   // <= 8
  const int64_t b0 = (int64_t)threadIdx.x * per;
  int loc[8];
  int sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    loc[j] = (j < per && b0 + j < n_blocks) ? col[b0 + j] : 0;
    sum += loc[j];
  }
  int total;
  int run = block_exclusive_scan(sum, &total);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < per && b0 + j < n_blocks) col[b0 + j] = run;
    run += loc[j];
  }
  if (threadIdx.x == 0) {
    counts[e] = total;
    __threadfence();
    is_last = (atomicAdd(&ws->done, 1u) == (unsigned)E - 1);
  }
  __syncthreads();
  if (!is_last) return;
  // last CTA: offsets = exclusive scan of counts (E <= 256, one per thread)
  __threadfence();
  const int c = threadIdx.x < E ? __ldcg(counts + threadIdx.x) : 0;
  int tot;
  const int pre = block_exclusive_scan(c, &tot);
  if (threadIdx.x < E) offsets[threadIdx.x] = pre;
  if (threadIdx.x == 0) {
    offsets[E] = tot;
    ws->done = 0;
  }
}

__global__ void __launch_bounds__(kThreads)
route_scatter(int64_t n_atoms, int32_t E, int32_t K, int64_t atoms_per_block, int64_t n_blocks,
              const int32_t* __restrict__ topk_e, const int32_t* __restrict__ blockcnt,
              const int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
              int32_t* __restrict__ slot_of) {
  __shared__ int32_t wcnt[kWarps][kMaxExperts];
  __shared__ int32_t base[kMaxExperts];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int e = threadIdx.x; e < E; e += kThreads) {
    base[e] = offsets[e] + blockcnt[(int64_t)e * n_blocks + blockIdx.x];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wcnt[w][e] = 0;
  }
  __syncthreads();
  const int64_t a0 = (int64_t)blockIdx.x * atoms_per_block;
  const int64_t a1 = min(a0 + atoms_per_block, n_atoms);
  const int64_t s0 = a0 * K, s1 = a1 * K;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int64_t c = s0; c < s1; c += kThreads) {
    const int64_t s = c + threadIdx.x;
    const int key = s < s1 ? topk_e[s] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, key);
    const int lrank = __popc(peers & lt_mask);
    if (key >= 0 && lrank == 0) wcnt[warp][key] = __popc(peers);
    __syncthreads();
    if (key >= 0) {
      int r = base[key] + lrank;
      for (int w = 0; w < warp; ++w) r += wcnt[w][key];
      perm[r] = (int32_t)s;
      slot_of[s] = r;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) {
      int tot = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        tot += wcnt[w][e];
        wcnt[w][e] = 0;
      }
      base[e] += tot;
    }
    __syncthreads();
  }
}

}  // namespace
}  // namespace janus

using namespace janus;

extern "C" janus_status janus_route_workspace_size(int64_t n_atoms, int32_t n_types,
                                                   int32_t n_experts, int32_t top_k,
                                                   size_t* bytes) {
  JANUS_CHECK_ARG(bytes != nullptr);
  JANUS_CHECK_ARG(n_atoms >= 0 && n_types >= 1 && n_types <= kMaxTypes);
  JANUS_CHECK_ARG(n_experts >= 1 && n_experts <= kMaxExperts && top_k >= 1 && top_k <= n_experts);
  JANUS_CHECK_ARG(n_atoms * (int64_t)top_k < (int64_t)INT32_MAX);
  *bytes = route_layout(n_atoms, n_types, n_experts, top_k).total;
  return JANUS_OK;
}

extern "C" janus_status janus_route(const int32_t* types, int64_t n_atoms, const float* gate,
                                    int32_t n_types, int32_t n_experts, int32_t top_k,
                                    int32_t* topk_expert, float* topk_weight, int32_t* counts,
                                    int32_t* offsets, int32_t* perm, int32_t* slot_of,
                                    void* workspace, size_t workspace_bytes,
                                    janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  size_t need = 0;
  janus_status st = janus_route_workspace_size(n_atoms, n_types, n_experts, top_k, &need);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(gate && counts && offsets && workspace);
  JANUS_CHECK_ARG(n_atoms == 0 || (types && topk_expert && topk_weight && perm && slot_of));
  JANUS_CHECK_ARG(workspace_bytes >= need);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;

  const int32_t T = n_types, E = n_experts, K = top_k;
  RouteLayout L = route_layout(n_atoms, T, E, K);
  char* w = (char*)workspace;
  WsHeader* hdr = (WsHeader*)w;
  int32_t* table_e = (int32_t*)(w + L.off_table_e);
  float* table_w = (float*)(w + L.off_table_w);
  int32_t* blockcnt = (int32_t*)(w + L.off_blockcnt);

  JANUS_CUDA_TRY(cudaMemsetAsync(hdr, 0, sizeof(WsHeader), stream));
  if (n_atoms == 0) {
    JANUS_CUDA_TRY(cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream));
    JANUS_CUDA_TRY(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream));
    return JANUS_OK;
  }
  route_table<<<(T + kWarps - 1) / kWarps, kThreads, 0, stream>>>(gate, T, E, K, table_e, table_w);
  route_count<<<(unsigned)L.n_blocks, kThreads, 0, stream>>>(
      types, n_atoms, T, E, K, table_e, table_w, L.atoms_per_block, L.n_blocks, topk_expert,
      topk_weight, blockcnt, hdr);
  route_scan<<<E, kThreads, 0, stream>>>(E, L.n_blocks, blockcnt, counts, offsets, hdr);
  route_scatter<<<(unsigned)L.n_blocks, kThreads, 0, stream>>>(
      n_atoms, E, K, L.atoms_per_block, L.n_blocks, topk_expert, blockcnt, offsets, perm, slot_of);
  return launch_status();
}
