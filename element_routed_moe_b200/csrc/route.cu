// janus_route: static per-element-type top-K routing, per-expert token counts
// and offsets, and the stable dispatch permutation.
//
// Source: paper review "Breaking the Training Barrier of Billion-Parameter
// Universal Machine Learning Interatomic Potentials" section 3.2 (each element
// type activates its own top-K experts); ScienceAI article (JIT planning:
// route before the step, count per-expert token load).
//
// janus_route_layers routes several MoE layers' gate tables for the same atoms
// in the same four launches (grid dimension y = layer), as JIT planning does
// for all layers of a step before it runs.
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

// Workspace: header | per-layer ticket counters [nl] | per-type tables
// [nl][T][K] (experts, weights) | per-block expert counts [nl][E][n_blocks].
struct RouteLayout {
  int64_t atoms_per_block;
  int64_t n_blocks;
  size_t off_done, off_table_e, off_table_w, off_blockcnt, total;
};

RouteLayout route_layout(int64_t n_atoms, int32_t T, int32_t E, int32_t K, int32_t nl) {
  RouteLayout L;
  int64_t apb = 64;
  if (n_atoms > apb * kMaxBlocks) apb = (n_atoms + kMaxBlocks - 1) / kMaxBlocks;
  L.atoms_per_block = apb;
  L.n_blocks = n_atoms > 0 ? (n_atoms + apb - 1) / apb : 0;
  size_t off = sizeof(WsHeader);
  L.off_done = off;
  off = align_up(off + sizeof(uint32_t) * (size_t)nl, 256);
  L.off_table_e = off;
  off = align_up(off + sizeof(int32_t) * (size_t)nl * T * K, 256);
  L.off_table_w = off;
  off = align_up(off + sizeof(float) * (size_t)nl * T * K, 256);
  L.off_blockcnt = off;
  off = align_up(off + sizeof(int32_t) * (size_t)nl * E * (L.n_blocks > 0 ? L.n_blocks : 1), 256);
  L.total = off;
  return L;
}

// true if (va, ia) ranks before (vb, ib): larger logit, ties to lower id
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// A gate row with a non-finite logit (NaN or +-inf) has no well-defined top-K
// and softmax: route_table records kFaultNonFinite for it (the selection it
// makes is still a valid set of K distinct experts).
__global__ void __launch_bounds__(kThreads)
route_table(const float* __restrict__ gate, int32_t T, int32_t E, int32_t K,
            int32_t* __restrict__ table_e, float* __restrict__ table_w, WsHeader* ws) {
  __shared__ float sel_logit[kWarps][kMaxExperts];
  // layer blockIdx.y: gate [T,E] and tables [T,K] of that layer
  gate += (int64_t)blockIdx.y * T * E;
  table_e += (int64_t)blockIdx.y * T * K;
  table_w += (int64_t)blockIdx.y * T * K;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T) return;
  constexpr int kPer = kMaxExperts / 32;
  float v[kPer];
  uint32_t taken = 0;   // bit j: expert lane + 32 j already selected
  bool finite = true;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? gate[(int64_t)t * E + e] : 0.0f;
    finite = finite && isfinite(v[j]);
  }
  if (!__all_sync(0xffffffffu, finite) && lane == 0) record_fault(ws, kFaultNonFinite);
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
  {  // layer blockIdx.y (types are shared by all layers)
    const int64_t l = blockIdx.y;
    table_e += l * T * K;
    table_w += l * T * K;
    topk_e += l * n_atoms * K;
    topk_w += l * n_atoms * K;
    blockcnt += l * E * n_blocks;
  }
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
           int32_t* __restrict__ counts, int32_t* __restrict__ offsets, uint32_t* done) {
  __shared__ bool is_last;
  {  // layer blockIdx.y
    const int64_t l = blockIdx.y;
    blockcnt += l * E * n_blocks;
    counts += l * E;
    offsets += l * (E + 1);
    done += l;
  }
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
    is_last = (atomicAdd(done, 1u) == (unsigned)E - 1);
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
    *done = 0;
  }
}

__global__ void __launch_bounds__(kThreads)
route_scatter(int64_t n_atoms, int32_t E, int32_t K, int64_t atoms_per_block, int64_t n_blocks,
              const int32_t* __restrict__ topk_e, const int32_t* __restrict__ blockcnt,
              const int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
              int32_t* __restrict__ slot_of) {
  __shared__ int32_t wcnt[kWarps][kMaxExperts];
  __shared__ int32_t base[kMaxExperts];
  {  // layer blockIdx.y
    const int64_t l = blockIdx.y, R = n_atoms * K;
    topk_e += l * R;
    blockcnt += l * E * n_blocks;
    offsets += l * (E + 1);
    perm += l * R;
    slot_of += l * R;
  }
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

static janus_status route_check(int64_t n_atoms, int32_t n_types, int32_t n_experts, int32_t top_k,
                                int32_t n_layers) {
  JANUS_CHECK_ARG(n_atoms >= 0 && n_types >= 1 && n_types <= kMaxTypes);
  JANUS_CHECK_ARG(n_experts >= 1 && n_experts <= kMaxExperts && top_k >= 1 && top_k <= n_experts);
  JANUS_CHECK_ARG(n_atoms * (int64_t)top_k < (int64_t)INT32_MAX);
  JANUS_CHECK_ARG(n_layers >= 1 && n_layers <= 65535);
  return JANUS_OK;
}

// Routes n_layers gate tables [nl][T][E] for the same atoms in one set of four
// launches (grid dimension y = layer); outputs are stacked per layer.
static janus_status route_impl(const int32_t* types, int64_t n_atoms, const float* gates, int32_t nl,
                               int32_t T, int32_t E, int32_t K, int32_t* topk_expert, float* topk_weight,
                               int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* slot_of,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  janus_status st = route_check(n_atoms, T, E, K, nl);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(gates && counts && offsets && workspace);
  JANUS_CHECK_ARG(n_atoms == 0 || (types && topk_expert && topk_weight && perm && slot_of));
  const RouteLayout L = route_layout(n_atoms, T, E, K, nl);
  JANUS_CHECK_ARG(workspace_bytes >= L.total);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;

  char* w = (char*)workspace;
  WsHeader* hdr = (WsHeader*)w;
  uint32_t* done = (uint32_t*)(w + L.off_done);
  int32_t* table_e = (int32_t*)(w + L.off_table_e);
  float* table_w = (float*)(w + L.off_table_w);
  int32_t* blockcnt = (int32_t*)(w + L.off_blockcnt);

  JANUS_CUDA_TRY(cudaMemsetAsync(hdr, 0, L.off_table_e, stream));   // header + ticket counters
  if (n_atoms == 0) {
    JANUS_CUDA_TRY(cudaMemsetAsync(counts, 0, sizeof(int32_t) * E * nl, stream));
    JANUS_CUDA_TRY(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1) * nl, stream));
    return JANUS_OK;
  }
  const unsigned nb = (unsigned)L.n_blocks, ly = (unsigned)nl;
  route_table<<<dim3((T + kWarps - 1) / kWarps, ly), kThreads, 0, stream>>>(gates, T, E, K, table_e, table_w,
                                                                            hdr);
  route_count<<<dim3(nb, ly), kThreads, 0, stream>>>(types, n_atoms, T, E, K, table_e, table_w,
                                                      L.atoms_per_block, L.n_blocks, topk_expert,
                                                      topk_weight, blockcnt, hdr);
  route_scan<<<dim3(E, ly), kThreads, 0, stream>>>(E, L.n_blocks, blockcnt, counts, offsets, done);
  route_scatter<<<dim3(nb, ly), kThreads, 0, stream>>>(n_atoms, E, K, L.atoms_per_block, L.n_blocks,
                                                        topk_expert, blockcnt, offsets, perm, slot_of);
  return launch_status();
}

extern "C" janus_status janus_route_workspace_size(int64_t n_atoms, int32_t n_types,
                                                   int32_t n_experts, int32_t top_k,
                                                   size_t* bytes) {
  JANUS_CHECK_ARG(bytes != nullptr);
  janus_status st = route_check(n_atoms, n_types, n_experts, top_k, 1);
  if (st != JANUS_OK) return st;
  *bytes = route_layout(n_atoms, n_types, n_experts, top_k, 1).total;
  return JANUS_OK;
}

extern "C" janus_status janus_route(const int32_t* types, int64_t n_atoms, const float* gate,
                                    int32_t n_types, int32_t n_experts, int32_t top_k,
                                    int32_t* topk_expert, float* topk_weight, int32_t* counts,
                                    int32_t* offsets, int32_t* perm, int32_t* slot_of,
                                    void* workspace, size_t workspace_bytes,
                                    janus_stream_t stream) {
  return route_impl(types, n_atoms, gate, 1, n_types, n_experts, top_k, topk_expert, topk_weight,
                    counts, offsets, perm, slot_of, workspace, workspace_bytes, (cudaStream_t)stream);
}

extern "C" janus_status janus_route_layers_workspace_size(int64_t n_atoms, int32_t n_types,
                                                          int32_t n_experts, int32_t top_k,
                                                          int32_t n_layers, size_t* bytes) {
  JANUS_CHECK_ARG(bytes != nullptr);
  janus_status st = route_check(n_atoms, n_types, n_experts, top_k, n_layers);
  if (st != JANUS_OK) return st;
  *bytes = route_layout(n_atoms, n_types, n_experts, top_k, n_layers).total;
  return JANUS_OK;
}

extern "C" janus_status janus_route_layers(const int32_t* types, int64_t n_atoms, const float* gates,
                                           int32_t n_layers, int32_t n_types, int32_t n_experts,
                                           int32_t top_k, int32_t* topk_expert, float* topk_weight,
                                           int32_t* counts, int32_t* offsets, int32_t* perm,
                                           int32_t* slot_of, void* workspace, size_t workspace_bytes,
                                           janus_stream_t stream) {
  return route_impl(types, n_atoms, gates, n_layers, n_types, n_experts, top_k, topk_expert, topk_weight,
                    counts, offsets, perm, slot_of, workspace, workspace_bytes, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// Active-expert lists: per layer, the ids of the experts with routed rows, in
// ascending order (a stable compaction of counts > 0).  One CTA per layer,
// one thread per expert; the rank of each active expert is its warp's ballot
// prefix plus the active experts of the warps before it.
// ---------------------------------------------------------------------------
namespace janus {
namespace {
__global__ void __launch_bounds__(kMaxExperts) active_experts_kernel(const int32_t* __restrict__ counts, int E,
                                                                    int32_t* __restrict__ active,
                                                                    int32_t* __restrict__ n_active) {
  __shared__ int warp_sum[kMaxExperts / 32];
  const int l = blockIdx.x, e = threadIdx.x, lane = e % 32, w = e / 32;
  const bool on = e < E && counts[(int64_t)l * E + e] > 0;
  const unsigned bal = __ballot_sync(0xffffffffu, on);
  if (lane == 0) warp_sum[w] = __popc(bal);
  __syncthreads();
  int base = 0;
  for (int i = 0; i < w; ++i) base += warp_sum[i];
  if (on) active[(int64_t)l * E + base + __popc(bal & ((1u << lane) - 1u))] = e;
  if (e == 0) {
    int tot = 0;
    for (int i = 0; i < kMaxExperts / 32; ++i) tot += warp_sum[i];
    n_active[l] = tot;
  }
}
}  // namespace
}  // namespace janus

extern "C" janus_status janus_active_experts(const int32_t* counts, int32_t n_layers, int32_t n_experts,
                                             int32_t* active, int32_t* n_active, janus_stream_t stream) {
  using namespace janus;
  JANUS_CHECK_ARG(n_layers >= 0 && n_experts >= 1 && n_experts <= kMaxExperts);
  if (n_layers == 0) return JANUS_OK;
  JANUS_CHECK_ARG(counts && active && n_active);
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  active_experts_kernel<<<n_layers, kMaxExperts, 0, (cudaStream_t)stream>>>(counts, n_experts, active, n_active);
  return launch_status();
}
