// janus_expert_ffn_fwd / janus_expert_ffn_vjp: the grouped expert MLP of the
// element-routed MoE layer and its input VJP.
//
// Sources: paper review "Breaking the Training Barrier of Billion-Parameter
// Universal Machine Learning Interatomic Potentials" section 3.1 Table II
// (MLP hidden size = feature size) and section 3.3 (forces and stress by
// autodiff of the energy, so training needs the input gradient).  The expert
// is read as bias-free Linear(d,h) -> SiLU -> Linear(h,d).
//
// Forward (two grouped GEMMs, SiLU fused into the first one's epilogue):
//   G1: a = xd W1[e]          -> act (optional), H = silu(a) (workspace)
//   G2: yd = H W2[e]
// Input VJP (SiLU' fused into the first GEMM's epilogue):
//   G0: a = xd W1[e]          (only when the forward's act is not supplied)
//   G3: dA = (gd W2[e]^T) * silu'(a)   (workspace)
//   G4: dxd = dA W1[e]^T
// Weight gradients (G3 also writes H = silu(a)):
//   G5: dW1[e] = Xd_e^T dA_e,  G6: dW2[e] = H_e^T Gd_e  (sums over expert e's rows)
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "ffn_simt.cuh"
#include "ffn_tc.cuh"

namespace janus {
namespace {

struct FfnLayout {
  size_t off_h, total;
};

FfnLayout ffn_layout(int64_t R, int32_t h, bool vjp, bool have_act) {
  FfnLayout L;
  const size_t rh = align_up(sizeof(float) * (size_t)R * (size_t)h, 256);
  L.off_h = sizeof(WsHeader);
  size_t n_bufs = vjp ? (have_act ? 1 : 2) : 1;
  L.total = L.off_h + n_bufs * rh + tc::workspace_extra();
  return L;
}

janus_status check_ffn(const float* xd, const int32_t* offsets, int32_t E, int64_t R, int32_t d,
                       int32_t h, const float* w1, const float* w2, const float* out,
                       janus_ffn_mode mode) {
  JANUS_CHECK_ARG(E >= 1 && E <= kMaxExperts);
  JANUS_CHECK_ARG(R >= 0 && R < (int64_t)INT32_MAX);
  JANUS_CHECK_ARG(d >= 1 && d <= kMaxDim && h >= 1 && h <= kMaxDim);
  JANUS_CHECK_ARG(mode == JANUS_FFN_FP32_SIMT || mode == JANUS_FFN_3XTF32);
  JANUS_CHECK_ALIGN(d % 4 == 0 && h % 4 == 0);
  JANUS_CHECK_ARG(offsets && w1 && w2);
  JANUS_CHECK_ARG(R == 0 || (xd && out));
  JANUS_CHECK_ALIGN(aligned(w1, 16) && aligned(w2, 16));
  JANUS_CHECK_ALIGN(R == 0 || (aligned(xd, 16) && aligned(out, 16)));
  return JANUS_OK;
}

template <bool kNT, int kEpi>
void launch_simt(const simt::Args& a, cudaStream_t s) {
  simt::grouped_gemm_kernel<kNT, kEpi><<<num_sms() * 2, simt::kThreads, 0, s>>>(a);
}

simt::Args make_args(const float* A, const float* B, int64_t bstride, float* C, float* C2,
                     const float* aux, const int32_t* offsets, int E, int Kd, int N, int64_t rows) {
  simt::Args a;
  a.A = A; a.B = B; a.b_expert_stride = bstride; a.C = C; a.C2 = C2; a.aux = aux;
  a.aux2 = nullptr; a.C3 = nullptr; a.c_rows = nullptr;
  a.offsets = offsets; a.E = E; a.Kd = Kd; a.N = N;
  a.rows = rows; a.dbg = debug_fault_word();
  return a;
}

// xd[p,:] = f32(payload[p,:]) * row_scale[p]: one warp per row, four values
// (8 bytes in, 16 out) per lane and step.  The SIMT path of the packed forward.
__global__ void __launch_bounds__(256)
unpack_rows_kernel(const uint2* __restrict__ payload, const float* __restrict__ row_scale, int64_t R, int d4,
                   float4* __restrict__ xd) {
  const int lane = threadIdx.x % 32;
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t p = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; p < R; p += nw) {
    const float sc = __ldg(row_scale + p);
    for (int c = lane; c < d4; c += 32) {
      const uint2 q = __ldcs(payload + p * d4 + c);
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&q.x));
      const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&q.y));
      xd[p * d4 + c] = make_float4(a.x * sc, a.y * sc, b.x * sc, b.y * sc);
    }
  }
}

// The MLP's second GEMM (H W2 in the forward, dA W1^T in the split VJP)
// runs on the kind::f16 path too when the layer has at least this many
// routed rows per expert: the activation's row split and the per-call split
// of the weights then cost less than the GEMMs save (measured break-even near
// 380 rows per expert; the S-shaped layer, 455, gains 8 %).
constexpr int64_t kF16SecondMinRowsPerExpert = 384;
bool use_f16_second(int64_t R, int32_t E, int32_t h) {
  return h % 8 == 0 && R >= kF16SecondMinRowsPerExpert * E;
}

// 1 / S of a weight split: per output feature (N) and K chunk of 256.
size_t winv_bytes(int32_t E, int32_t Kd, int32_t N) {
  return align_up(sizeof(float) * (size_t)E * (size_t)((Kd + 255) / 256) * (size_t)N, 256);
}

// Scratch of the FP16 second GEMM (see tc::F16Second), starting at `base`.
size_t f16_second_bytes(int64_t R, int32_t E, int32_t d, int32_t h) {
  return align_up(2 * sizeof(uint16_t) * (size_t)R * h, 256) + align_up(sizeof(float) * (size_t)R, 256) +
         align_up(2 * sizeof(uint16_t) * (size_t)E * d * h, 256) + winv_bytes(E, h, d);
}
tc::F16Second f16_second_at(char* base, int64_t R, int32_t E, int32_t d, int32_t h) {
  tc::F16Second f;
  f.h16 = (uint16_t*)base;
  base += align_up(2 * sizeof(uint16_t) * (size_t)R * h, 256);
  f.hscale = (float*)base;
  base += align_up(sizeof(float) * (size_t)R, 256);
  f.w16 = (uint16_t*)base;
  base += align_up(2 * sizeof(uint16_t) * (size_t)E * d * h, 256);
  f.winv = (float*)base;
  return f;
}

// Past the forward's activations: SIMT, the unpacked rows [R,d] FP32;
// 3xTF32, the FP16 split of W1 (hi and mid, [E][h][d] each), 1 / S [E][ceil(d/256)][h],
// and the FP16 second GEMM's scratch when it is used (the weight splits in
// it stay unused when the call is given a weight-split set).
size_t packed_extra(int64_t R, int32_t E, int32_t d, int32_t h, janus_ffn_mode mode) {
  if (mode == JANUS_FFN_FP32_SIMT) return align_up(sizeof(float) * (size_t)R * (size_t)d, 256);
  return align_up(2 * sizeof(uint16_t) * (size_t)E * d * h, 256) + winv_bytes(E, d, h) +
         (use_f16_second(R, E, h) ? f16_second_bytes(R, E, d, h) : 0);
}

// The weight splits of a layer written ahead of its MLP calls
// (janus_expert_weights_f16): four parts, each the planes [2][E][N][Kd]
// FP16 then 1 / S [E][ceil(Kd/256)][N]:
//   0  W1 for x W1     (Kd = d, N = h)   forward, first GEMM
//   1  W2 for H W2     (Kd = h, N = d)   forward, second GEMM
//   2  W2 for gd W2^T  (Kd = d, N = h)   input VJP, first GEMM
//   3  W1 for dA W1^T  (Kd = h, N = d)   input VJP, second GEMM
struct W16Set {
  size_t off_w16[4], off_winv[4], total;
};
W16Set w16_set_layout(int32_t E, int32_t d, int32_t h) {
  W16Set S;
  const int32_t kd[4] = {d, h, d, h}, nn[4] = {h, d, h, d};
  size_t off = 0;
  for (int i = 0; i < 4; ++i) {
    S.off_w16[i] = off;
    off += align_up(2 * sizeof(uint16_t) * (size_t)E * d * h, 256);
    S.off_winv[i] = off;
    off += winv_bytes(E, kd[i], nn[i]);
  }
  S.total = off;
  return S;
}
// The pointers of part `i` (first GEMM) and `i + 1` (second GEMM).
void w16_set_parts(const void* set, int32_t E, int32_t d, int32_t h, int i, uint16_t** w16, float** winv,
                   tc::F16Second* second) {
  const W16Set S = w16_set_layout(E, d, h);
  char* b = (char*)set;
  *w16 = (uint16_t*)(b + S.off_w16[i]);
  *winv = (float*)(b + S.off_winv[i]);
  second->w16 = (uint16_t*)(b + S.off_w16[i + 1]);
  second->winv = (float*)(b + S.off_winv[i + 1]);
}
janus_status check_w16_set(const void* set, size_t bytes, int32_t E, int32_t d, int32_t h) {
  if (!set) return JANUS_OK;
  JANUS_CHECK_ALIGN(aligned(set, 256));
  JANUS_CHECK_ARG(bytes >= w16_set_layout(E, d, h).total);
  return JANUS_OK;
}

}  // namespace
}  // namespace janus

using namespace janus;

extern "C" int32_t janus_expert_ffn_f16_min_rows_per_expert(void) { return (int32_t)kF16SecondMinRowsPerExpert; }

extern "C" janus_status janus_expert_weights_f16_size(int32_t n_experts, int32_t d, int32_t h, size_t* bytes) {
  JANUS_CHECK_ARG(bytes && n_experts >= 1 && n_experts <= kMaxExperts);
  JANUS_CHECK_ARG(d >= 1 && d <= kMaxDim && h >= 1 && h <= kMaxDim);
  *bytes = w16_set_layout(n_experts, d, h).total;
  return JANUS_OK;
}

extern "C" janus_status janus_expert_weights_f16(const float* w1, const float* w2, int32_t n_experts, int32_t d,
                                                 int32_t h, uint32_t which, void* out, size_t out_bytes,
                                                 janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  JANUS_CHECK_ARG(n_experts >= 1 && n_experts <= kMaxExperts);
  JANUS_CHECK_ARG(d >= 1 && d <= kMaxDim && h >= 1 && h <= kMaxDim);
  JANUS_CHECK_ARG(which >= 1 && which <= (JANUS_W16_FWD | JANUS_W16_VJP));
  JANUS_CHECK_ALIGN(d % 8 == 0 && h % 4 == 0);
  JANUS_CHECK_ARG(w1 && w2 && out);
  JANUS_CHECK_ALIGN(aligned(w1, 16) && aligned(w2, 16) && aligned(out, 256));
  const W16Set S = w16_set_layout(n_experts, d, h);
  JANUS_CHECK_ARG(out_bytes >= S.total);
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  char* b = (char*)out;
  auto w16 = [&](int i) { return (uint16_t*)(b + S.off_w16[i]); };
  auto winv = [&](int i) { return (float*)(b + S.off_winv[i]); };
  janus_status st = JANUS_OK;
  if (which == (JANUS_W16_FWD | JANUS_W16_VJP)) {
    // W1 [E][d][h]: x W1's split (part 0) and dA W1^T's (part 3); W2 [E][h][d]:
    // H W2's (part 1) and gd W2^T's (part 2), each weight read once
    st = tc::split_weights_f16_both(w1, n_experts, d, h, w16(0), winv(0), w16(3), winv(3), stream);
    if (st == JANUS_OK)
      st = tc::split_weights_f16_both(w2, n_experts, h, d, w16(1), winv(1), w16(2), winv(2), stream);
    return st != JANUS_OK ? st : launch_status();
  }
  if (which & JANUS_W16_FWD) {
    st = tc::split_weights_f16(w1, n_experts, d, h, true, w16(0), winv(0), stream);
    if (st == JANUS_OK) st = tc::split_weights_f16(w2, n_experts, h, d, true, w16(1), winv(1), stream);
  } else {
    st = tc::split_weights_f16(w2, n_experts, d, h, false, w16(2), winv(2), stream);
    if (st == JANUS_OK) st = tc::split_weights_f16(w1, n_experts, h, d, false, w16(3), winv(3), stream);
  }
  return st != JANUS_OK ? st : launch_status();
}

extern "C" janus_status janus_expert_ffn_packed_workspace_size(int64_t n_rows, int32_t n_experts, int32_t d,
                                                               int32_t h, janus_ffn_mode mode, size_t* bytes) {
  JANUS_CHECK_ARG(bytes && n_rows >= 0 && d >= 1 && h >= 1 && n_experts >= 1 && n_experts <= kMaxExperts);
  JANUS_CHECK_ARG(mode == JANUS_FFN_FP32_SIMT || mode == JANUS_FFN_3XTF32);
  *bytes = ffn_layout(n_rows, h, false, true).total + packed_extra(n_rows, n_experts, d, h, mode);
  return JANUS_OK;
}

extern "C" janus_status janus_expert_ffn_fwd_packed(const uint16_t* payload, const float* row_scale,
                                                    const int32_t* offsets, int32_t n_experts, int64_t n_rows,
                                                    int32_t d, int32_t h, const float* w1, const float* w2,
                                                    float* yd, float* const* yd_rows, float* act,
                                                    const void* weights16, size_t weights16_bytes,
                                                    janus_ffn_mode mode, void* workspace, size_t workspace_bytes,
                                                    janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  JANUS_CHECK_ARG((yd == nullptr) != (yd_rows == nullptr) || n_rows == 0);
  const float* outp = yd_rows ? reinterpret_cast<const float*>(yd_rows) : yd;
  // check_ffn validates the shapes, weights and output; the payload is checked here
  janus_status st = check_ffn(reinterpret_cast<const float*>(payload), offsets, n_experts, n_rows, d, h, w1, w2,
                              outp, mode);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(n_rows == 0 || row_scale);
  JANUS_CHECK_ALIGN(mode != JANUS_FFN_3XTF32 || d % 8 == 0);   // FP16 rows: 16-byte TMA strides
  JANUS_CHECK_ALIGN(act == nullptr || aligned(act, 16));
  JANUS_CHECK_ARG(weights16 == nullptr || mode == JANUS_FFN_3XTF32);
  st = check_w16_set(weights16, weights16_bytes, n_experts, d, h);
  if (st != JANUS_OK) return st;
  const FfnLayout L = ffn_layout(n_rows, h, false, true);
  const size_t extra = packed_extra(n_rows, n_experts, d, h, mode);
  JANUS_CHECK_ARG(workspace && workspace_bytes >= L.total + extra);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  if (n_rows == 0) return JANUS_OK;
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  float* H = (float*)((char*)workspace + L.off_h);
  // the error word starts clear in both modes, so janus_check on this
  // workspace reports only this call's faults
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream));
  if (mode == JANUS_FFN_3XTF32) {
    uint16_t* w16 = (uint16_t*)((char*)workspace + L.total);
    const size_t w16_bytes = align_up(2 * sizeof(uint16_t) * (size_t)n_experts * d * h, 256);
    float* winv = (float*)((char*)workspace + L.total + w16_bytes);
    char* second_base = (char*)workspace + L.total + w16_bytes + winv_bytes(n_experts, d, h);
    tc::F16Second second = f16_second_at(second_base, n_rows, n_experts, d, h);
    if (weights16) w16_set_parts(weights16, n_experts, d, h, 0, &w16, &winv, &second);
    st = tc::expert_ffn_fwd_packed(payload, row_scale, offsets, n_experts, n_rows, d, h, w1, w2, yd, act, H, w16,
                                   winv, &((WsHeader*)workspace)->error, stream, yd_rows,
                                   use_f16_second(n_rows, n_experts, h) ? &second : nullptr, weights16 != nullptr);
    if (st != JANUS_OK) return st;
    return launch_status();
  }
  // FP32 SIMT: unpack into the workspace, then the plain forward
  float* xd = (float*)((char*)workspace + L.total);
  const int64_t blocks = std::min<int64_t>((n_rows + 7) / 8, (int64_t)num_sms() * 8);
  unpack_rows_kernel<<<(unsigned)blocks, 256, 0, stream>>>((const uint2*)payload, row_scale, n_rows, d / 4,
                                                         (float4*)xd);
  const int64_t sw = (int64_t)d * h;
  launch_simt<false, simt::kEpiSilu>(make_args(xd, w1, sw, H, act, nullptr, offsets, n_experts, d, h, n_rows), stream);
  simt::Args a2 = make_args(H, w2, sw, yd, nullptr, nullptr, offsets, n_experts, h, d, n_rows);
  a2.c_rows = yd_rows;
  launch_simt<false, simt::kEpiStore>(a2, stream);
  return launch_status();
}

// ---------------------------------------------------------------------------
// The expert MLP on rows given as two FP16 terms with a per-row scale
// (janus_dispatch_split): the first GEMM of the forward (x W1) or of the VJP
// (gd W2^T) on the kind::f16 tensor path; the second on 3xTF32, or on the
// kind::f16 path from kF16SecondMinRowsPerExpert rows per expert with h % 8 == 0.  Workspace:
// header | H, dH or dA [R,h] | the FP16 split of the first GEMM's weights
// (hi and mid, [E][h][d] each) | 1 / S [E][ceil(d/256)][h] | the FP16 second GEMM's
// scratch when it is used.  With a weight-split set the weight parts of this
// layout are not written; the GEMMs read the set's.
// ---------------------------------------------------------------------------
namespace {
struct SplitLayout {
  size_t off_h, off_w16, off_winv, off_second, total;
};
SplitLayout split_layout(int64_t R, int32_t E, int32_t d, int32_t h) {
  SplitLayout L;
  L.off_h = sizeof(WsHeader);
  L.off_w16 = L.off_h + align_up(sizeof(float) * (size_t)R * (size_t)h, 256);
  L.off_winv = L.off_w16 + align_up(2 * sizeof(uint16_t) * (size_t)E * d * h, 256);
  L.off_second = L.off_winv + winv_bytes(E, d, h);
  L.total = L.off_second + (use_f16_second(R, E, h) ? f16_second_bytes(R, E, d, h) : 0);
  return L;
}

janus_status check_split(const uint16_t* rows16, const float* row_scale, const int32_t* offsets, int32_t E,
                         int64_t R, int32_t d, int32_t h, const float* w1, const float* w2, const void* out,
                         void* workspace, size_t workspace_bytes) {
  JANUS_CHECK_ARG(E >= 1 && E <= kMaxExperts);
  JANUS_CHECK_ARG(R >= 0 && R < (int64_t)INT32_MAX / 2);
  JANUS_CHECK_ARG(d >= 1 && d <= kMaxDim && h >= 1 && h <= kMaxDim);
  JANUS_CHECK_ALIGN(d % 8 == 0 && h % 4 == 0);
  JANUS_CHECK_ARG(offsets && w1 && w2);
  JANUS_CHECK_ARG(R == 0 || (rows16 && row_scale && out));
  JANUS_CHECK_ALIGN(aligned(w1, 16) && aligned(w2, 16));
  JANUS_CHECK_ALIGN(R == 0 || (aligned(rows16, 16) && aligned(out, 16)));
  JANUS_CHECK_ARG(workspace && workspace_bytes >= split_layout(R, E, d, h).total);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  return JANUS_OK;
}
}  // namespace

extern "C" janus_status janus_expert_ffn_split_workspace_size(int64_t n_rows, int32_t n_experts, int32_t d,
                                                              int32_t h, size_t* bytes) {
  JANUS_CHECK_ARG(bytes && n_rows >= 0 && d >= 1 && h >= 1 && n_experts >= 1 && n_experts <= kMaxExperts);
  *bytes = split_layout(n_rows, n_experts, d, h).total;
  return JANUS_OK;
}

extern "C" janus_status janus_expert_ffn_fwd_split(const uint16_t* rows16, const float* row_scale,
                                                   const int32_t* offsets, int32_t n_experts, int64_t n_rows,
                                                   int32_t d, int32_t h, const float* w1, const float* w2,
                                                   float* yd, float* const* yd_rows, float* act,
                                                   const void* weights16, size_t weights16_bytes, void* workspace,
                                                   size_t workspace_bytes, janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  JANUS_CHECK_ARG((yd == nullptr) != (yd_rows == nullptr) || n_rows == 0);
  const void* outp = yd_rows ? (const void*)yd_rows : (const void*)yd;
  janus_status st = check_split(rows16, row_scale, offsets, n_experts, n_rows, d, h, w1, w2, outp, workspace,
                                workspace_bytes);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ALIGN(act == nullptr || aligned(act, 16));
  st = check_w16_set(weights16, weights16_bytes, n_experts, d, h);
  if (st != JANUS_OK) return st;
  if (n_rows == 0) return JANUS_OK;
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const SplitLayout L = split_layout(n_rows, n_experts, d, h);
  char* w = (char*)workspace;
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream));
  tc::F16Second second = f16_second_at(w + L.off_second, n_rows, n_experts, d, h);
  uint16_t* w16 = (uint16_t*)(w + L.off_w16);
  float* winv = (float*)(w + L.off_winv);
  if (weights16) w16_set_parts(weights16, n_experts, d, h, 0, &w16, &winv, &second);
  st = tc::expert_ffn_fwd_split(rows16, row_scale, offsets, n_experts, n_rows, d, h, w1, w2, yd, act,
                                (float*)(w + L.off_h), w16, winv, &((WsHeader*)workspace)->error, stream, yd_rows,
                                use_f16_second(n_rows, n_experts, h) ? &second : nullptr, weights16 != nullptr);
  if (st != JANUS_OK) return st;
  return launch_status();
}

extern "C" janus_status janus_expert_ffn_vjp_split(const uint16_t* gd16, const float* gd_scale, const float* act,
                                                   const int32_t* offsets, int32_t n_experts, int64_t n_rows,
                                                   int32_t d, int32_t h, const float* w1, const float* w2,
                                                   float* dxd, float* const* dxd_rows, const void* weights16,
                                                   size_t weights16_bytes, void* workspace,
                                                   size_t workspace_bytes, janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  JANUS_CHECK_ARG((dxd == nullptr) != (dxd_rows == nullptr) || n_rows == 0);
  const void* outp = dxd_rows ? (const void*)dxd_rows : (const void*)dxd;
  janus_status st = check_split(gd16, gd_scale, offsets, n_experts, n_rows, d, h, w1, w2, outp, workspace,
                                workspace_bytes);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(n_rows == 0 || act);
  JANUS_CHECK_ALIGN(act == nullptr || aligned(act, 16));
  st = check_w16_set(weights16, weights16_bytes, n_experts, d, h);
  if (st != JANUS_OK) return st;
  if (n_rows == 0) return JANUS_OK;
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const SplitLayout L = split_layout(n_rows, n_experts, d, h);
  char* w = (char*)workspace;
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream));
  tc::F16Second second = f16_second_at(w + L.off_second, n_rows, n_experts, d, h);
  uint16_t* w16 = (uint16_t*)(w + L.off_w16);
  float* winv = (float*)(w + L.off_winv);
  if (weights16) w16_set_parts(weights16, n_experts, d, h, 2, &w16, &winv, &second);
  st = tc::expert_ffn_vjp_split(gd16, gd_scale, act, offsets, n_experts, n_rows, d, h, w1, w2, dxd,
                                (float*)(w + L.off_h), w16, winv, &((WsHeader*)workspace)->error, stream, dxd_rows,
                                use_f16_second(n_rows, n_experts, h) ? &second : nullptr, weights16 != nullptr);
  if (st != JANUS_OK) return st;
  return launch_status();
}

extern "C" janus_status janus_expert_ffn_workspace_size(int64_t n_rows, int32_t d, int32_t h,
                                                        int32_t n_experts, int32_t vjp,
                                                        int32_t have_act, janus_ffn_mode mode,
                                                        size_t* bytes) {
  JANUS_CHECK_ARG(bytes && n_rows >= 0 && d >= 1 && h >= 1 && n_experts >= 1);
  JANUS_CHECK_ARG(mode == JANUS_FFN_FP32_SIMT || mode == JANUS_FFN_3XTF32);
  *bytes = ffn_layout(n_rows, h, vjp != 0, have_act != 0).total;
  return JANUS_OK;
}

namespace {

// yd_rows (device array of n_rows row pointers) replaces yd when set.
janus_status ffn_fwd(const float* xd, const int32_t* offsets, int32_t n_experts, int64_t n_rows, int32_t d,
                     int32_t h, const float* w1, const float* w2, float* yd, float* const* yd_rows, float* act,
                     uint32_t flags, janus_ffn_mode mode, void* workspace, size_t workspace_bytes,
                     janus_stream_t stream_) {
  JANUS_CHECK_ARG((flags & ~(uint32_t)JANUS_FFN_X_DEQUANTIZED) == 0);
  cudaStream_t stream = (cudaStream_t)stream_;
  janus_status st = check_ffn(xd, offsets, n_experts, n_rows, d, h, w1, w2,
                              yd_rows ? reinterpret_cast<const float*>(yd_rows) : yd, mode);
  if (st != JANUS_OK) return st;
  const FfnLayout L = ffn_layout(n_rows, h, false, act != nullptr);
  JANUS_CHECK_ARG(workspace && workspace_bytes >= L.total);
  JANUS_CHECK_ALIGN(aligned(workspace, 256) && (act == nullptr || aligned(act, 16)));
  if (n_rows == 0) return JANUS_OK;
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  float* H = (float*)((char*)workspace + L.off_h);
  const int64_t sw = (int64_t)d * h;
  // the error word starts clear in both modes, so janus_check on this
  // workspace reports only this call's faults
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream));
  if (mode == JANUS_FFN_3XTF32) {
    st = tc::expert_ffn_fwd(xd, offsets, n_experts, n_rows, d, h, w1, w2, yd, act, H,
                            &((WsHeader*)workspace)->error, stream, yd_rows,
                            (flags & JANUS_FFN_X_DEQUANTIZED) != 0);
    if (st != JANUS_OK) return st;
    return launch_status();
  }
  launch_simt<false, simt::kEpiSilu>(make_args(xd, w1, sw, H, act, nullptr, offsets, n_experts, d, h, n_rows), stream);
  simt::Args a2 = make_args(H, w2, sw, yd, nullptr, nullptr, offsets, n_experts, h, d, n_rows);
  a2.c_rows = yd_rows;
  launch_simt<false, simt::kEpiStore>(a2, stream);
  return launch_status();
}

// dxd_rows (device array of n_rows row pointers) replaces dxd when set.
janus_status ffn_vjp(const float* xd, const float* gd, const float* act, const int32_t* offsets,
                     int32_t n_experts, int64_t n_rows, int32_t d, int32_t h, const float* w1, const float* w2,
                     float* dxd, float* const* dxd_rows, janus_ffn_mode mode, void* workspace,
                     size_t workspace_bytes, janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  janus_status st = check_ffn(xd, offsets, n_experts, n_rows, d, h, w1, w2,
                              dxd_rows ? reinterpret_cast<const float*>(dxd_rows) : dxd, mode);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(n_rows == 0 || gd);
  JANUS_CHECK_ALIGN(n_rows == 0 || aligned(gd, 16));
  JANUS_CHECK_ALIGN(act == nullptr || aligned(act, 16));
  const FfnLayout L = ffn_layout(n_rows, h, true, act != nullptr);
  JANUS_CHECK_ARG(workspace && workspace_bytes >= L.total);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  if (n_rows == 0) return JANUS_OK;
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const size_t rh = align_up(sizeof(float) * (size_t)n_rows * (size_t)h, 256);
  float* dA = (float*)((char*)workspace + L.off_h);
  float* A = act ? const_cast<float*>(act) : (float*)((char*)workspace + L.off_h + rh);
  const int64_t sw = (int64_t)d * h;
  // the error word starts clear in both modes, so janus_check on this
  // workspace reports only this call's faults
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream));
  if (mode == JANUS_FFN_3XTF32) {
    st = tc::expert_ffn_vjp(xd, gd, act, A, offsets, n_experts, n_rows, d, h, w1, w2, dxd, dA,
                            &((WsHeader*)workspace)->error, stream, dxd_rows);
    if (st != JANUS_OK) return st;
    return launch_status();
  }
  if (!act)
    launch_simt<false, simt::kEpiStore>(make_args(xd, w1, sw, A, nullptr, nullptr, offsets, n_experts, d, h, n_rows), stream);
  launch_simt<true, simt::kEpiDSilu>(make_args(gd, w2, sw, dA, nullptr, A, offsets, n_experts, d, h, n_rows), stream);
  simt::Args a4 = make_args(dA, w1, sw, dxd, nullptr, nullptr, offsets, n_experts, h, d, n_rows);
  a4.c_rows = dxd_rows;
  launch_simt<true, simt::kEpiStore>(a4, stream);
  return launch_status();
}

}  // namespace

extern "C" janus_status janus_expert_ffn_fwd(const float* xd, const int32_t* offsets,
                                             int32_t n_experts, int64_t n_rows, int32_t d,
                                             int32_t h, const float* w1, const float* w2,
                                             float* yd, float* act, janus_ffn_mode mode,
                                             void* workspace, size_t workspace_bytes,
                                             janus_stream_t stream) {
  return ffn_fwd(xd, offsets, n_experts, n_rows, d, h, w1, w2, yd, nullptr, act, 0, mode, workspace,
                 workspace_bytes, stream);
}

extern "C" janus_status janus_expert_ffn_fwd_rows(const float* xd, const int32_t* offsets,
                                                  int32_t n_experts, int64_t n_rows, int32_t d,
                                                  int32_t h, const float* w1, const float* w2,
                                                  float* const* yd_rows, float* act, janus_ffn_mode mode,
                                                  void* workspace, size_t workspace_bytes,
                                                  janus_stream_t stream) {
  JANUS_CHECK_ARG(n_rows == 0 || yd_rows);
  return ffn_fwd(xd, offsets, n_experts, n_rows, d, h, w1, w2, nullptr, yd_rows, act, 0, mode, workspace,
                 workspace_bytes, stream);
}

extern "C" janus_status janus_expert_ffn_fwd_ex(const float* xd, const int32_t* offsets, int32_t n_experts,
                                                int64_t n_rows, int32_t d, int32_t h, const float* w1,
                                                const float* w2, float* yd, float* const* yd_rows, float* act,
                                                uint32_t flags, janus_ffn_mode mode, void* workspace,
                                                size_t workspace_bytes, janus_stream_t stream) {
  JANUS_CHECK_ARG((yd == nullptr) != (yd_rows == nullptr) || n_rows == 0);
  return ffn_fwd(xd, offsets, n_experts, n_rows, d, h, w1, w2, yd, yd_rows, act, flags, mode, workspace,
                 workspace_bytes, stream);
}

extern "C" janus_status janus_expert_ffn_vjp(const float* xd, const float* gd, const float* act,
                                             const int32_t* offsets, int32_t n_experts,
                                             int64_t n_rows, int32_t d, int32_t h,
                                             const float* w1, const float* w2, float* dxd,
                                             janus_ffn_mode mode, void* workspace,
                                             size_t workspace_bytes, janus_stream_t stream) {
  return ffn_vjp(xd, gd, act, offsets, n_experts, n_rows, d, h, w1, w2, dxd, nullptr, mode, workspace,
                 workspace_bytes, stream);
}

extern "C" janus_status janus_expert_ffn_vjp_rows(const float* xd, const float* gd, const float* act,
                                                  const int32_t* offsets, int32_t n_experts,
                                                  int64_t n_rows, int32_t d, int32_t h,
                                                  const float* w1, const float* w2, float* const* dxd_rows,
                                                  janus_ffn_mode mode, void* workspace,
                                                  size_t workspace_bytes, janus_stream_t stream) {
  JANUS_CHECK_ARG(n_rows == 0 || dxd_rows);
  return ffn_vjp(xd, gd, act, offsets, n_experts, n_rows, d, h, w1, w2, nullptr, dxd_rows, mode, workspace,
                 workspace_bytes, stream);
}

extern "C" janus_status janus_expert_ffn_weight_grad_workspace_size(int64_t n_rows, int32_t h,
                                                                    int32_t have_act, size_t* bytes) {
  JANUS_CHECK_ARG(bytes && n_rows >= 0 && h >= 1);
  const size_t rh = align_up(sizeof(float) * (size_t)n_rows * (size_t)h, 256);
  *bytes = sizeof(WsHeader) + (have_act ? 2 : 3) * rh;
  return JANUS_OK;
}

extern "C" janus_status janus_expert_ffn_weight_grad(const float* xd, const float* gd, const float* act,
                                                     const int32_t* offsets, int32_t n_experts,
                                                     int64_t n_rows, int32_t d, int32_t h,
                                                     const float* w1, const float* w2, float* dw1,
                                                     float* dw2, janus_ffn_mode mode, void* workspace,
                                                     size_t workspace_bytes, janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  janus_status st = check_ffn(xd, offsets, n_experts, n_rows, d, h, w1, w2, dw1, mode);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(dw1 && dw2 && (n_rows == 0 || gd));
  JANUS_CHECK_ALIGN(aligned(dw1, 16) && aligned(dw2, 16));
  JANUS_CHECK_ALIGN(n_rows == 0 || aligned(gd, 16));
  JANUS_CHECK_ALIGN(act == nullptr || aligned(act, 16));
  size_t need = 0;
  st = janus_expert_ffn_weight_grad_workspace_size(n_rows, h, act != nullptr, &need);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(workspace && workspace_bytes >= need);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  const size_t wbytes = sizeof(float) * (size_t)n_experts * (size_t)d * (size_t)h;
  if (n_rows == 0) {   // no rows routed anywhere: every gradient is zero
    JANUS_CUDA_TRY(cudaMemsetAsync(dw1, 0, wbytes, stream));
    JANUS_CUDA_TRY(cudaMemsetAsync(dw2, 0, wbytes, stream));
    return JANUS_OK;
  }
  const size_t rh = align_up(sizeof(float) * (size_t)n_rows * (size_t)h, 256);
  char* w = (char*)workspace + sizeof(WsHeader);
  float* dA = (float*)w;
  float* H = (float*)(w + rh);
  float* A = act ? const_cast<float*>(act) : (float*)(w + 2 * rh);
  // the error word starts clear in both modes, so janus_check on this
  // workspace reports only this call's faults
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream));
  if (mode == JANUS_FFN_3XTF32) {
    st = tc::expert_ffn_weight_grad(xd, gd, act, A, offsets, n_experts, n_rows, d, h, w1, w2, dw1, dw2, dA,
                                    H, &((WsHeader*)workspace)->error, stream);
    if (st != JANUS_OK) return st;
    return launch_status();
  }
  const int64_t sw = (int64_t)d * h;
  if (!act)
    launch_simt<false, simt::kEpiStore>(make_args(xd, w1, sw, A, nullptr, nullptr, offsets, n_experts, d, h, n_rows), stream);
  launch_simt<true, simt::kEpiDSilu>(make_args(gd, w2, sw, dA, H, A, offsets, n_experts, d, h, n_rows), stream);
  simt::TnArgs t1{xd, dA, dw1, offsets, n_experts, d, h, 0, n_rows, debug_fault_word()};
  simt::grouped_tn_kernel<<<num_sms() * 2, simt::kThreads, 0, stream>>>(t1);
  simt::TnArgs t2{H, gd, dw2, offsets, n_experts, h, d, 0, n_rows, debug_fault_word()};
  simt::grouped_tn_kernel<<<num_sms() * 2, simt::kThreads, 0, stream>>>(t2);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Second-order pass: gradients of L = <dxd(xd, gd; W1, W2), vd> (the VJP of
// the input VJP, which force training differentiates).
//   G0: a = xd W1                  (only without the forward's act)
//   G1: dh = gd W2^T
//   G2: ub = vd W1 -> t1 = ub silu'(a), t2 = ub dh silu''(a), u = dh silu'(a)
//   G3: d_gd = t1 W2,  G4: d_xd = t2 W1^T
//   G5: dW2[e] = T1_e^T Gd_e,  G6/G7: dW1[e] = Vd_e^T U_e + Xd_e^T T2_e
// Workspace: header | dh | t1 | t2 | u (weight gradients) | a (no act), each
// [R,h] FP32 rounded up to 256 bytes.
// ---------------------------------------------------------------------------
extern "C" janus_status janus_expert_ffn_vjp_vjp_workspace_size(int64_t n_rows, int32_t h, int32_t have_act,
                                                                int32_t want_weight_grad, size_t* bytes) {
  JANUS_CHECK_ARG(bytes && n_rows >= 0 && h >= 1);
  const size_t rh = align_up(sizeof(float) * (size_t)n_rows * (size_t)h, 256);
  *bytes = sizeof(WsHeader) + (3 + (want_weight_grad ? 1 : 0) + (have_act ? 0 : 1)) * rh;
  return JANUS_OK;
}

extern "C" janus_status janus_expert_ffn_vjp_vjp(const float* xd, const float* gd, const float* vd,
                                                 const float* act, const int32_t* offsets, int32_t n_experts,
                                                 int64_t n_rows, int32_t d, int32_t h, const float* w1,
                                                 const float* w2, float* d_xd, float* d_gd, float* dw1,
                                                 float* dw2, janus_ffn_mode mode, void* workspace,
                                                 size_t workspace_bytes, janus_stream_t stream_) {
  cudaStream_t stream = (cudaStream_t)stream_;
  janus_status st = check_ffn(xd, offsets, n_experts, n_rows, d, h, w1, w2, d_xd, mode);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(n_rows == 0 || (gd && vd && d_gd));
  JANUS_CHECK_ARG((dw1 == nullptr) == (dw2 == nullptr));
  JANUS_CHECK_ALIGN(n_rows == 0 || (aligned(gd, 16) && aligned(vd, 16) && aligned(d_gd, 16)));
  JANUS_CHECK_ALIGN(act == nullptr || aligned(act, 16));
  JANUS_CHECK_ALIGN(dw1 == nullptr || (aligned(dw1, 16) && aligned(dw2, 16)));
  const bool wg = dw1 != nullptr;
  size_t need = 0;
  st = janus_expert_ffn_vjp_vjp_workspace_size(n_rows, h, act != nullptr, wg, &need);
  if (st != JANUS_OK) return st;
  JANUS_CHECK_ARG(workspace && workspace_bytes >= need);
  JANUS_CHECK_ALIGN(aligned(workspace, 256));
  if (consume_injected_failure()) return JANUS_ERR_CUDA;
  if (n_rows == 0) {   // no rows: the weight gradients are zero, nothing else to write
    if (wg) {
      const size_t wbytes = sizeof(float) * (size_t)n_experts * (size_t)d * (size_t)h;
      JANUS_CUDA_TRY(cudaMemsetAsync(dw1, 0, wbytes, stream));
      JANUS_CUDA_TRY(cudaMemsetAsync(dw2, 0, wbytes, stream));
    }
    return JANUS_OK;
  }
  const size_t rh = align_up(sizeof(float) * (size_t)n_rows * (size_t)h, 256);
  char* w = (char*)workspace + sizeof(WsHeader);
  float* dh = (float*)w;
  float* t1 = (float*)(w + rh);
  float* t2 = (float*)(w + 2 * rh);
  float* u = wg ? (float*)(w + 3 * rh) : nullptr;
  float* A = act ? const_cast<float*>(act) : (float*)(w + (wg ? 4 : 3) * rh);
  // the error word starts clear in both modes, so janus_check on this
  // workspace reports only this call's faults
  JANUS_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), stream));
  if (mode == JANUS_FFN_3XTF32) {
    st = tc::expert_ffn_vjp_vjp(xd, gd, vd, act, A, offsets, n_experts, n_rows, d, h, w1, w2, d_xd, d_gd, dw1,
                                dw2, dh, t1, t2, u, &((WsHeader*)workspace)->error, stream);
    if (st != JANUS_OK) return st;
    return launch_status();
  }
  const int64_t sw = (int64_t)d * h;
  if (!act)
    launch_simt<false, simt::kEpiStore>(make_args(xd, w1, sw, A, nullptr, nullptr, offsets, n_experts, d, h, n_rows), stream);
  launch_simt<true, simt::kEpiStore>(make_args(gd, w2, sw, dh, nullptr, nullptr, offsets, n_experts, d, h, n_rows), stream);
  simt::Args a2 = make_args(vd, w1, sw, t1, t2, A, offsets, n_experts, d, h, n_rows);
  a2.aux2 = dh;
  a2.C3 = u;
  launch_simt<false, simt::kEpiD2>(a2, stream);
  launch_simt<false, simt::kEpiStore>(make_args(t1, w2, sw, d_gd, nullptr, nullptr, offsets, n_experts, h, d, n_rows), stream);
  launch_simt<true, simt::kEpiStore>(make_args(t2, w1, sw, d_xd, nullptr, nullptr, offsets, n_experts, h, d, n_rows), stream);
  if (wg) {
    simt::TnArgs g2{t1, gd, dw2, offsets, n_experts, h, d, 0, n_rows, debug_fault_word()};
    simt::grouped_tn_kernel<<<num_sms() * 2, simt::kThreads, 0, stream>>>(g2);
    simt::TnArgs g1a{vd, u, dw1, offsets, n_experts, d, h, 0, n_rows, debug_fault_word()};
    simt::grouped_tn_kernel<<<num_sms() * 2, simt::kThreads, 0, stream>>>(g1a);
    simt::TnArgs g1b{xd, t2, dw1, offsets, n_experts, d, h, 1, n_rows, debug_fault_word()};
    simt::grouped_tn_kernel<<<num_sms() * 2, simt::kThreads, 0, stream>>>(g1b);
  }
  return launch_status();
}
