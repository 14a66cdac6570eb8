// Grouped expert MLP on the tcgen05 tensor cores with the 3xTF32 split
// (JANUS_FFN_3XTF32).  Internal header, included by expert_ffn.cu.
#pragma once

#include "common.cuh"

namespace janus {
namespace tc {

// extra workspace bytes the tensor-core path needs beyond the activations
size_t workspace_extra();

// `err` is the workspace header's error word (a bounded wait that ran out
// records a timeout there).
// yd_rows (nullable): row p of yd is written to yd_rows[p] instead of yd + p d.
// x_tf32_exact: every xd value is exact in TF32 (dequantized FP16 rows), so the
// first GEMM drops the product with xd's residual; inexact rows are reported
// as a data fault.
janus_status expert_ffn_fwd(const float* xd, const int32_t* offsets, int32_t E, int64_t R,
                            int32_t d, int32_t h, const float* w1, const float* w2, float* yd,
                            float* act, float* H, int32_t* err, cudaStream_t stream,
                            float* const* yd_rows = nullptr, bool x_tf32_exact = false);

// Scratch of the MLP's second GEMM on the kind::f16 path (H W2 in the
// forward, dA W1^T in the VJP, the [R][h] activation split into two FP16
// terms per row): the activation's planes [2R][h] and row scales [R], the
// FP16 split of the weights ([2E][d][h]) and its 1 / S [E][ceil(h/256)][d].
struct F16Second {
  uint16_t* h16;
  float* hscale;
  uint16_t* w16;
  float* winv;
};

// The FP16 split of a GEMM's weights for the kind::f16 path: w16 = [hi | mid],
// each [E][N][Kd] FP16 (2 * E * N * Kd values), winv [E][ceil(Kd/256)][N] =
// 1 / S per output feature and K chunk of 256.  transposed: w is [E][Kd][N]
// (x W); else [E][N][Kd] (x W^T).
// One kernel; N % 4 == 0 and Kd % 4 == 0 (JANUS_ERR_MISALIGNED otherwise).
janus_status split_weights_f16(const float* w, int32_t E, int32_t Kd, int32_t N, bool transposed, uint16_t* w16,
                               float* winv, cudaStream_t stream);
// Both splits of W [E][A][B] from one read: (w16t, winvt) = the transposed
// split (Kd = A, N = B) and (w16r, winvr) = the row split (N = A, Kd = B),
// the same bits as the two split_weights_f16 calls.  A % 4 == 0, B % 4 == 0.
janus_status split_weights_f16_both(const float* w, int32_t E, int32_t A, int32_t B, uint16_t* w16t, float* winvt,
                                    uint16_t* w16r, float* winvr, cudaStream_t stream);

// Forward / input VJP on rows given as two FP16 terms (hi plane [R][d] then
// mid plane [R][d]) with a per-row scale (janus_dispatch_split): the first
// GEMM (x W1, or gd W2^T) on the kind::f16 path with three products against
// the FP16 split of W1 / W2 (written into w16 / winv).  The second GEMM runs
// on 3xTF32 (the VJP's first GEMM then applies silu'(a) in its epilogue into
// dA), or, with `second`, on the kind::f16 path after one pass splits the
// activation (H = silu(a), or dA = dH silu'(a) with dH stored into dA's
// buffer) into two FP16 terms per row.  d % 8 == 0; h % 8 == 0 with second.
// weights_presplit: w16 / winv (and second's w16 / winv) already hold the
// weights' splits, and no split of the weights is launched.
janus_status expert_ffn_fwd_split(const uint16_t* rows16, const float* row_scale, const int32_t* offsets, int32_t E,
                                  int64_t R, int32_t d, int32_t h, const float* w1, const float* w2, float* yd,
                                  float* act, float* H, uint16_t* w16, float* winv, int32_t* err,
                                  cudaStream_t stream, float* const* yd_rows = nullptr,
                                  const F16Second* second = nullptr, bool weights_presplit = false);
janus_status expert_ffn_vjp_split(const uint16_t* gd16, const float* gd_scale, const float* act,
                                  const int32_t* offsets, int32_t E, int64_t R, int32_t d, int32_t h,
                                  const float* w1, const float* w2, float* dxd, float* dA, uint16_t* w16,
                                  float* winv, int32_t* err, cudaStream_t stream, float* const* dxd_rows = nullptr,
                                  const F16Second* second = nullptr, bool weights_presplit = false);

// The forward on the FP16 payload itself: row p of xd is f32(payload[p]) *
// row_scale[p].  The first GEMM runs on the kind::f16 tensor path against the
// FP16 split of W1 (written into w16 / winv first); d % 8 == 0, payload
// 16-byte aligned.
// second (nullable): run the second GEMM (H W2) on the kind::f16 path too.
// weights_presplit as in expert_ffn_fwd_split.
janus_status expert_ffn_fwd_packed(const uint16_t* payload, const float* row_scale, const int32_t* offsets,
                                   int32_t E, int64_t R, int32_t d, int32_t h, const float* w1, const float* w2,
                                   float* yd, float* act, float* H, uint16_t* w16, float* winv, int32_t* err,
                                   cudaStream_t stream, float* const* yd_rows = nullptr,
                                   const F16Second* second = nullptr, bool weights_presplit = false);
janus_status expert_ffn_vjp(const float* xd, const float* gd, const float* act_in, float* A,
                            const int32_t* offsets, int32_t E, int64_t R, int32_t d, int32_t h,
                            const float* w1, const float* w2, float* dxd, float* dA, int32_t* err,
                            cudaStream_t stream, float* const* dxd_rows = nullptr);

// Per-expert weight gradients: dW1[e] = Xd_e^T dA_e, dW2[e] = H_e^T Gd_e with
// dA = (gd W2^T) * silu'(a) and H = silu(a) computed into dA and H.
janus_status expert_ffn_weight_grad(const float* xd, const float* gd, const float* act_in, float* A,
                                    const int32_t* offsets, int32_t E, int64_t R, int32_t d, int32_t h,
                                    const float* w1, const float* w2, float* dw1, float* dw2, float* dA,
                                    float* H, int32_t* err, cudaStream_t stream);

// Second-order pass (the VJP of the input VJP) for the cotangent vd of dxd:
//   dh = gd W2^T, t1 = (vd W1) silu'(a), t2 = (vd W1) dh silu''(a), u = dh silu'(a)
//   d_gd = t1 W2, d_xd = t2 W1^T;  with dw1/dw2 (both or neither):
//   dW2[e] = T1_e^T Gd_e, dW1[e] = Vd_e^T U_e + Xd_e^T T2_e.
// dh, t1, t2 (and u with the weight gradients) are [R,h] scratch; A receives a
// when act_in is NULL.
janus_status expert_ffn_vjp_vjp(const float* xd, const float* gd, const float* vd, const float* act_in, float* A,
                                const int32_t* offsets, int32_t E, int64_t R, int32_t d, int32_t h,
                                const float* w1, const float* w2, float* d_xd, float* d_gd, float* dw1,
                                float* dw2, float* dh, float* t1, float* t2, float* u, int32_t* err,
                                cudaStream_t stream);

}  // namespace tc
}  // namespace janus
