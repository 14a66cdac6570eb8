/*
 * janus.h - C ABI of libjanus.so: the element-type-routed sparse MoE layer over
 * atom feature tokens and the edge-to-atom aggregation that feeds it, as
 * hand-written CUDA kernels for B200 (sm_100a).
 *
 * Sources (web pages on the method, cited by title and section):
 *   [Review]    "Breaking the Training Barrier of Billion-Parameter Universal
 *               Machine Learning Interatomic Potentials" (xllm-io paper review)
 *   [News]      "11.5B参数、1.2EFLOPS、训练从数周压到数小时" (ScienceAI)
 *   [Blueprint] "MatRIS-MoE与Janus框架：构建百亿参数通用机器学习原子间势"
 *
 * Notation: N atoms, T element types, E experts, K experts per atom (top-K),
 * R = N*K routed tokens ("slots"), d feature size, h expert hidden size,
 * Ed edges.  Flat slot s = i*K + k is atom i's k-th expert.  The dispatch
 * buffer holds one row per slot, grouped by expert: rows
 * [offsets[e], offsets[e+1]) belong to expert e, atoms ascending inside.
 *
 * Conventions for every call:
 *   - Every array argument is a DEVICE pointer (cudaMalloc'd or managed),
 *     owned by the caller.  The library never allocates or frees memory; a
 *     call that needs scratch space takes a caller-owned `workspace` whose
 *     size is given by the matching *_workspace_size query.
 *   - Every call is asynchronous on the given stream (0 = legacy default
 *     stream), never synchronises (except janus_check), and is thread-safe.
 *   - Arrays are dense row-major.  FP32 feature rows ([*, d]) need a 16-byte
 *     aligned base and d % 4 == 0; FP16 payload rows need an 8-byte aligned
 *     base (same d rule).  Otherwise JANUS_ERR_MISALIGNED.
 *   - Limits: 1 <= K <= E <= 256, 1 <= T <= 4096, N*K < 2^31, 1 <= d, h <= 2^20.
 *     Edge counts and feature element offsets are 64-bit.
 *   - Arguments are checked before anything is launched: a failed check
 *     returns an error and launches nothing.  Index arrays that a call takes
 *     as input (perm, slot_of, offsets, row_ptr) must be what janus_route /
 *     a valid CSR would produce; the release build does not re-validate them
 *     on the device (edge ranges are clamped), the debug build does (see
 *     janus_debug_check).
 *   - Data-dependent faults (a type id outside [0,T), a non-finite gate
 *     logit, a non-finite feature to be packed, a bounded tensor-core wait
 *     that ran out, rows that break JANUS_FFN_X_DEQUANTIZED, expert-parallel
 *     rows beyond the receive capacity) are recorded in the workspace's error
 *     word and reported by janus_check(); the call still writes every output
 *     (bad type ids are treated as type 0) so no out-of-bounds access can
 *     follow.
 */
#ifndef JANUS_H_
#define JANUS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* janus_stream_t; /* == cudaStream_t */

typedef enum {
  JANUS_OK = 0,
  JANUS_ERR_INVALID_ARG = 1, /* null pointer, size/limit violation, workspace too small */
  JANUS_ERR_MISALIGNED = 2,  /* feature pointer not 16-byte (FP32) / 8-byte (FP16) aligned, or d % 4 != 0 */
  JANUS_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
  JANUS_ERR_DATA = 4         /* data-dependent fault recorded on the device (see janus_check) */
} janus_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* janus_status_string(janus_status s);

/* Library ABI version (major*10000 + minor*100 + patch). */
int32_t janus_version(void);

/* Synchronises `stream`, then reads the error word at the start of a
 * workspace used by a call that takes one (routing, packing, the expert MLP
 * calls, the expert-parallel sends); each such call clears the word when it
 * starts (janus_ep_dispatch: see there).  Returns JANUS_OK, JANUS_ERR_DATA
 * if a kernel recorded a data fault, or JANUS_ERR_CUDA. */
janus_status janus_check(const void* workspace, janus_stream_t stream);

/* -------------------------------------------------------------------------
 * Routing.  [Review] section 3.2 (sparse MoE design): each element type
 * activates its own top-K experts, so the active set does not depend on the
 * coordinates; [News] (model architecture paragraph) says the same.  [News]
 * (training framework paragraph): JIT planning routes a batch before the
 * step and counts the tokens per expert.
 *
 *   S_t = the K experts with the largest gate[t, :], descending logit, ties
 *         to the lower expert id;
 *   topk_expert[i,k] = S_{types[i]}[k];
 *   topk_weight[i,k] = softmax over the K selected logits of gate[types[i],:];
 *   counts[e]  = number of slots routed to e;  offsets = exclusive scan
 *                (offsets[0] = 0, offsets[E] = R);
 *   perm[p]    = the slot held by dispatch row p (stable: slots ascending
 *                inside each expert);  slot_of[perm[p]] = p.
 *
 * in : types [N] int32, gate [T,E] float32 (finite)
 * out: topk_expert [N,K] int32, topk_weight [N,K] float32, counts [E] int32,
 *      offsets [E+1] int32, perm [R] int32, slot_of [R] int32
 * workspace: janus_route_workspace_size() bytes; its error word records type
 *      ids outside [0,T) (those atoms are routed as type 0) and gate rows
 *      holding a non-finite logit (their top-K is still K distinct experts,
 *      but its order and weights are undefined).
 * N == 0 is allowed (counts and offsets are zeroed).
 * ------------------------------------------------------------------------- */
janus_status janus_route_workspace_size(int64_t n_atoms, int32_t n_types,
                                        int32_t n_experts, int32_t top_k,
                                        size_t* bytes);
janus_status janus_route(const int32_t* types, int64_t n_atoms, const float* gate,
                         int32_t n_types, int32_t n_experts, int32_t top_k,
                         int32_t* topk_expert, float* topk_weight, int32_t* counts,
                         int32_t* offsets, int32_t* perm, int32_t* slot_of,
                         void* workspace, size_t workspace_bytes,
                         janus_stream_t stream);

/* Routing of several MoE layers at once, as JIT planning does for every MoE
 * layer of a step before it runs ([News], training-framework paragraph: route
 * all layers in a batch, count each expert's token load).  gates is
 * [L][T][E]; every output is stacked per layer: topk_expert/topk_weight
 * [L][N][K], counts [L][E], offsets [L][E+1], perm/slot_of [L][R].  Layer l's
 * outputs equal janus_route(types, gates[l]).  1 <= L <= 65535; the workspace
 * grows with L (janus_route_layers_workspace_size). */
janus_status janus_route_layers_workspace_size(int64_t n_atoms, int32_t n_types, int32_t n_experts,
                                               int32_t top_k, int32_t n_layers, size_t* bytes);
janus_status janus_route_layers(const int32_t* types, int64_t n_atoms, const float* gates,
                                int32_t n_layers, int32_t n_types, int32_t n_experts, int32_t top_k,
                                int32_t* topk_expert, float* topk_weight, int32_t* counts,
                                int32_t* offsets, int32_t* perm, int32_t* slot_of, void* workspace,
                                size_t workspace_bytes, janus_stream_t stream);

/* Active-expert lists ([News], JIT planning: the experts a batch activates are
 * restored before the expert stage).  For each of L layers, the experts with
 * at least one routed row, in ascending id order:
 *   active[l*E + j] = the j-th e with counts[l*E + e] > 0, j < n_active[l]
 * in : counts [L,E] (device int32, e.g. janus_route_layers' counts)
 * out: active [L,E] (entries past n_active[l] untouched), n_active [L]
 * One CTA per layer; E <= 256.  Errors: JANUS_ERR_INVALID_ARG on bad sizes. */
janus_status janus_active_experts(const int32_t* counts, int32_t n_layers, int32_t n_experts,
                                  int32_t* active, int32_t* n_active, janus_stream_t stream);

/* -------------------------------------------------------------------------
 * Dispatch.  [Review] section 3.5 (CNIS kernels, MoE dispatch/combine).
 *   xd[slot_of[i*K+k], :] = x[i, :] * (topk_weight ? topk_weight[i*K+k] : 1)
 * The weighted form is the first step of the input VJP (upstream gradient
 * times gate weight).  Each atom row is read once and written K times.
 * in : x [N,d] float32, slot_of [R] int32, topk_weight [N,K] float32 or NULL
 * out: xd [R,d] float32
 * ------------------------------------------------------------------------- */
janus_status janus_dispatch(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                            const int32_t* slot_of, const float* topk_weight,
                            float* xd, janus_stream_t stream);

/* Dispatch into two FP16 terms per value, for the expert MLP's FP16
 * tensor-core GEMMs (janus_expert_ffn_fwd_split / _vjp_split).  Same rows
 * and values as janus_dispatch, v = x[i,:] * (topk_weight[i*K+k] or 1) in
 * FP32, written for dispatch row p = slot_of[i*K+k] as
 *   hi[p,:] = fp16(v * S_p),  mid[p,:] = fp16(v * S_p - hi[p,:]),
 *   row_scale[p] = 1 / S_p,
 * with S_p the power of two that puts the row's largest |v| in [2^14, 2^15)
 * (1 for a zero row; clamped to [2^-126, 2^126]).  hi + mid carries 22
 * significant bits of every value within 2^18 of the row's largest; smaller
 * values keep an absolute error below 2^-40 of it.  Not on the pages: an
 * implementation layout of the dispatch buffer for the FP16 tensor path.
 * out: rows16 = [hi | mid], 2 R rows of d binary16 (16-byte aligned),
 *      row_scale [R] float32
 * workspace: janus_dispatch_split_workspace_size bytes (the rows' maxima),
 *      256-byte aligned.  Two passes over x (row maxima, then the dispatch). */
janus_status janus_dispatch_split_workspace_size(int64_t n_atoms, size_t* bytes);
janus_status janus_dispatch_split(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                                  const int32_t* slot_of, const float* topk_weight, uint16_t* rows16,
                                  float* row_scale, void* workspace, size_t workspace_bytes,
                                  janus_stream_t stream);

/* -------------------------------------------------------------------------
 * Atom-type-aware FP16 packing.  [Review] section 3.5 (CNIS, atom-type-aware
 * FP16 compression): after routing, the dispatch buffer's tokens are grouped
 * by atom type, quantised with one scale per type, carried as FP16 (half the
 * FP32 bytes) and dequantised afterwards.
 *   amax_t  = max |x[i,j]| over atoms i of type t;
 *   scale_t = the smallest power of two 2^e with amax_t <= 65504 * 2^e,
 *             e clamped to [-126, 127]; 1 if amax_t == 0 or type t is absent;
 *   payload[slot_of[i*K+k], j] = binary16_rne(x[i,j] / scale_{types[i]}).
 * Fused gather: x is read twice (amax pass, pack pass); payload is written in
 * dispatch order.
 * in : x [N,d] float32, types [N], slot_of [R]
 * out: payload [R,d] IEEE binary16 bit patterns, scale [T] float32
 * workspace: janus_quant_by_type_workspace_size() bytes; its error word
 *      records bad type ids and non-finite features.
 * ------------------------------------------------------------------------- */
janus_status janus_quant_by_type_workspace_size(int32_t n_types, size_t* bytes);
janus_status janus_quant_by_type(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                                 const int32_t* types, int32_t n_types,
                                 const int32_t* slot_of, uint16_t* payload, float* scale,
                                 void* workspace, size_t workspace_bytes,
                                 janus_stream_t stream);

/* Same packing as janus_quant_by_type, for callers that cannot allocate
 * device memory (no workspace argument).  The paper has no counterpart: this
 * is a library convenience.  It is meant for code that must not call
 * cudaMalloc or any allocating routine where it packs (for example inside a
 * step run under an allocator that forbids allocation, or a plug-in that is
 * handed fixed buffers); the caller still provides x, types, slot_of, payload
 * and scale.  Scratch lives in a library-owned device array of 16,640 bytes
 * (a 256-byte header plus one 32-bit word per element type), which every GPU
 * that loads the library keeps until the process exits.
 *   - n_types must be <= 4096; larger values return JANUS_ERR_INVALID_ARG.
 *   - The first call in each CUDA context (the device's primary context, or
 *     a context the caller created with the driver API) looks up the array's
 *     device address there (cudaGetSymbolAddress, once per context, with
 *     that context current); make that first call before any stream capture.
 *     The cached address does not survive cudaDeviceReset: after a reset,
 *     do not call this entry point again in the same process.
 *   - Every call clears and reuses the same array, so calls whose work
 *     overlaps on the GPU (different streams, or different host threads on one
 *     device) race and may produce wrong scales; serialise them.
 *   - Data faults are not reported (there is no workspace to hand to
 *     janus_check); bad type ids are packed as type 0.
 * Calls no cudaMalloc/cudaFree and no allocating library routine. */
janus_status janus_quant_by_type_noalloc(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                                         const int32_t* types, int32_t n_types,
                                         const int32_t* slot_of, uint16_t* payload, float* scale,
                                         janus_stream_t stream);

/* Dequantisation of a packed dispatch buffer (same passage):
 *   xd[p, j] = float(payload[p, j]) * scale[types[perm[p] / K]]   (exact)
 * in : payload [R,d] binary16 bits, types [N], perm [R], scale [T]
 * out: xd [R,d] float32 */
janus_status janus_dequant_by_type(const uint16_t* payload, int64_t n_atoms, int32_t d,
                                   int32_t top_k, const int32_t* types, int32_t n_types,
                                   const int32_t* perm, const float* scale, float* xd,
                                   janus_stream_t stream);

/* Per-row scales of the packed dispatch: row_scale[p] = scale[types[perm[p] /
 * top_k]] for the R = n_atoms * top_k dispatch rows (bad type ids as type 0),
 * the per-row form janus_expert_ffn_fwd_packed takes.  row_scale: device
 * float [R]. */
janus_status janus_dispatch_row_scales(int64_t n_atoms, int32_t top_k, const int32_t* types, int32_t n_types,
                                       const int32_t* perm, const float* scale, float* row_scale,
                                       janus_stream_t stream);

/* -------------------------------------------------------------------------
 * Grouped expert MLP.  [Review] section 3.1, Table II (MLP hidden size);
 * each expert is read as bias-free Linear(d,h) -> SiLU -> Linear(h,d):
 *   for rows p in [offsets[e], offsets[e+1]):
 *     a = xd[p,:] W1[e]      (W1 [E,d,h] row-major)
 *     yd[p,:] = silu(a) W2[e] (W2 [E,h,d] row-major),  silu(a) = a / (1 + exp(-a))
 * Input VJP ([Review] section 3.3: forces and stress are autodiff gradients
 * of the energy, so the layer's input gradient is needed):
 *   dxd[p,:] = W1[e] ( (W2[e] gd[p,:]) * silu'(a) ),  silu'(a) = sig(a)(1 + a(1 - sig(a)))
 * offsets stays on the device (the tile scheduler reads it there; no host
 * synchronisation).  n_rows = R = offsets[E].
 * FP32 inputs/outputs; accuracy mode:
 *   JANUS_FFN_FP32_SIMT : FP32 FFMA on the CUDA cores;
 *   JANUS_FFN_3XTF32    : tcgen05 tensor cores, each FP32 operand split into
 *                         a TF32 high part and a TF32 residual, three products.
 * fwd: act [R,h] (nullable) receives a; the workspace holds silu(a).
 * vjp: act (nullable) is a from the forward; NULL recomputes it.
 * The workspace's error word (janus_check) is cleared by every call and
 * receives a bounded tensor-core wait that ran out, rows that break
 * JANUS_FFN_X_DEQUANTIZED, and (debug build) a malformed offsets array.
 * ------------------------------------------------------------------------- */
typedef enum { JANUS_FFN_FP32_SIMT = 0, JANUS_FFN_3XTF32 = 1 } janus_ffn_mode;

janus_status janus_expert_ffn_workspace_size(int64_t n_rows, int32_t d, int32_t h,
                                             int32_t n_experts, int32_t vjp,
                                             int32_t have_act, janus_ffn_mode mode,
                                             size_t* bytes);
janus_status janus_expert_ffn_fwd(const float* xd, const int32_t* offsets, int32_t n_experts,
                                  int64_t n_rows, int32_t d, int32_t h, const float* w1,
                                  const float* w2, float* yd, float* act, janus_ffn_mode mode,
                                  void* workspace, size_t workspace_bytes,
                                  janus_stream_t stream);
janus_status janus_expert_ffn_vjp(const float* xd, const float* gd, const float* act,
                                  const int32_t* offsets, int32_t n_experts, int64_t n_rows,
                                  int32_t d, int32_t h, const float* w1, const float* w2,
                                  float* dxd, janus_ffn_mode mode, void* workspace,
                                  size_t workspace_bytes, janus_stream_t stream);

/* The same two calls with each output row stored at its own address:
 * row p of yd (dxd) goes to yd_rows[p][0..d) (dxd_rows[p][0..d)) instead of
 * yd + p d.  yd_rows / dxd_rows: device array of n_rows pointers (16-byte
 * aligned array); each pointer 16-byte aligned with room for d floats,
 * possibly in a peer GPU's mapped memory (janus_ep_return_rows builds the
 * expert-parallel return table).  Only the rows of the offsets' segments are
 * read from the table.  The final GEMM's stores are made visible system-wide
 * before it completes. */
janus_status janus_expert_ffn_fwd_rows(const float* xd, const int32_t* offsets, int32_t n_experts,
                                       int64_t n_rows, int32_t d, int32_t h, const float* w1,
                                       const float* w2, float* const* yd_rows, float* act,
                                       janus_ffn_mode mode, void* workspace, size_t workspace_bytes,
                                       janus_stream_t stream);
/* The general forward: yd or yd_rows (exactly one non-NULL), and flags.
 * JANUS_FFN_X_DEQUANTIZED: every xd value is an FP16 value times a power of
 * two (rows written by janus_dequant_by_type or janus_ep_dequant_rows), hence
 * exact in TF32; the 3xTF32 first GEMM then skips the product with xd's
 * residual (two tensor-core products instead of three).  A row that breaks
 * the promise is reported by janus_check as a data fault (its results then
 * miss that product).  No effect in JANUS_FFN_FP32_SIMT.  Other flag bits:
 * JANUS_ERR_INVALID_ARG. */
#define JANUS_FFN_X_DEQUANTIZED 1u
janus_status janus_expert_ffn_fwd_ex(const float* xd, const int32_t* offsets, int32_t n_experts,
                                     int64_t n_rows, int32_t d, int32_t h, const float* w1,
                                     const float* w2, float* yd, float* const* yd_rows, float* act,
                                     uint32_t flags, janus_ffn_mode mode, void* workspace,
                                     size_t workspace_bytes, janus_stream_t stream);
/* The forward on the FP16 payload itself (the unpack fused into the GEMM):
 * row p of xd is f32(payload[p,:]) * row_scale[p] (payload from
 * janus_quant_by_type or an expert-parallel receive buffer; row_scale from
 * janus_dispatch_row_scales or the receive buffer's scales).  yd or yd_rows
 * (exactly one non-NULL) as in janus_expert_ffn_fwd_ex.
 * JANUS_FFN_3XTF32: the first GEMM multiplies the FP16 rows, as they are,
 * on the tcgen05 kind::f16 tensor path against an FP16 split of W1 that the
 * call writes into the workspace first: per expert, output feature f and K
 * chunk c of 256, a power-of-two scale S_fc puts the chunk's largest |w| in
 * [2^14, 2^15), and w S_fc = hi + mid (two binary16 terms, 22 bits), so
 *   a[p,f] = row_scale[p] sum_c (1 / S_fc) sum_{k in c} payload[p,k] (hi + mid)[f,k]
 * with exact FP16 products and FP32 accumulation per chunk (the chunks of the
 * 3xTF32 GEMM): FP32-accurate, within 1e-5 of the unpacked FP32 forward, at
 * half the tensor-core work of the two-product TF32 form.  The second GEMM
 * (H W2) runs on 3xTF32, or, when n_rows >= M * n_experts and h % 8 == 0,
 * on the same kind::f16 path with three products: the first GEMM then
 * stores a only, one pass over each row writes H = silu(a) as two FP16 terms
 * with a per-row power-of-two scale into the workspace, and W2 is split like
 * W1.  d must be a multiple of 8 (JANUS_ERR_MISALIGNED otherwise) and the
 * payload 16-byte aligned.
 * JANUS_FFN_FP32_SIMT: the rows are unpacked into the workspace first; the
 * result is bit-identical to janus_dequant_by_type followed by
 * janus_expert_ffn_fwd.
 * workspace: janus_expert_ffn_packed_workspace_size bytes (it depends on
 * n_experts through the weight split), 256-byte aligned. */
janus_status janus_expert_ffn_packed_workspace_size(int64_t n_rows, int32_t n_experts, int32_t d, int32_t h,
                                                    janus_ffn_mode mode, size_t* bytes);
/* M, the rows per expert (n_rows / n_experts) from which the packed and split
 * MLP calls run their second GEMM on the kind::f16 path too (384): below it
 * the per-call splits of the weights and the activation cost more than the
 * FP16 GEMMs save.  Callers choosing between the 3xTF32 and the split entry
 * points can use the same rule. */
int32_t janus_expert_ffn_f16_min_rows_per_expert(void);

/* The FP16 splits of a layer's expert weights (the expert MLP of [Review]
 * section 3.1 and its input VJP, section 3.3, kept FP32-accurate on the FP16
 * tensor cores; the split is this library's arithmetic, the pages have none),
 * written once ahead of the MLP calls that use them (weights16 of janus_expert_ffn_fwd_packed,
 * janus_expert_ffn_fwd_split and janus_expert_ffn_vjp_split), so that a
 * forward followed by its input VJP splits each weight tensor in one pass
 * instead of two.  Each part is what those calls otherwise write into their
 * workspace for the same GEMM (power-of-two scale per output feature and K
 * chunk of 256, two binary16 terms; the same bits):
 *   JANUS_W16_FWD: W1 for x W1 and W2 for H W2 (the forward's GEMMs);
 *   JANUS_W16_VJP: W2 for gd W2^T and W1 for dA W1^T (the input VJP's).
 * Both flags: one kernel per weight tensor reads it from DRAM once and writes
 * both of its splits.  A set stays valid while w1 and w2 are unchanged.
 * w1 [E,d,h], w2 [E,h,d] float32, 16-byte aligned; d % 8 == 0, h % 4 == 0
 * (JANUS_ERR_MISALIGNED otherwise).  out: janus_expert_weights_f16_size
 * bytes, 256-byte aligned, owned by the caller (parts not named in `which`
 * are left as they were).  Launches 2 kernels. */
#define JANUS_W16_FWD 1u
#define JANUS_W16_VJP 2u
janus_status janus_expert_weights_f16_size(int32_t n_experts, int32_t d, int32_t h, size_t* bytes);
janus_status janus_expert_weights_f16(const float* w1, const float* w2, int32_t n_experts, int32_t d, int32_t h,
                                      uint32_t which, void* out, size_t out_bytes, janus_stream_t stream);

/* weights16 (nullable; JANUS_FFN_3XTF32 only), weights16_bytes: a set from
 * janus_expert_weights_f16 for these w1, w2 holding the JANUS_W16_FWD parts;
 * the call then launches no split of the weights and reads the set's. */
janus_status janus_expert_ffn_fwd_packed(const uint16_t* payload, const float* row_scale, const int32_t* offsets,
                                         int32_t n_experts, int64_t n_rows, int32_t d, int32_t h, const float* w1,
                                         const float* w2, float* yd, float* const* yd_rows, float* act,
                                         const void* weights16, size_t weights16_bytes, janus_ffn_mode mode,
                                         void* workspace, size_t workspace_bytes, janus_stream_t stream);
janus_status janus_expert_ffn_vjp_rows(const float* xd, const float* gd, const float* act,
                                       const int32_t* offsets, int32_t n_experts, int64_t n_rows,
                                       int32_t d, int32_t h, const float* w1, const float* w2,
                                       float* const* dxd_rows, janus_ffn_mode mode, void* workspace,
                                       size_t workspace_bytes, janus_stream_t stream);

/* The expert MLP on dispatch rows given as two FP16 terms with a per-row
 * scale (janus_dispatch_split), on the tensor cores: the first GEMM of the
 * forward (a = xd W1 -> act, silu(a)) or of the input VJP (dA = (gd W2^T) *
 * silu'(a)) runs on the tcgen05 kind::f16 path with three products,
 *   hi_x hi_w + hi_x mid_w + mid_x hi_w,
 * against an FP16 split of the weights written into the workspace first (per
 * output feature and K chunk of 256 a power-of-two scale and two binary16
 * terms, as in janus_expert_ffn_fwd_packed); products are exact and
 * accumulate in FP32 per chunk, each chunk's sum is scaled by the feature's
 * 1 / S for that chunk, and the result by row_scale[p].  The second GEMM (H W2, or dA W1^T) runs on 3xTF32, or, with
 * n_rows >= M * n_experts and h % 8 == 0, on the same kind::f16 path: the
 * first GEMM then stores a (fwd) or dH = gd W2^T (vjp) plainly, and one pass
 * over each row writes H = silu(a), or dA = dH * silu'(a), as two FP16 terms
 * with a per-row power-of-two scale into the workspace, after which the
 * weights of the second GEMM are split in the same way.  FP32-accurate as
 * the 3xTF32 forms (within 1e-5), at half their tensor-core work per FP16
 * GEMM.
 * fwd: rows16 = [hi | mid] of xd, act [R,h] nullable, yd or yd_rows (one).
 * vjp: gd16 = [hi | mid] of the gate-weighted upstream gradient rows, act
 *      = the forward's pre-activations (required), dxd or dxd_rows (one).
 * d % 8 == 0, h % 4 == 0 (JANUS_ERR_MISALIGNED otherwise); N*K < 2^30.
 * weights16 (nullable), weights16_bytes: a set from janus_expert_weights_f16
 * for these w1, w2 holding the JANUS_W16_FWD parts (fwd) or the
 * JANUS_W16_VJP parts (vjp); the call then launches no split of the weights.
 * workspace: janus_expert_ffn_split_workspace_size bytes, 256-byte aligned;
 * its error word reports as in janus_expert_ffn_fwd. */
janus_status janus_expert_ffn_split_workspace_size(int64_t n_rows, int32_t n_experts, int32_t d, int32_t h,
                                                   size_t* bytes);
janus_status janus_expert_ffn_fwd_split(const uint16_t* rows16, const float* row_scale, const int32_t* offsets,
                                        int32_t n_experts, int64_t n_rows, int32_t d, int32_t h, const float* w1,
                                        const float* w2, float* yd, float* const* yd_rows, float* act,
                                        const void* weights16, size_t weights16_bytes, void* workspace,
                                        size_t workspace_bytes, janus_stream_t stream);
janus_status janus_expert_ffn_vjp_split(const uint16_t* gd16, const float* gd_scale, const float* act,
                                        const int32_t* offsets, int32_t n_experts, int64_t n_rows, int32_t d,
                                        int32_t h, const float* w1, const float* w2, float* dxd,
                                        float* const* dxd_rows, const void* weights16, size_t weights16_bytes,
                                        void* workspace, size_t workspace_bytes, janus_stream_t stream);

/* Expert weight gradients, the parameter side of the same backward pass
 * (force training differentiates the energy w.r.t. inputs and weights,
 * [Review] section 3.3).  For L = sum_p <yd[p,:], gd[p,:]>:
 *   dW1[e] = sum_{p in expert e} xd[p,:]^T dA[p,:],  dA = (gd W2[e]^T) * silu'(a)
 *   dW2[e] = sum_{p in expert e} silu(a[p,:])^T gd[p,:]
 * out: dw1 [E,d,h], dw2 [E,h,d] float32 (overwritten; experts without rows
 * get zeros).  act (nullable) is a from the forward; NULL recomputes it.
 * workspace: janus_expert_ffn_weight_grad_workspace_size() bytes (dA, silu(a)
 * and, without act, a: [R,h] each). */
janus_status janus_expert_ffn_weight_grad_workspace_size(int64_t n_rows, int32_t h, int32_t have_act,
                                                         size_t* bytes);
janus_status janus_expert_ffn_weight_grad(const float* xd, const float* gd, const float* act,
                                          const int32_t* offsets, int32_t n_experts, int64_t n_rows,
                                          int32_t d, int32_t h, const float* w1, const float* w2,
                                          float* dw1, float* dw2, janus_ffn_mode mode, void* workspace,
                                          size_t workspace_bytes, janus_stream_t stream);

/* Second-order pass: the VJP of the input VJP.  Force training fits forces,
 * which are input gradients of the energy ([Review] section 3.3), so a loss on
 * them sends its gradient back through janus_expert_ffn_vjp.  With
 * dxd = W1((W2 gd) * silu'(a)), a = xd W1, per row, and vd the cotangent of dxd
 * (L = sum_p <dxd[p,:], vd[p,:]>):
 *   ub = vd W1,  t1 = ub * silu'(a),  t2 = ub * (gd W2^T) * silu''(a)
 *   d_xd = dL/dxd = t2 W1^T,  d_gd = dL/dgd = t1 W2
 *   dW1[e] = sum_{p in e} vd[p]^T u[p] + xd[p]^T t2[p],  u = (gd W2^T) * silu'(a)
 *   dW2[e] = sum_{p in e} t1[p]^T gd[p]
 *   silu''(a) = sig(a) (1 - sig(a)) (2 + a (1 - 2 sig(a))).
 * in : xd, gd, vd [R,d]; act [R,h] from the forward, or NULL to recompute;
 *      offsets [E+1]; w1 [E,d,h], w2 [E,h,d] (all device, float32, 16-byte
 *      aligned, d and h multiples of 4)
 * out: d_xd, d_gd [R,d]; dw1 [E,d,h] and dw2 [E,h,d], both or neither
 *      (NULL skips the weight part; experts without rows get zeros).
 * workspace: janus_expert_ffn_vjp_vjp_workspace_size() bytes, 256-byte
 *      aligned (dh, t1, t2, u with the weight part, a without act: [R,h]
 *      each).  Errors as janus_expert_ffn_fwd; JANUS_ERR_INVALID_ARG if only one
 *      of dw1, dw2 is given.  3xTF32 timeouts are reported by janus_check. */
janus_status janus_expert_ffn_vjp_vjp_workspace_size(int64_t n_rows, int32_t h, int32_t have_act,
                                                     int32_t want_weight_grad, size_t* bytes);
janus_status janus_expert_ffn_vjp_vjp(const float* xd, const float* gd, const float* vd,
                                      const float* act, const int32_t* offsets, int32_t n_experts,
                                      int64_t n_rows, int32_t d, int32_t h, const float* w1,
                                      const float* w2, float* d_xd, float* d_gd, float* dw1, float* dw2,
                                      janus_ffn_mode mode, void* workspace, size_t workspace_bytes,
                                      janus_stream_t stream);

/* -------------------------------------------------------------------------
 * Expert-parallel exchange.  [Review] section 3.4 (FSEP: experts sharded over
 * ranks) and section 3.5 (the MoE all-to-all moves atom-type-aware FP16 rows,
 * half the FP32 volume).  P ranks, one process per GPU of a node; rank o owns
 * experts [o*E/P, (o+1)*E/P) (E a multiple of P, P <= JANUS_EP_MAX_RANKS).
 * Every rank calls janus_route on its own atoms; the counts of all ranks,
 * gathered in rank order into counts_all [P,E] (device int32), fix the layout:
 *   src_off [P,E+1]: src_off[s][e] = sum_{e'<e} counts_all[s][e'] (sender s's
 *                    local dispatch order; equals its janus_route offsets)
 *   recv_off [P,E/P+1]: owner o's rows per local expert, summed over senders
 *                    (o's receive buffer: grouped by local expert, then sender;
 *                    the expert MLP runs on recv_off[o] directly), each entry
 *                    clamped to recv_cap
 *   dst_off [P,E]:  dst_off[s][e] = (unclamped) rows of owner(e)'s local
 *                    experts before e + sum_{s'<s} counts_all[s'][e]
 * Row i of (s, e) moves from sender row src_off[s][e] + i to owner row
 * dst_off[s][e] + i, and back.
 *
 * Capacity: every rank's receive buffers hold recv_cap rows (the caller picks
 * it, e.g. a capacity factor times the fair share N*K; the worst case is
 * P*N*K).  A send whose owner row would be at or past recv_cap is skipped and
 * recorded as a data fault (JANUS_ERR_DATA from janus_check on the send's
 * workspace): no call ever stores past recv_cap, and the owner's kernels see
 * at most recv_cap rows.  The layer's output is then incomplete.
 *
 * The send and return calls store straight into the other ranks' buffers:
 * the pointer arrays (host arrays of P device pointers, index = rank) hold the
 * local buffer at this rank's index and peer-mapped buffers elsewhere
 * (janus_ipc_open_handle).  No call waits on another rank: a call's stores are
 * complete when its stream work is, and the caller orders the phases (a
 * collective barrier after each send/return, before the receiver reads).
 * Buffers are sized by the caller: a receive buffer holds at least the
 * owner's recv_off[o][E/P] rows (max_rows is its capacity); rows past the
 * received count are left untouched.  top_k <= 32 for the send calls.
 * ------------------------------------------------------------------------- */
#define JANUS_EP_MAX_RANKS 8

/* One CTA; writes src_off, dst_off, recv_off (device int32, layouts above)
 * for receive buffers of recv_cap rows (0 <= recv_cap < 2^31). */
janus_status janus_ep_layout(const int32_t* counts_all, int32_t world, int32_t n_experts,
                             int64_t recv_cap, int32_t* src_off, int32_t* dst_off, int32_t* recv_off,
                             janus_stream_t stream);

/* Forward send with the FP16 packing of janus_quant_by_type (this rank's
 * per-type power-of-two absmax scales, written to scale [T]): for each of
 * this rank's atoms i and k < K, with e = topk_expert[i*K+k] and
 * p = slot_of[i*K+k], owner o = e/(E/P), row r = dst_off[rank][e] + p -
 * src_off[rank][e]:  recv_payload[o][r,:] = fp16(x[i,:] / scale[types[i]]),
 * recv_scale[o][r] = scale[types[i]], for every r < recv_cap (the owner's
 * receive capacity, as given to janus_ep_layout).  recv_payload[o]: 8-byte
 * aligned.  workspace: janus_quant_by_type_workspace_size(n_types) bytes
 * (cleared by the call); bad type ids, non-finite rows and rows past recv_cap
 * are reported by janus_check. */
janus_status janus_ep_dispatch_quant(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                                     const int32_t* types, int32_t n_types, const int32_t* slot_of,
                                     const int32_t* topk_expert, const int32_t* src_off,
                                     const int32_t* dst_off, int32_t rank, int32_t world,
                                     int32_t n_experts, int64_t recv_cap, uint16_t* const* recv_payload,
                                     float* const* recv_scale, float* scale, void* workspace,
                                     size_t workspace_bytes, janus_stream_t stream);

/* FP32 send (the gradient direction): recv_rows[o][r,:] = w * x[i,:] with
 * w = topk_weight[i*K+k] (1 when topk_weight is NULL), same (o, r) as above,
 * r < recv_cap.  workspace: NULL, or a 256-byte aligned workspace whose error
 * word receives a row past recv_cap (it is not cleared by this call, so the
 * forward send's workspace can collect both directions). */
janus_status janus_ep_dispatch(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                               const int32_t* slot_of, const int32_t* topk_expert,
                               const float* topk_weight, const int32_t* src_off, const int32_t* dst_off,
                               int32_t rank, int32_t world, int32_t n_experts, int64_t recv_cap,
                               float* const* recv_rows, void* workspace, janus_stream_t stream);

/* Owner side of the FP16 send: xd[r,:] = f32(payload[r,:]) * row_scale[r] for
 * r < recv_off[rank][E/P] (read on the device; at most max_rows). */
janus_status janus_ep_dequant_rows(const uint16_t* payload, const float* row_scale, const int32_t* recv_off,
                                   int32_t rank, int32_t world, int32_t n_experts, int64_t max_rows,
                                   int32_t d, float* xd, janus_stream_t stream);

/* Owner side of the return: for each received row r (r < recv_off[rank][E/P],
 * at most max_rows) of sender s and expert e, ret_rows[s][src_off[s][e] + r -
 * dst_off[s][e], :] = yd[r,:].  The sender then runs janus_combine on its
 * return buffer as on a local expert output. */
janus_status janus_ep_return(const float* yd, const int32_t* counts_all, const int32_t* src_off,
                             const int32_t* dst_off, const int32_t* recv_off, int32_t rank, int32_t world,
                             int32_t n_experts, int64_t max_rows, int32_t d, float* const* ret_rows,
                             janus_stream_t stream);

/* The fused return: instead of copying yd, the owner's expert MLP stores each
 * output row straight into its sender's return buffer.  This call writes the
 * row table for janus_expert_ffn_fwd_rows / janus_expert_ffn_vjp_rows:
 * rows[r] = ret_rows[s] + (src_off[s][e] + r - dst_off[s][e]) * d for every
 * received row r (r < recv_off[rank][E/P], at most max_rows) of sender s and
 * expert e; rows[r] past the received count are left untouched.  rows: device
 * array of max_rows pointers, 8-byte aligned.  ret_rows: as in
 * janus_ep_return (16-byte aligned buffers).  The table depends only on the
 * layout, so one table serves the forward and the VJP of a layer pass. */
janus_status janus_ep_return_rows(const int32_t* src_off, const int32_t* dst_off, const int32_t* recv_off,
                                  int32_t rank, int32_t world, int32_t n_experts, int64_t max_rows, int32_t d,
                                  float* const* ret_rows, float** rows, janus_stream_t stream);

/* CUDA IPC, so ranks on one node can map each other's buffers.  A handle names
 * the allocation that holds dev_ptr plus dev_ptr's byte offset in it (callers
 * may pass pointers into a caching allocator's blocks).  Open returns the
 * mapped pointer with the offset applied; close takes that pointer and the
 * same offset.  Opening a handle in the process that created it fails. */
typedef struct {
  unsigned char bytes[64];
  uint64_t offset;
} janus_ipc_handle;
janus_status janus_ipc_get_handle(const void* dev_ptr, janus_ipc_handle* out);
janus_status janus_ipc_open_handle(const janus_ipc_handle* handle, void** dev_ptr);
janus_status janus_ipc_close_handle(void* dev_ptr, uint64_t offset);

/* -------------------------------------------------------------------------
 * Combine.  [Blueprint] section 3.2 (aggregation and output layer): the
 * activated experts' outputs are summed with the gate weights.  Gather form
 * of the weighted scatter-add (deterministic, no atomics):
 *   y[i,:] = sum_{k = 0..K-1, ascending} w[i,k] * yd[slot_of[i*K+k], :]
 * topk_weight == NULL means w = 1 (the VJP combine).
 * in : yd [R,d], slot_of [R], topk_weight [N,K] or NULL;  out: y [N,d]
 * ------------------------------------------------------------------------- */
janus_status janus_combine(const float* yd, const int32_t* slot_of, const float* topk_weight,
                           int64_t n_atoms, int32_t top_k, int32_t d, float* y,
                           janus_stream_t stream);

/* -------------------------------------------------------------------------
 * Edge -> atom aggregation.  [Review] section 3.5 (CNIS kernels: neighbour
 * aggregation with fused indexing, edge aggregation): edge messages are
 * reduced into their receiver atoms.  Segment sum over a receiver-sorted CSR:
 *   out[i,:] = sum_{e in [row_ptr[i], row_ptr[i+1])} msg[e,:]   (0 if empty)
 * in : msg [Ed,d] float32 with Ed = n_edges (NULL is accepted only when
 *      n_edges == 0), row_ptr [N+1] int64 (non-decreasing, row_ptr[N] -
 *      row_ptr[0] = n_edges);  out: out [N,d] float32.
 * Message row 0 is edge row_ptr[0] (0 for a whole CSR), so a range of
 * receivers [i0, i1) of a larger CSR is aggregated by passing row_ptr + i0,
 * N = i1 - i0 and the messages of edges [row_ptr[i0], row_ptr[i1]).
 * Every edge range is clamped to [0, n_edges], so a malformed row_ptr cannot
 * make the kernel read outside msg (the debug build also reports it through
 * janus_debug_check).  A NULL msg with n_edges > 0 is JANUS_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------- */
janus_status janus_edge_aggregate(const float* msg, int64_t n_edges, const int64_t* row_ptr,
                                  int64_t n_atoms, int32_t d, float* out, janus_stream_t stream);

/* Gradient of the edge aggregation (same passage): every edge of receiver i
 * receives that atom's gradient row,  dmsg[e,:] = dx[i,:]  for e in
 * [row_ptr[i], row_ptr[i+1]).  in : dx [N,d], row_ptr [N+1];  out: dmsg
 * [Ed,d] with Ed = n_edges (NULL accepted only when n_edges == 0; a NULL dmsg
 * with n_edges > 0 is JANUS_ERR_INVALID_ARG).  As in janus_edge_aggregate,
 * dmsg row 0 is edge row_ptr[0] and edge ranges are clamped to [0, n_edges]. */
janus_status janus_edge_broadcast(const float* dx, const int64_t* row_ptr, int64_t n_atoms,
                                  int32_t d, float* dmsg, int64_t n_edges, janus_stream_t stream);

/* Neighbour aggregation with fused indexing ([Review] section 3.5, CNIS
 * kernels): node features are gathered through the sender index instead of a
 * materialised message buffer,
 *   out[i,:] = sum_{e in [row_ptr[i], row_ptr[i+1])} x[senders[e], :]
 * in : x [N,d] float32, row_ptr [N+1] int64, senders [Ed] int32 with Ed =
 * n_edges (NULL accepted only when n_edges == 0; a NULL senders with
 * n_edges > 0 is JANUS_ERR_INVALID_ARG);  out: out [N,d].  Sender ids outside
 * [0,N) are skipped (they add nothing; the debug build reports them).  As in
 * janus_edge_aggregate, senders[0] is edge row_ptr[0] and edge ranges are
 * clamped to [0, n_edges].  N < 2^31. */
janus_status janus_neighbor_aggregate(const float* x, const int64_t* row_ptr, const int32_t* senders,
                                      int64_t n_edges, int64_t n_atoms, int32_t d, float* out,
                                      janus_stream_t stream);

/* -------------------------------------------------------------------------
 * Debug build.  The library built with -DJANUS_DEBUG (libjanus_debug.so)
 * checks, on the device and before using them, the index arrays that calls
 * take as input: slot_of and perm in [0, R), offsets non-decreasing from 0
 * with offsets[E] <= R, row_ptr non-decreasing inside [0, n_edges], senders in
 * [0, N), and the expert-parallel tables.  A kernel that finds a bad index
 * records a data fault and skips that access, so a corrupted index array
 * cannot make it read or write outside its buffers.  Calls with a workspace
 * record the fault there (janus_check); calls without one record it in the
 * library's per-GPU debug fault word, which janus_debug_check reads.  Both
 * builds export the same symbols; the release build records nothing in the
 * debug word.
 * ------------------------------------------------------------------------- */

/* 1 for the debug build, 0 for the release build. */
int32_t janus_debug_build(void);

/* Synchronises `stream`, then reads and clears the debug fault word of the
 * current device.  JANUS_ERR_DATA if a call without a workspace found a bad
 * index since the last check, else JANUS_OK (always JANUS_OK in the release
 * build); JANUS_ERR_CUDA if a CUDA call failed. */
janus_status janus_debug_check(janus_stream_t stream);

/* Launch trace, for measuring the kernels inside a call.  janus_trace_start
 * creates `capacity` pairs of CUDA events on the current device (1 <= capacity
 * <= 2^20; any earlier records are dropped) and starts recording: from then on
 * each traced launch of this library (the expert MLP's tensor-core GEMMs, its
 * weight and activation splits) is bracketed by two events recorded on the
 * launch's stream, until janus_trace_stop or until `capacity` launches have
 * been recorded.  janus_trace_count gives the number of records;
 * janus_trace_get(i) waits for record i's end event and returns its kernel's
 * name (a static string owned by the library) and its duration in ms.
 * janus_trace_release stops recording and destroys the events.  The trace is
 * process-wide; one device at a time.  JANUS_ERR_CUDA if an event cannot be
 * created or read; JANUS_ERR_INVALID_ARG for a bad capacity or index. */
janus_status janus_trace_start(int32_t capacity);
janus_status janus_trace_stop(void);
janus_status janus_trace_count(int32_t* n);
janus_status janus_trace_get(int32_t i, const char** name, float* ms);
janus_status janus_trace_release(void);

/* Host-side fault injection for tests: the next `n_calls` library calls that
 * would launch work return JANUS_ERR_CUDA before launching anything. */
void janus_debug_inject_launch_failures(int32_t n_calls);

#ifdef __cplusplus
}
#endif

#endif /* JANUS_H_ */
