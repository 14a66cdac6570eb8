// Grouped expert-MLP GEMM on the 5th-generation tensor cores (tcgen05), for
// JANUS_FFN_3XTF32: the 3xTF32 split on kind::tf32, and (kBF16W / kBF16S
// below) an FP16 form on kind::f16 for rows that arrive as FP16 values or as
// two FP16 terms: the FP16-packed dispatch, the split dispatch and the
// activations' row split (act_split_blk_kernel below).
//
// FP32 accuracy from TF32 tensor cores (Ootomo & Yokota 2022, "Recovering
// single precision accuracy from Tensor Cores while surpassing the FP32
// theoretical peak performance"): every FP32 operand x is split into
//   hi = x truncated to TF32 (10 fraction bits), lo = x - hi (exact in FP32),
// and a*b is accumulated as a_lo*b_hi + a_hi*b_lo + a_hi*b_hi; the dropped
// a_lo*b_lo term is below 2^-20 of the product.  The tensor core adds into its
// FP32 accumulator with truncation, so a long reduction drifts (about 2e-5
// relative at K = 2560 when accumulated in one pass).  As in the same paper,
// accumulation is therefore split: each chunk of 16 k-blocks (K = 256) is
// accumulated from zero in TMEM and then added, with round-to-nearest FP32
// adds, into running sums held in the epilogue warps' registers.  (Error
// through the MLP's two GEMMs at K = 2560, measured: 2.6e-6 with K = 128
// chunks, 4.4e-6 with K = 256, 8.1e-6 with K = 512; K = 256 chunks halve the
// hand-offs and run 4-12 % faster than K = 128.)
//
// Three operand layouts share the kernel:
//   x W   (forward)  and  x W^T (input VJP) run swapped, C^T = W^T X^T: the
//         MMA's A is the expert's weights (128 output features per CTA, so
//         M = 256 per pair is always full) and its B is the tile's dispatch
//         rows (N = the valid rows rounded up to 32, half of them per CTA), so
//         a Zipf-small expert pads at most 31 rows;
//   X^T Y (weight gradients) runs direct, both operands MN-major, K = the
//         expert's rows.
// Structure: one persistent CTA per SM, clusters of two CTAs sharing each
// output tile through tcgen05 cta_group::2 MMAs (each CTA holds its 128 rows
// of A, its half of B and its 128 accumulator lanes, so shared-memory traffic
// per CTA is a third lower than with 1-CTA MMAs).  16 warps:
//   warp 0       TMA producer: this CTA's A and B tiles per 16-wide k-block
//                into a 6-stage ring (32 KB per stage: raw + lo; 64-byte
//                swizzle for K-major, 128-byte swizzle with 32-byte atoms for
//                MN-major operands);
//   warp 1       TMEM allocator (paired) and, in the leader CTA, the MMA
//                issuer: 3 products x 2 k-steps of tcgen05.mma.cta_group::2
//                .kind::tf32 per k-block into one of two 256-column TMEM chunk
//                buffers, commits signalling both CTAs; the peer's splitters
//                and epilogues arrive on the leader's barriers;
//   warps 2,3,12..15  splitters, each owning every sixth k-block: write the
//                landed tile's residual lo = x - hi into a twin buffer (same
//                swizzled offsets; the landed FP32 tile is read by the MMA as hi);
//                when the rows are dequantized FP16 values (exact in TF32,
//                kBExact) only the weights are split, the rows are only
//                checked, and the product with the rows' zero residual is
//                not issued;
//   warps 4..11  epilogue (two warpgroups, one half of the tile each):
//                tcgen05.ld of each chunk, FP32 running sums in registers
//                (setmaxnreg: 184 per thread here, 72 elsewhere), then the
//                fused epilogue: SiLU (a and silu(a)), SiLU' (pre-activation
//                reads pipelined and prefetched to L2), the second-order
//                silu'/silu'' terms, a plain store, or an accumulating store.
// Tiles come from per-expert block counts built on the device from `offsets`
// (expert, then 256-row block, then 256-feature block), so the host never
// reads the routing.  Every mbarrier wait is bounded: on timeout the CTA
// records an error in the workspace header, every role leaves its loop,
// issued MMAs and loads are drained (bounded) and TMEM is freed.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>
#include <string>

#include "ffn_tc.cuh"

namespace janus {
namespace tc {
namespace {

// A CTA pair (cluster of 2) computes a 256 x 256 output tile with M = 256
// MMAs (tcgen05 cta_group::2): each CTA holds its own 128 rows of A, half of
// the 256 B columns, and its 128 rows of the accumulator in its own TMEM.
constexpr int BM = 128, BN = 256, BK = 16;
constexpr int BNH = BN / 2;               // B columns held by one CTA
constexpr int kStages = 6;
constexpr int kThreads = 512;
constexpr int kNumSplitWarps = 6;
// Splitter warp i splits every k-block with (k-block index) % kNumSplitWarps
// == i, i.e. always the same stages.  That is what makes its parity wait on a
// stage's `full` barrier safe: a parity wait cannot tell the phase it wants
// from the one two phases later, so each stage's consecutive uses must be
// waited for by one warp, in order.  (A 7-stage ring with 6 splitters, where
// uses rotate between warps, split tiles before they had landed.)
static_assert(kStages % kNumSplitWarps == 0, "every stage is split by one fixed warp");
constexpr int kNumEpiWarps = 8;
constexpr int kEpiCols = BN / 2;         // columns per epilogue thread
constexpr int kChunkKb = 256 / BK;       // k-blocks accumulated per TMEM chunk (K = 256)
constexpr int kEpiRegs = 184, kOtherRegs = 72;
static_assert(2 * 128 * kEpiRegs + 2 * 128 * kOtherRegs == 65536, "register split must match the launch");
constexpr uint32_t kTileABytes = BM * BK * 4;              // 8 KB
constexpr uint32_t kTileBBytes = BNH * BK * 4;             // 8 KB (this CTA's half)
constexpr uint32_t kStageBytes = 2 * (kTileABytes + kTileBBytes);   // raw + lo
constexpr uint32_t kTxBytes = kTileABytes + kTileBBytes;
constexpr uint32_t kTmemCols = 512;
constexpr long long kWaitLimitCycles = 4000000000LL;     // ~2 s at 2 GHz

// kEpiD2 (second-order pass, x·W): acc = v W1, aux = a, aux2 = dh;
//   C = acc silu'(a), C2 = acc dh silu''(a), C3 = dh silu'(a) (if C3).
// kEpiAccum (weight-gradient layout only): C += acc.
enum Epilogue : int { kEpiStore = 0, kEpiSilu = 1, kEpiDSilu = 2, kEpiD2 = 3, kEpiAccum = 4 };

// Operand layouts:  kModeNN  C = X W       (W stored [E][Kd][N])
//                   kModeNT  C = X W^T     (W stored [E][N][Kd])
//                   kModeTN  C_e = (X_e^T Y_e)^T = Y_e^T X_e per expert (weight
//                            gradient; both operands MN-major, K = the expert's
//                            row segment; the X^T Y product is stored transposed)
// NN and NT run with the operands swapped (C^T = W^T X^T): the MMA's M is the
// output feature (256 per CTA pair: the weights fill it without padding) and
// its N is the expert's rows, chosen per tile as the valid rows rounded up to
// 32, so a small expert wastes at most 31 rows instead of up to 255.
enum Mode : int { kModeNN = 0, kModeNT = 1, kModeTN = 2 };

// What the B tile (the dispatch rows, kModeNN) holds:
//   kBSplit   FP32 rows, split into hi and lo by the splitters (3 products);
//   kBExact   FP32 rows exact in TF32 (dequantized FP16): no lo, 2 products,
//             the splitters only check the rows;
//   kBF16W    the FP16 payload against an FP16 split of the weights, on the
//             kind::f16 tensor path (below): no splitter work, 2 products;
//   kBF16S    FP32 rows given as two FP16 terms (hi and mid planes of a
//             [2R][Kd] tensor, from janus_dispatch_split) with a per-row
//             power-of-two scale, against the FP16 split of the weights:
//             3 products, hi.hi + hi.mid + mid.hi (mid.mid, below 2^-22 of
//             the product, is dropped as in 3xTF32).
enum BKind : int { kBSplit = 0, kBExact = 1, kBF16W = 3, kBF16S = 4 };

// kBF16W: FP16 rows x FP16-split weights on tcgen05 kind::f16.
// A packed row is q * s (q binary16, s a power of two), exact in FP16 up to
// its scale.  Each weight column f of expert e is scaled, per K chunk c of
// 256, by a power of two S_fc that puts the chunk's largest magnitude in
// [2^14, 2^15) and split into two FP16 terms, w S_fc = hi + mid + r with
// |r| <= 2^-22 |w S_fc| (the split the weight kernels below write).  The
// tensor core multiplies FP16 operands exactly and accumulates each chunk in
// FP32, and the epilogue scales each chunk's sum as it folds it, so
//   a[p, f] = s_p * sum_c (1 / S_fc) sum_{k in c} q[p, k] (hi[f, k] + mid[f, k])
// is as accurate as the 3xTF32 product, with two kind::f16 MMAs per 16-wide
// k-step (a kind::f16 MMA covers twice the K of a TF32 one in the same time).
// Both operands are K-major FP16 tiles with the 128-byte swizzle: a k-block is
// 64 wide (128 bytes per row), a stage holds the weights' hi and mid tiles and
// this CTA's rows (3 x 16 KB), 4 stages.
constexpr int BK16 = 64;
constexpr int kStages16 = 4, kStages16S = 3;
constexpr uint32_t kTile16Bytes = BM * BK16 * 2;          // 16 KB: 128 rows x 128 bytes
constexpr uint32_t kStage16Bytes = 3 * kTile16Bytes;      // A hi | A mid | B
constexpr uint32_t kStage16SBytes = 4 * kTile16Bytes;     // A hi | A mid | B hi | B mid
static_assert(kStages16 * kStage16Bytes <= kStages * kStageBytes, "the FP16 ring fits the same shared memory");
static_assert(kStages16S * kStage16SBytes <= kStages * kStageBytes, "the FP16 ring fits the same shared memory");
static_assert(kStages16 <= kNumSplitWarps && kStages16S <= kNumSplitWarps, "one relay warp per FP16 stage");
template <int kBK> __host__ __device__ constexpr bool f16_path() { return kBK == kBF16W || kBK == kBF16S; }
template <int kBK> __host__ __device__ constexpr int ring_stages() {
  return kBK == kBF16W ? kStages16 : (kBK == kBF16S ? kStages16S : kStages);
}
template <int kBK> __host__ __device__ constexpr uint32_t ring_stage_bytes() {
  return kBK == kBF16W ? kStage16Bytes : (kBK == kBF16S ? kStage16SBytes : kStageBytes);
}
template <int kBK> __host__ __device__ constexpr int kblock_width() { return f16_path<kBK>() ? BK16 : BK; }
// k-blocks per TMEM chunk (K = 256 in both geometries)
template <int kBK> __host__ __device__ constexpr int chunk_kblocks() { return 256 / kblock_width<kBK>(); }

struct Args {
  float* C;
  float* C2;
  float* C3;
  const float* aux;
  const float* aux2;
  float* const* c_rows;   // NN/NT plain store: if set, row p goes to c_rows[p] (e.g. a peer's buffer)
  const float* row_scale; // kBF16W, kBF16S: scale of dispatch row p
  const float* col_scale; // kBF16W, kBF16S: 1 / S of output feature f of expert e, [E][N]
  int64_t rows;           // rows of the dispatch operand; offsets[E] <= rows
  const int32_t* offsets;
  int E, Kd, N;
  int M;            // kModeTN: MMA rows of each expert's product; C is [E][N][M] (stored transposed)
  int32_t* err;
};

struct Smem {
  uint64_t full[kStages];     // this CTA's TMA landed (tx count)
  uint64_t split[kStages];    // leader: residuals written in both CTAs (1 warp x 2)
  uint64_t empty[kStages];    // MMAs done reading the stage (commit to both CTAs)
  uint64_t chunk_full[2];     // a k-chunk's partial product is in TMEM (commit to both)
  uint64_t chunk_empty[2];    // leader: both epilogues folded that chunk (8 warps x 2)
  uint64_t drain;             // final commit (both CTAs) before TMEM is freed
  uint32_t tmem_base;
  int abort;
  int off[kMaxExperts + 1];
  int start[kMaxExperts + 1];
};

// ---- PTX wrappers ---------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false if the CTA aborted or the wait ran out (then aborts it).
__device__ __forceinline__ bool mbar_wait(Smem* s, uint64_t* bar, uint32_t parity, int32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*(volatile int*)&s->abort) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *(volatile int*)&s->abort = 1;
      atomicCAS(err, 0, kFaultTimeout);
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(const CUtensorMap* map, uint64_t* bar, void* dst, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on the barrier at the same shared-memory offset in the leader CTA of
// the pair: a plain local arrive in the leader itself, a remote arrive (default
// release semantics) from the peer.  The data behind these arrivals is read
// by the arriving CTA's own tensor core, so a cluster-scope release (about a
// thousand cycles per arrive on B200) is not needed.
__device__ __forceinline__ void mbar_arrive_leader(uint64_t* bar, uint32_t rank) {
  if (rank == 0) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
  } else {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(bar)), "r"(0));
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
  }
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// completion of the pair's MMAs arrives on the barrier at this offset in both CTAs
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      ::"r"(smem_u32(bar)), "h"((uint16_t)0x3)
      : "memory");
}
// A-operand collector use of an MMA: kCollNone reads A from shared memory;
// kCollFill reads it and keeps it in the tensor core's A collector;
// kCollLast takes A from the collector (filled by the MMA just before, with
// the same A descriptor) instead of shared memory, and releases it.  Two
// consecutive products with the same A (hi_w x hi_x, hi_w x lo_x) then fetch
// the weights' tile once, which matters where operand fetch, not the MMA
// rate, bounds a tile (few dispatch rows).
enum Collector : int { kCollNone = 0, kCollFill = 1, kCollLast = 2 };

template <int kColl = kCollNone>
__device__ __forceinline__ void tc_mma_tf32_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  if (kColl == kCollFill)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32.collector::a::fill [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else if (kColl == kCollLast)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32.collector::a::lastuse [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int kColl = kCollNone>
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  if (kColl == kCollFill)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16.collector::a::fill [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else if (kColl == kCollLast)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16.collector::a::lastuse [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets (16-byte units), version 1, swizzle mode.
// K-major operands use the 128-byte swizzle (mode 2; 16-byte granules XOR the
// row mod 8).  An MN-major TF32 operand must use the 128-byte swizzle with
// 32-byte atoms (mode 1; 32-byte granules XOR the row mod 4), which TMA writes
// with CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B.
constexpr uint32_t kSwizzle64B = 4, kSwizzle128B32B = 1, kSwizzle128B = 2;
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t mode) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)mode << 61;
  return d;
}

// Instruction descriptor: D=F32, A=B=TF32, A and B K- or MN-major,
// M=256 (the CTA pair), N=256.
__host__ __device__ constexpr uint32_t instr_desc(bool a_mn_major, bool b_mn_major, uint32_t n = BN) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((n >> 3) << 17) | ((uint32_t)((2 * BM) >> 4) << 24);
}

// kind::f16 instruction descriptor: D=F32, A=B=F16 (format 0), both K-major,
// M=256 (the CTA pair), N = n.
__host__ __device__ constexpr uint32_t instr_desc_f16(uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((uint32_t)((2 * BM) >> 4) << 24);
}

// Epilogue activations.  The store phase is unrolled over 128 columns per
// thread, so every instruction here is repeated 128 times in the kernel's code;
// a long sequence (an accurate expf plus an IEEE divide, twice) overflows the
// instruction cache and stalls the MMA-issuing warp with it.  The sigmoid is
// therefore computed once per element with the fast exponential and divide
// (relative error a few 1e-7 against ~1e-6 from the 3xTF32 products).
__device__ __forceinline__ float sigmoid_fast(float a) { return __fdividef(1.0f, 1.0f + __expf(-a)); }
__device__ __forceinline__ float silu_f(float a) { return a * sigmoid_fast(a); }

// TF32 high part: the FP32 value with its 13 low fraction bits cleared (exact
// for every input, no overflow); the residual x - hi is exact in FP32.
// tcgen05.mma.kind::tf32 reads a 32-bit operand by ignoring those same 13
// bits (checked on B200: results are bit-identical to feeding it the cleared
// value), so the landed FP32 tile serves as the high part unchanged and only
// the residual tile is written.
constexpr uint32_t kTf32Mask = 0xFFFFE000u;

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct TileCoord {
  int e;
  int m0, m_end;    // MMA M: this CTA's first row (TN: output row; NN/NT: output feature) and bound
  int n0;           // MMA N: TN: first output column; NN/NT: first dispatch row of the tile
  int n_valid;      // NN/NT: valid rows in the tile
  int n_mma;        // the MMA's N for this tile
  int k_row0;       // kModeTN: first row of the expert's segment (the K range)
  int k_rows;       // kModeTN: rows in the segment
  int nk;           // k-blocks of this tile
};

// Pair tile `tile` -> expert, this CTA's 128-row block and the 256-column block.
//   kModeNN/NT: start[e] counts 256-row blocks of expert e's row segment.
//   kModeTN:    every expert has ceil(M/256) row blocks of its [M x N] output.
template <int kMode>
__device__ __forceinline__ TileCoord decode_tile(const Smem* s, const Args& args, int n_tiles_n, int nk_fixed,
                                                 int tile, uint32_t rank) {
  TileCoord c;
  const int mt = tile / n_tiles_n, nt = tile % n_tiles_n;
  if (kMode == kModeTN) {
    const int n_mp = (args.M + 2 * BM - 1) / (2 * BM);
    c.e = mt / n_mp;
    c.m0 = ((mt % n_mp) * 2 + (int)rank) * BM;
    c.m_end = args.M;
    c.n0 = nt * BN;
    c.n_valid = min(BN, args.N - c.n0);
    c.n_mma = BN;
    c.k_row0 = s->off[c.e];
    c.k_rows = s->off[c.e + 1] - c.k_row0;
    c.nk = (c.k_rows + BK - 1) / BK;
  } else {
    // mt: 256-row block of the expert's segment; nt: 256-feature block
    int lo = 0, hi = args.E;   // start[lo] <= mt < start[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s->start[mid] <= mt) lo = mid; else hi = mid;
    }
    c.e = lo;
    c.n0 = s->off[lo] + (mt - s->start[lo]) * (2 * BM);
    c.n_valid = min(2 * BM, s->off[lo + 1] - c.n0);
    c.n_mma = (c.n_valid + 31) & ~31;
    c.m0 = nt * BN + (int)rank * BNH;
    c.m_end = args.N;
    c.k_row0 = 0;
    c.k_rows = 0;
    c.nk = nk_fixed;
  }
  return c;
}

// Second-order epilogue for one thread's 128 columns (swapped layout: output
// feature f of dispatch rows n0 + j0 + j), 4 columns per batch with both
// inputs loaded before use.
__device__ __forceinline__ void d2_store(const Args& args, const float (&acc)[kEpiCols], const TileCoord& c,
                                         int j0, int f, int N) {
  constexpr int kB = 4;
#pragma unroll
  for (int jb = 0; jb < kEpiCols; jb += kB) {
    float a[kB], g[kB];
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const bool ok = j0 + jb + j < c.n_valid;
      const int64_t o = (int64_t)(c.n0 + j0 + jb + j) * N + f;
      a[j] = ok ? __ldg(args.aux + o) : 0.f;
      g[j] = ok ? __ldg(args.aux2 + o) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      if (j0 + jb + j < c.n_valid) {
        const int64_t o = (int64_t)(c.n0 + j0 + jb + j) * N + f;
        // silu'(a) = s (1 + a (1 - s)), silu''(a) = s (1 - s) (2 + a (1 - 2 s))
        const float sg = sigmoid_fast(a[j]);
        const float s1 = sg * (1.0f + a[j] * (1.0f - sg));
        const float s2 = sg * (1.0f - sg) * (2.0f + a[j] * (1.0f - 2.0f * sg));
        args.C[o] = acc[jb + j] * s1;
        args.C2[o] = acc[jb + j] * g[j] * s2;
        if (args.C3) args.C3[o] = g[j] * s1;
      }
    }
  }
}

// Epilogue warpgroups: fold each TMEM chunk into FP32 running sums, then apply
// the fused epilogue and store this CTA's 128 x 256 part of the tile.
template <int kMode, int kEpi, int kBK>
__device__ __forceinline__ void epilogue_role(Smem* s, const Args& args, uint32_t tmem_base, int warp, int lane,
                                              int n_tiles_n, int total, int nk_fixed, uint32_t rank, int n_pairs) {
  constexpr int kChunk = chunk_kblocks<kBK>();
  const int wg = warp / 4;
  const int N = args.N;
  const int q = warp % 4;                  // TMEM lane quarter = 32 rows
  const int half = wg - 1;                 // columns [128*half, 128*half + 128)
  const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
  uint32_t ch = 0;
  for (int tile = blockIdx.x / 2; tile < total; tile += n_pairs) {
    const TileCoord c = decode_tile<kMode>(s, args, n_tiles_n, nk_fixed, tile, rank);
    float acc[kEpiCols];
#pragma unroll
    for (int j = 0; j < kEpiCols; ++j) acc[j] = 0.f;     // a tile with no k-blocks stores zeros
    // FP16 path: this half-tile's 128 row scales, four per lane, loaded while
    // the tile accumulates; the store phase takes column j's from lane j % 32
    // by a shuffle instead of a load per column (the dSiLU store phase, short
    // of registers for them, loads each column's)
    constexpr bool kShflScale = f16_path<kBK>() && kMode != kModeTN && kEpi != kEpiDSilu;
    float rsr[kEpiCols / 32];
#pragma unroll
    for (int u = 0; u < kEpiCols / 32; ++u) {
      const int col = (wg - 1) * kEpiCols + u * 32 + lane;
      rsr[u] = (kShflScale && col < c.n_valid) ? __ldg(args.row_scale + c.n0 + col) : 0.f;
    }
    bool ok = true;
    for (int c0 = 0; c0 < c.nk; c0 += kChunk, ++ch) {
      const uint32_t p = ch & 1, cuse = ch >> 1;
      // FP16 path: the weights' 1 / S for this lane's feature and this K
      // chunk (the split scales each feature per chunk of 256), loaded before
      // the wait; the chunk's sum is scaled by it as it is folded (exact)
      float wsc = 1.0f;
      if (f16_path<kBK>()) {
        const int f = c.m0 + q * 32 + lane;
        const int nch = (args.Kd + 255) / 256;
        wsc = f < c.m_end ? __ldg(args.col_scale + ((int64_t)c.e * nch + c0 / kChunk) * N + f) : 0.f;
      }
      // the warp leaves together (a timeout seen by one lane ends the tile for
      // all 32: the TMEM loads and the row-scale shuffles are warp-wide)
      if (!__all_sync(0xffffffffu, mbar_wait(s, &s->chunk_full[p], cuse & 1, args.err))) { ok = false; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + lane_addr + p * BN + half * kEpiCols;
#pragma unroll
      for (int j = 0; j < kEpiCols; j += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + j, r);
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          if (f16_path<kBK>())
            acc[j + t] = fmaf(__uint_as_float(r[t]), wsc, acc[j + t]);
          else
            acc[j + t] += __uint_as_float(r[t]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader(&s->chunk_empty[p], rank);
      // the tile's pre-activations travel to L2 while its last two chunks
      // accumulate (late enough that they are still there for the store
      // phase: 1-3 % faster than prefetching at the first chunk)
      const int pf_c0 = max(0, ((c.nk - 1) / kChunk - 1) * kChunk);
      if (kMode != kModeTN && (kEpi == kEpiDSilu || kEpi == kEpiD2) && c0 == pf_c0) {
        const int f = c.m0 + q * 32 + lane;
        const int jn = min(kEpiCols, c.n_valid - half * kEpiCols);
        if (f < c.m_end) {
#pragma unroll 1
          for (int j = 0; j < jn; ++j) {
            const int64_t o = (int64_t)(c.n0 + half * kEpiCols + j) * N + f;
            asm volatile("prefetch.global.L2 [%0];" ::"l"(args.aux + o));
            if (kEpi == kEpiD2) asm volatile("prefetch.global.L2 [%0];" ::"l"(args.aux2 + o));
          }
        }
      }
    }
    if (!ok) break;
    if (kMode != kModeTN) {
      // TMEM lane = output feature, column = dispatch row: for one row the 32
      // lanes of a warp write 32 consecutive features (128-byte stores)
      const int f = c.m0 + q * 32 + lane;
      const int j0 = half * kEpiCols;
      if (kEpi == kEpiD2) {
        if (f < c.m_end) d2_store(args, acc, c, j0, f, N);
        continue;
      }
      // with the row-scale shuffles every lane runs the loop (they need the
      // whole warp); lanes past the tile's last feature store nothing
      const bool f_ok = f < c.m_end;
      if (kShflScale || f_ok) {
        // FP16 path: the product is q (hi + mid) S (kBF16S: q = the row's
        // two terms); the sums already carry the weights' 1 / S (folded per
        // chunk); scale column j by its row's s_p (a power of two: exact)
        // batches of 8 columns; the pre-activations of batch b + 1 are in
        // flight while batch b is finished, so two loads per column overlap
        constexpr int kB = 8;
        const float* arow = args.aux + (int64_t)(c.n0 + j0) * N + f;
        float a_cur[kB], a_nxt[kB];
        if (kEpi == kEpiDSilu) {
#pragma unroll
          for (int j = 0; j < kB; ++j) a_cur[j] = (f_ok && j0 + j < c.n_valid) ? __ldg(arow + (int64_t)j * N) : 0.f;
        }
#pragma unroll
        for (int jb = 0; jb < kEpiCols; jb += kB) {
          if (kEpi == kEpiDSilu && jb + kB < kEpiCols) {
#pragma unroll
            for (int j = 0; j < kB; ++j)
              a_nxt[j] = (f_ok && j0 + jb + kB + j < c.n_valid) ? __ldg(arow + (int64_t)(jb + kB + j) * N) : 0.f;
          }
#pragma unroll
          for (int j = 0; j < kB; ++j) {
            const float rs = kShflScale ? __shfl_sync(0xffffffffu, rsr[(jb + j) / 32], (jb + j) % 32) : 1.0f;
            if (f_ok && j0 + jb + j < c.n_valid) {
              const int64_t o = (int64_t)(c.n0 + j0 + jb + j) * N + f;
              float v = acc[jb + j];
              if (kShflScale) v = v * rs;
              else if (f16_path<kBK>()) v = v * __ldg(args.row_scale + c.n0 + j0 + jb + j);
              if (kEpi == kEpiStore && args.c_rows) {   // the row's own destination
                args.c_rows[c.n0 + j0 + jb + j][f] = v;
                continue;
              }
              if (kEpi == kEpiSilu) {
                if (args.C2) args.C2[o] = v;
                v = silu_f(v);
              } else if (kEpi == kEpiDSilu) {
                // silu'(a) = s (1 + a (1 - s)), s = sigmoid(a); C2 = silu(a) = a s
                const float a = a_cur[j];
                const float sg = sigmoid_fast(a);
                v *= sg * (1.0f + a * (1.0f - sg));
                if (args.C2) args.C2[o] = a * sg;
              }
              args.C[o] = v;
            }
          }
          if (kEpi == kEpiDSilu) {
#pragma unroll
            for (int j = 0; j < kB; ++j) a_cur[j] = a_nxt[j];
          }
        }
      }
      continue;
    }
    // weight gradient: TMEM lane = MMA row i (< M), column = j (< N).  The
    // product is stored transposed, C[e][j][i], so the 32 lanes of a warp
    // write 32 consecutive floats (one 128-byte segment) of one output row per
    // instruction; row-per-lane float4 stores touched 32 rows per instruction
    // and bound the short-K tiles of small experts.
    static_assert(kMode != kModeTN || kEpi == kEpiStore || kEpi == kEpiAccum,
                  "the weight-gradient GEMM has no fused activation");
    const int row = c.m0 + q * 32 + lane;
    const int colb = c.n0 + half * kEpiCols;
    if (row < c.m_end && colb < N) {
      float* base = args.C + (int64_t)c.e * args.M * N + (int64_t)colb * args.M + row;
      constexpr int kB = 8;
#pragma unroll
      for (int jb = 0; jb < kEpiCols; jb += kB) {
        float old[kB];
        if (kEpi == kEpiAccum) {
#pragma unroll
          for (int j = 0; j < kB; ++j) old[j] = colb + jb + j < N ? base[(int64_t)(jb + j) * args.M] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < kB; ++j)
          if (colb + jb + j < N) base[(int64_t)(jb + j) * args.M] = kEpi == kEpiAccum ? old[j] + acc[jb + j] : acc[jb + j];
      }
    }
  }
  // rows stored through c_rows may sit in another GPU's memory: make them
  // visible system-wide before the kernel completes
  if (kEpi == kEpiStore && args.c_rows) __threadfence_system();
}

template <int kMode, int kEpi, int kBK>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB, Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Smem* s = (Smem*)(tiles + kStages * kStageBytes);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int wg = warp / 4;
  const uint32_t rank = cluster_rank();       // 0 = leader (issues the MMAs)
  const int n_pairs = gridDim.x / 2;
  const int E = args.E, Kd = args.Kd, N = args.N;

  for (int e = tid; e <= E; e += kThreads) s->off[e] = args.offsets[e];
  if (tid == 0) {
    s->abort = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s->full[i], 1);
      mbar_init(&s->split[i], 2);   // one splitter warp per CTA per stage
      mbar_init(&s->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s->chunk_full[i], 1);
      mbar_init(&s->chunk_empty[i], 2 * kNumEpiWarps);
    }
    mbar_init(&s->drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    // the pair's TMEM: same column range in both CTAs
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s->tmem_base)),
                 "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  if (tid == 0) {
    if (kDebug) {
      // offsets must be non-decreasing inside [0, rows]; otherwise every
      // expert is treated as empty (no tile touches memory) and the fault recorded
      bool ok = s->off[0] >= 0 && s->off[E] <= args.rows;
      for (int e = 0; e < E; ++e) ok = ok && s->off[e + 1] >= s->off[e];
      if (!ok) {
        debug_fault(args.err);
        for (int e = 0; e <= E; ++e) s->off[e] = 0;
      }
    }
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      s->start[e] = acc;
      acc += kMode == kModeTN ? (args.M + 2 * BM - 1) / (2 * BM)
                              : (s->off[e + 1] - s->off[e] + 2 * BM - 1) / (2 * BM);
    }
    s->start[E] = acc;
  }
  // both CTAs' barriers are initialised before any remote arrive
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = s->tmem_base;
  const int n_tiles_n = (N + BN - 1) / BN;
  const int total = s->start[E] * n_tiles_n;
  constexpr int kRing = ring_stages<kBK>();
  constexpr uint32_t kRingBytes = ring_stage_bytes<kBK>();
  constexpr int kKb = kblock_width<kBK>();
  constexpr int kChunk = chunk_kblocks<kBK>();
  const int nk = (Kd + kKb - 1) / kKb;

  if (wg == 1 || wg == 2) {
    // the epilogue warpgroups hold 128 FP32 running sums per thread
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpiRegs));
    epilogue_role<kMode, kEpi, kBK>(s, args, tmem_base, warp, lane, n_tiles_n, total, nk, rank, n_pairs);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
    if (warp == 0) {
      // ---------------- TMA producer (each CTA loads its own A rows and B half) ----------------
      if (lane == 0) {
        uint32_t it = 0;
        bool ok = true;
        for (int tile = blockIdx.x / 2; tile < total && ok; tile += n_pairs) {
          const TileCoord c = decode_tile<kMode>(s, args, n_tiles_n, nk, tile, rank);
          const int nb = c.n0 + (int)rank * BNH;   // kModeTN: this CTA's B columns
          for (int kb = 0; kb < c.nk; ++kb, ++it) {
            const uint32_t st = it % kRing, use = it / kRing;
            if (!mbar_wait(s, &s->empty[st], (use & 1) ^ 1, args.err)) { ok = false; break; }
            uint8_t* base = tiles + st * kRingBytes;
            if (f16_path<kBK>()) {
              // the weights' hi and mid tiles (expert e and E + e of the split
              // tensor) and this CTA's rows (kBF16S: their hi and mid planes,
              // rows r and R + r), 64 k wide, 128-byte swizzle
              const int row = c.n0 + (int)rank * (c.n_mma / 2);
              mbar_arrive_expect_tx(&s->full[st], kRingBytes);
              tma_load_3d(&mapA, &s->full[st], base, kb * BK16, c.m0, c.e);
              tma_load_3d(&mapA, &s->full[st], base + kTile16Bytes, kb * BK16, c.m0, E + c.e);
              tma_load_2d(&mapB, &s->full[st], base + 2 * kTile16Bytes, kb * BK16, row);
              if (kBK == kBF16S)
                tma_load_2d(&mapB, &s->full[st], base + 3 * kTile16Bytes, kb * BK16, (int)args.rows + row);
              continue;
            }
            mbar_arrive_expect_tx(&s->full[st], kTxBytes);
            if (kMode == kModeTN) {
              // both operands MN-major: 32-column boxes of 16 segment rows
              const int row = c.k_row0 + kb * BK;
#pragma unroll
              for (int j = 0; j < BM / 32; ++j)
                tma_load_2d(&mapA, &s->full[st], base + j * (32 * BK * 4), c.m0 + 32 * j, row);
#pragma unroll
              for (int j = 0; j < BNH / 32; ++j)
                tma_load_2d(&mapB, &s->full[st], base + kTileABytes + j * (32 * BK * 4), nb + 32 * j, row);
            } else {
              // A: this CTA's 128 features of expert e's weights
              if (kMode == kModeNT) {
                tma_load_3d(&mapA, &s->full[st], base, kb * BK, c.m0, c.e);
              } else {
#pragma unroll
                for (int j = 0; j < BM / 32; ++j)
                  tma_load_3d(&mapA, &s->full[st], base + j * (32 * BK * 4), c.m0 + 32 * j, kb * BK, c.e);
              }
              // B: this CTA's half of the tile's dispatch rows (n_mma / 2 of them)
              tma_load_2d(&mapB, &s->full[st], base + kTileABytes, kb * BK, c.n0 + (int)rank * (c.n_mma / 2));
            }
          }
        }
        // the last issued loads must land before the CTA may exit
        const uint32_t n_last = it < (uint32_t)kRing ? it : (uint32_t)kRing;
        for (uint32_t j = 0; j < n_last; ++j) {
          const uint32_t i2 = it - 1 - j, st = i2 % kRing, use = i2 / kRing;
          const long long t0 = clock64();
          while (!mbar_try_wait(&s->full[st], use & 1) && clock64() - t0 < kWaitLimitCycles) {
          }
        }
      }
    } else if (warp == 1) {
      // ---------------- MMA issuer (leader CTA only) ----------------
      // Each chunk of kChunkKb k-blocks is accumulated from zero into one of two
      // TMEM buffers; the epilogues of both CTAs fold it into FP32 running sums.
      if (lane == 0 && rank == 0) {
        constexpr bool kAMN = kMode != kModeNT;       // TN: X^T; NN: W (features contiguous)
        constexpr bool kBMN = kMode == kModeTN;       // NN/NT: dispatch rows, K-major
        uint32_t it = 0, ch = 0;
        bool ok = true;
        for (int tile = blockIdx.x / 2; tile < total && ok; tile += n_pairs) {
          const TileCoord tc = decode_tile<kMode>(s, args, n_tiles_n, nk, tile, rank);
          const int tnk = tc.nk;
          const uint32_t idesc = f16_path<kBK>() ? instr_desc_f16((uint32_t)tc.n_mma)
                                                 : instr_desc(kAMN, kBMN, (uint32_t)tc.n_mma);

          for (int c0 = 0; c0 < tnk && ok; c0 += kChunk, ++ch) {
            const uint32_t p = ch & 1, cuse = ch >> 1;
            if (!mbar_wait(s, &s->chunk_empty[p], (cuse & 1) ^ 1, args.err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + p * BN;
            const int c1 = min(c0 + kChunk, tnk);
            for (int kb = c0; kb < c1; ++kb, ++it) {
              const uint32_t st = it % kRing, use = it / kRing;
              if (!mbar_wait(s, &s->split[st], use & 1, args.err)) { ok = false; break; }
              tc_fence_after();
              if (f16_path<kBK>()) {
                // K-major FP16 tiles, 128-byte swizzle: 8-row groups 1024 B
                // apart (SBO), a 16-wide k-step = +32 B inside the swizzle row
                const uint32_t a16 = smem_u32(tiles + st * kRingBytes);
                const uint32_t m16 = a16 + kTile16Bytes, b16 = a16 + 2 * kTile16Bytes, bm16 = a16 + 3 * kTile16Bytes;
#pragma unroll
                for (int kk = 0; kk < BK16 / 16; ++kk) {
                  const uint64_t ad = smem_desc(a16 + kk * 32, 16, 1024, kSwizzle128B);
                  const uint64_t bd = smem_desc(b16 + kk * 32, 16, 1024, kSwizzle128B);
                  if (kBK == kBF16S) {
                    // hi_w x hi_x and hi_w x mid_x share A: one fetch of hi_w
                    tc_mma_f16_pair<kCollFill>(d_tmem, ad, bd, idesc, (kb > c0 || kk > 0) ? 1u : 0u);
                    tc_mma_f16_pair<kCollLast>(d_tmem, ad, smem_desc(bm16 + kk * 32, 16, 1024, kSwizzle128B), idesc,
                                               1u);
                  } else {
                    tc_mma_f16_pair(d_tmem, ad, bd, idesc, (kb > c0 || kk > 0) ? 1u : 0u);
                  }
                  tc_mma_f16_pair(d_tmem, smem_desc(m16 + kk * 32, 16, 1024, kSwizzle128B), bd, idesc, 1u);
                }
                tc_commit_pair(&s->empty[st]);
                continue;
              }
              const uint32_t a_hi = smem_u32(tiles + st * kStageBytes);
              const uint32_t b_hi = a_hi + kTileABytes;
              const uint32_t a_lo = a_hi + kTxBytes, b_lo = b_hi + kTxBytes;
#pragma unroll
              for (int kk = 0; kk < BK / 8; ++kk) {
                // K-major: 8 rows x 64 B per 512-byte group (SBO), k-step = +32 B.
                // MN-major B: 32-column chunks 32*BK*4 B apart (LBO), 4 k-rows per
                // 512-byte group (SBO), k-step of 8 rows = +1024 B.
                uint64_t adh, adl, bdh, bdl;
                if (kAMN) {
                  adh = smem_desc(a_hi + kk * 1024, 32 * BK * 4, 512, kSwizzle128B32B);
                  adl = smem_desc(a_lo + kk * 1024, 32 * BK * 4, 512, kSwizzle128B32B);
                } else {
                  adh = smem_desc(a_hi + kk * 32, 16, 512, kSwizzle64B);
                  adl = smem_desc(a_lo + kk * 32, 16, 512, kSwizzle64B);
                }
                if (kBMN) {
                  bdh = smem_desc(b_hi + kk * 1024, 32 * BK * 4, 512, kSwizzle128B32B);
                  bdl = smem_desc(b_lo + kk * 1024, 32 * BK * 4, 512, kSwizzle128B32B);
                } else {
                  bdh = smem_desc(b_hi + kk * 32, 16, 512, kSwizzle64B);
                  bdl = smem_desc(b_lo + kk * 32, 16, 512, kSwizzle64B);
                }
                tc_mma_tf32_pair(d_tmem, adl, bdh, idesc, (kb > c0 || kk > 0) ? 1u : 0u);
                if (kBK == kBSplit) {
                  // hi_a x lo_b and hi_a x hi_b share A: one fetch of hi_a
                  // (a runtime choice per tile here cost 30 % on small
                  // experts: the collector is used on every tile)
                  tc_mma_tf32_pair<kCollFill>(d_tmem, adh, bdl, idesc, 1u);
                  tc_mma_tf32_pair<kCollLast>(d_tmem, adh, bdh, idesc, 1u);
                } else {
                  tc_mma_tf32_pair(d_tmem, adh, bdh, idesc, 1u);   // B's residual is zero
                }
              }
              tc_commit_pair(&s->empty[st]);
            }
            if (!ok) break;
            tc_commit_pair(&s->chunk_full[p]);
          }
        }
        // every issued MMA completes before TMEM can be freed (in both CTAs)
        tc_commit_pair(&s->drain);
      }
      if (lane == 0) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&s->drain, 0) && clock64() - t0 < kWaitLimitCycles) {
        }
      }
    } else {
      // ---------------- splitters: x -> lo = x - hi in the twin buffer ----------------
      // Each splitter warp owns whole k-blocks (every kNumSplitWarps-th), so a
      // stage costs one proxy fence and one arrive, and the ring depth hides a
      // warp's latency.  The raw tile itself is the high part (the MMA ignores
      // the 13 low bits of an FP32 operand).
      const int ci = warp < 4 ? warp - 2 : warp - 10;
      // kBExact: only A (the weights) is split; B's rows are exact in TF32 and
      // are only checked (low 13 bits zero), a violation recorded as a fault.
      constexpr int kVec = (int)((kBK != kBSplit ? kTileABytes : kTxBytes) / 16);
      constexpr int kBatch = 8;
      static_assert(kVec % (32 * kBatch) == 0, "split batches divide the stage");
      uint32_t it = 0;
      bool ok = true;
      if (f16_path<kBK>()) {
        // nothing to split: warp ci relays stage ci's landing (its own CTA's
        // TMA) to the leader's MMA issuer, one fixed warp per stage
        for (int tile = blockIdx.x / 2; tile < total && ok && ci < kRing; tile += n_pairs) {
          const TileCoord c = decode_tile<kMode>(s, args, n_tiles_n, nk, tile, rank);
          for (int kb = 0; kb < c.nk; ++kb, ++it) {
            if ((int)(it % kRing) != ci) continue;
            const uint32_t st = it % kRing, use = it / kRing;
            if (!mbar_wait(s, &s->full[st], use & 1, args.err)) { ok = false; break; }
            __syncwarp();
            if (lane == 0) mbar_arrive_leader(&s->split[st], rank);
          }
        }
      }
      for (int tile = blockIdx.x / 2; !f16_path<kBK>() && tile < total && ok; tile += n_pairs) {
        const TileCoord c = decode_tile<kMode>(s, args, n_tiles_n, nk, tile, rank);
        for (int kb = 0; kb < c.nk; ++kb, ++it) {
          if ((int)(it % kNumSplitWarps) != ci) continue;
          // kModeTN: rows past the expert's segment belong to the next expert
          const int k_valid = kMode == kModeTN ? c.k_rows - kb * BK : BK;
          const uint32_t st = it % kStages, use = it / kStages;
          if (!mbar_wait(s, &s->full[st], use & 1, args.err)) { ok = false; break; }
          uint4* raw = reinterpret_cast<uint4*>(tiles + st * kStageBytes);
          uint4* lo = reinterpret_cast<uint4*>(tiles + st * kStageBytes + kTxBytes);
#pragma unroll 1
          for (int b0 = lane; b0 < kVec; b0 += 32 * kBatch) {
            uint4 x[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) x[j] = raw[b0 + 32 * j];
            if (kMode == kModeTN && k_valid < BK) {
              // MN-major tiles are [chunk][16 k-rows][128 B]: zero k-rows >= k_valid
#pragma unroll
              for (int j = 0; j < kBatch; ++j)
                if ((((b0 + 32 * j) >> 3) & (BK - 1)) >= k_valid) {
                  x[j] = make_uint4(0u, 0u, 0u, 0u);
                  raw[b0 + 32 * j] = x[j];
                }
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
              lo[b0 + 32 * j] = make_uint4(
                  __float_as_uint(__uint_as_float(x[j].x) - __uint_as_float(x[j].x & kTf32Mask)),
                  __float_as_uint(__uint_as_float(x[j].y) - __uint_as_float(x[j].y & kTf32Mask)),
                  __float_as_uint(__uint_as_float(x[j].z) - __uint_as_float(x[j].z & kTf32Mask)),
                  __float_as_uint(__uint_as_float(x[j].w) - __uint_as_float(x[j].w & kTf32Mask)));
          }
          if (kBK == kBExact) {
            // only the tile's own rows (a K-major row is 4 consecutive 16-byte
            // chunks: the 64-byte swizzle permutes chunks within a row); the box
            // may reach rows past the caller's data
            const uint4* rb = raw + kTileABytes / 16;
            const int half_rows = c.n_mma / 2;
            const int vrows = max(0, min(half_rows, c.n_valid - (int)rank * half_rows));
            uint32_t low = 0;
#pragma unroll 4
            for (int i = lane; i < 4 * vrows; i += 32) {
              const uint4 x = rb[i];
              low |= (x.x | x.y | x.z | x.w) & ~kTf32Mask;
            }
            if (__any_sync(0xffffffffu, low != 0) && lane == 0) atomicCAS(args.err, 0, kFaultNotTf32);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive_leader(&s->split[st], rank);
        }
      }
    }
  }

  // no CTA leaves (or frees TMEM) while its peer may still signal its barriers
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// ---- host side -------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  });
  return fn;
}

// A: [R, Kd] row-major FP32, box 16 (k) x 128 (rows), 64-byte swizzle
bool map_a(CUtensorMap* m, const float* A, int64_t R, int Kd) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)Kd, (cuuint64_t)R};
  cuuint64_t strides[1] = {(cuuint64_t)Kd * 4};
  cuuint32_t box[2] = {BK, BM};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, (void*)A, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// B for "x W": W [E, Kd, N] (N contiguous), box 32 (n) x 16 (k) x 1, 128-byte
//   swizzle with 32-byte atoms (MN-major); 4 boxes per CTA and k-block
// B for "x W^T": W [E, N, Kd] (Kd contiguous), box 16 (k) x 128 (n) x 1, 64-byte swizzle
bool map_b(CUtensorMap* m, const float* W, int E, int Kd, int N, bool nt) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], es[3] = {1, 1, 1};
  if (nt) {
    dims[0] = Kd; dims[1] = N; dims[2] = E;
    strides[0] = (cuuint64_t)Kd * 4; strides[1] = (cuuint64_t)Kd * N * 4;
    box[0] = BK; box[1] = BNH; box[2] = 1;
  } else {
    dims[0] = N; dims[1] = Kd; dims[2] = E;
    strides[0] = (cuuint64_t)N * 4; strides[1] = (cuuint64_t)Kd * N * 4;
    box[0] = 32; box[1] = BK; box[2] = 1;
  }
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, (void*)W, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE,
             nt ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// kBF16W operands, both K-major FP16 with the 128-byte swizzle and a 64-wide
// (128-byte) k-box: the split weights [2E][N][Kd] (box 64 x 128 x 1) and the
// payload rows [R][Kd] (box 64 x 128).  Kd % 8 == 0 (16-byte strides).
bool map_w16(CUtensorMap* m, const uint16_t* W16, int E, int Kd, int N) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)Kd, (cuuint64_t)N, (cuuint64_t)(2 * E)};
  cuuint64_t strides[2] = {(cuuint64_t)Kd * 2, (cuuint64_t)Kd * N * 2};
  cuuint32_t box[3] = {BK16, BM, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, (void*)W16, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool map_rows16(CUtensorMap* m, const uint16_t* A, int64_t R, int Kd) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)Kd, (cuuint64_t)R};
  cuuint64_t strides[1] = {(cuuint64_t)Kd * 2};
  cuuint32_t box[2] = {BK16, BM};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void*)A, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// kModeTN operands: X [R, M] and Y [R, N] row-major, read as MN-major 32-column
// boxes of 16 rows (128-byte swizzle with 32-byte atoms)
bool map_rows_mn(CUtensorMap* m, const float* X, int64_t R, int cols) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)R};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {32, BK};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, (void*)X, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + sizeof(Smem);

// kModeNN/NT: C [R,N] = A [R,Kd] x W_e;  kModeTN: C [E,N,M] with C_e = W_e^T A_e
// (the product A_e^T W_e stored transposed) over expert e's rows of A [R,M] and
// W [R,N] (Kd unused).
// Launch-trace name of a GEMM variant: "tc_gemm <product> <epilogue> <operands>",
// products x.W / x.Wt / Xt.Y, operands tf32x3 (FP32 rows split in the
// kernel), tf32x2 (rows exact in TF32), f16x2 (FP16 payload), f16x3 (two-term
// FP16 rows).
template <int kMode, int kEpi, int kBK>
const char* gemm_trace_name() {
  static const std::string name = [] {
    static const char* modes[] = {"x.W", "x.Wt", "Xt.Y"};
    static const char* epis[] = {"store", "silu", "dsilu", "d2", "accum"};
    const char* ops = kBK == kBSplit ? "tf32x3" : kBK == kBExact ? "tf32x2" : kBK == kBF16W ? "f16x2" : "f16x3";
    return std::string("tc_gemm ") + modes[kMode] + " " + epis[kEpi] + " " + ops;
  }();
  return name.c_str();
}

template <int kMode, int kEpi, int kBK = kBSplit>
janus_status launch(const float* A, const float* W, int64_t R, int E, int Kd, int N, float* C, float* C2,
                    const float* aux, const int32_t* offsets, int32_t* err, cudaStream_t stream, int M = 0,
                    const float* aux2 = nullptr, float* C3 = nullptr, float* const* c_rows = nullptr,
                    const float* row_scale = nullptr, const float* col_scale = nullptr) {
  static_assert(kBK == kBSplit || kMode == kModeNN, "exact or FP16 rows: the forward layout only");
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(tc_gemm_kernel<kMode, kEpi, kBK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmemBytes);
  });
  if (attr != cudaSuccess) return JANUS_ERR_CUDA;
  CUtensorMap ma, mb;
  if (f16_path<kBK>()) {
    // W: the split weights [2E][N][Kd] FP16 (hi for expert e, mid for E + e);
    // A: the payload [R][Kd] (kBF16W) or the rows' hi and mid planes [2R][Kd] (kBF16S)
    if (!map_w16(&ma, reinterpret_cast<const uint16_t*>(W), E, Kd, N) ||
        !map_rows16(&mb, reinterpret_cast<const uint16_t*>(A), kBK == kBF16S ? 2 * R : R, Kd))
      return JANUS_ERR_CUDA;
  } else if (kMode == kModeTN) {
    if (!map_rows_mn(&ma, A, R, M) || !map_rows_mn(&mb, W, R, N)) return JANUS_ERR_CUDA;
  } else if (!map_b(&ma, W, E, Kd, N, kMode == kModeNT) ||
             !map_a(&mb, A, R, Kd)) {
    // operands swapped: the weights are the MMA's A, the dispatch rows its B
    return JANUS_ERR_CUDA;
  }
  Args a;
  a.C = C; a.C2 = C2; a.C3 = C3; a.aux = aux; a.aux2 = aux2; a.c_rows = c_rows;
  a.row_scale = row_scale; a.col_scale = col_scale; a.rows = R;
  a.offsets = offsets; a.E = E; a.Kd = Kd; a.N = N; a.M = M; a.err = err;
  // one CTA per SM, in clusters of two (the MMA pairs)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(num_sms() / 2 * 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute cluster_attr[1];
  cluster_attr[0].id = cudaLaunchAttributeClusterDimension;
  cluster_attr[0].val.clusterDim.x = 2;
  cluster_attr[0].val.clusterDim.y = 1;
  cluster_attr[0].val.clusterDim.z = 1;
  cfg.attrs = cluster_attr;
  cfg.numAttrs = 1;
  TraceScope trace(gemm_trace_name<kMode, kEpi, kBK>(), stream);
  if (cudaLaunchKernelEx(&cfg, tc_gemm_kernel<kMode, kEpi, kBK>, ma, mb, a) != cudaSuccess)
    return JANUS_ERR_CUDA;
  return launch_status();
}

// ---- the FP16 split of the weights for the kind::f16 GEMMs ------------------
// x W (W [E][Kd][N]) or x W^T (W [E][N][Kd]) FP32 -> w16 = [hi | mid], each
// [E][N][Kd] FP16 (K-major for the kind::f16 MMA: x W's weights are
// transposed on the way), and winv [E][nch][N] = 1 / S per output feature and
// K chunk of 256 (nch = ceil(Kd / 256), the GEMM's TMEM chunk, so the
// epilogue applies each chunk's scale as it folds the chunk).  S = 2^(141 -
// b), b = the biased exponent of the largest magnitude of the feature's
// chunk, so that magnitude times S lies in [2^14, 2^15) (below FP16's 65504);
// S is clamped to [2^-126, 2^126] and is 1 for an all-zero chunk.  hi = fp16(w
// S) and mid = fp16(w S - hi): w S - hi is exact in FP32 and the pair carries
// 22 bits of w S.  One kernel, W read once.  N % 4 == 0 and Kd % 4 == 0
// (JANUS_ERR_MISALIGNED otherwise).

__device__ __forceinline__ uint32_t half2_bits(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ int w16_scale_exp(uint32_t max_bits) {
  if (max_bits == 0) return 0;
  const int b = max((int)(max_bits >> 23), 1);
  return min(max(141 - b, -126), 126);
}

// x W: tiles of one expert's 256 k x 32 features (W[e] is [Kd][N]).  Each
// thread loads eight float4 (128-byte row segments, all in flight), the 32
// column maxima of the tile go through shared memory, and the tile is scaled,
// split and transposed through shared memory into the K-major planes, each
// warp writing four features' 256 k as half2 pairs: W is read once.
constexpr int kChunkK = 256;           // the K chunk of the scales (= the GEMM's TMEM chunk)
__global__ void __launch_bounds__(256) w16_split_cols_kernel(const float* __restrict__ w, int E, int Kd, int N,
                                                             __half* __restrict__ w16, float* __restrict__ winv) {
  __shared__ uint32_t red[32][33];
  __shared__ float s_scale[32];
  __shared__ __align__(16) __half t_hi[32][kChunkK + 2];
  __shared__ __align__(16) __half t_mid[32][kChunkK + 2];
  const int tid = threadIdx.x, tx = tid % 8, ty = tid / 8;
  const int warp = tid / 32, lane = tid % 32;
  const int strips_n = (N + 31) / 32, nch = (Kd + kChunkK - 1) / kChunkK;
  const int64_t n_tiles = (int64_t)E * nch * strips_n;
  const int64_t plane = (int64_t)E * N * Kd;                 // mid follows hi
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const int st = (int)(t % strips_n);
    const int64_t ec = t / strips_n;
    const int e = (int)(ec / nch), ci = (int)(ec % nch), f0 = st * 32, k0 = ci * kChunkK;
    const float* we = w + (int64_t)e * Kd * N;
    const int fc = f0 + 4 * tx;
    const bool col_ok = fc < N;                              // N % 4 == 0: all four columns
    float4 v[kChunkK / 32];
#pragma unroll
    for (int u = 0; u < kChunkK / 32; ++u) {
      const int k = k0 + ty + 32 * u;
      v[u] = (col_ok && k < Kd) ? __ldcs(reinterpret_cast<const float4*>(we + (int64_t)k * N + fc)) : zero;
    }
    uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int u = 0; u < kChunkK / 32; ++u) {
      m[0] = max(m[0], __float_as_uint(v[u].x) & 0x7fffffffu);
      m[1] = max(m[1], __float_as_uint(v[u].y) & 0x7fffffffu);
      m[2] = max(m[2], __float_as_uint(v[u].z) & 0x7fffffffu);
      m[3] = max(m[3], __float_as_uint(v[u].w) & 0x7fffffffu);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) red[ty][4 * tx + j] = m[j];
    __syncthreads();
    if (tid < 32) {
      uint32_t mm = 0;
      for (int j = 0; j < 32; ++j) mm = max(mm, red[j][tid]);
      const int ex = w16_scale_exp(mm);
      s_scale[tid] = __uint_as_float((uint32_t)(127 + ex) << 23);
      if (f0 + tid < N) winv[((int64_t)e * nch + ci) * N + f0 + tid] = __uint_as_float((uint32_t)(127 - ex) << 23);
    }
    __syncthreads();
    float sc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) sc[j] = s_scale[4 * tx + j];
#pragma unroll
    for (int u = 0; u < kChunkK / 32; ++u) {
      const int kr = ty + 32 * u;
      const float val[4] = {v[u].x * sc[0], v[u].y * sc[1], v[u].z * sc[2], v[u].w * sc[3]};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half hi = __float2half_rn(val[j]);
        t_hi[4 * tx + j][kr] = hi;
        t_mid[4 * tx + j][kr] = __float2half_rn(val[j] - __half2float(hi));
      }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int fl = warp * 4 + j, fo = f0 + fl;
      if (fo >= N) continue;
      const int64_t row = ((int64_t)e * N + fo) * Kd;
#pragma unroll
      for (int q = 0; q < kChunkK / 64; ++q) {
        const int kk = 2 * (lane + 32 * q), ko = k0 + kk;
        if (ko + 1 < Kd) {
          __stcs(reinterpret_cast<__half2*>(w16 + row + ko), *reinterpret_cast<const __half2*>(&t_hi[fl][kk]));
          __stcs(reinterpret_cast<__half2*>(w16 + plane + row + ko), *reinterpret_cast<const __half2*>(&t_mid[fl][kk]));
        } else if (ko < Kd) {
          w16[row + ko] = t_hi[fl][kk];
          w16[plane + row + ko] = t_mid[fl][kk];
        }
      }
    }
    __syncthreads();
  }
}

// x W^T: W [E][N][Kd] is K-major already: one warp per (row, K chunk of 256),
// two float4 per lane, the chunk's maximum by shuffles, then hi and mid; a
// warp loads two such items before working on either.
__global__ void __launch_bounds__(256) w16_split_rows_kernel(const float4* __restrict__ w, int64_t rows, int Kd,
                                                             int N, uint2* __restrict__ w16,
                                                             float* __restrict__ winv) {
  constexpr int kItems = 2, kU = kChunkK / 128;
  const int lane = threadIdx.x % 32;
  const int k4 = Kd / 4, nch = (Kd + kChunkK - 1) / kChunkK;
  const int64_t items = rows * nch;
  uint2* __restrict__ mid = w16 + rows * k4;
  const int64_t nw = (int64_t)gridDim.x * 8;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t it0 = ((int64_t)blockIdx.x * 256 + threadIdx.x) / 32; it0 < items; it0 += kItems * nw) {
    float4 v[kItems][kU];
#pragma unroll
    for (int q = 0; q < kItems; ++q) {
      const int64_t it = it0 + q * nw;
      const int64_t base = (it / nch) * k4;
      const int cb = (int)(it % nch) * (kChunkK / 4);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = cb + u * 32 + lane;
        v[q][u] = (it < items && c < k4) ? __ldcs(w + base + c) : zero;
      }
    }
#pragma unroll
    for (int q = 0; q < kItems; ++q) {
      const int64_t it = it0 + q * nw;
      if (it >= items) break;                       // the same in every lane
      const int64_t r = it / nch;
      const int ci = (int)(it % nch);
      const int64_t base = r * k4;
      uint32_t m = 0;
#pragma unroll
      for (int u = 0; u < kU; ++u)
        m = max(m, max(max(__float_as_uint(v[q][u].x) & 0x7fffffffu, __float_as_uint(v[q][u].y) & 0x7fffffffu),
                       max(__float_as_uint(v[q][u].z) & 0x7fffffffu, __float_as_uint(v[q][u].w) & 0x7fffffffu)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int ex = w16_scale_exp(m);
      const float S = __uint_as_float((uint32_t)(127 + ex) << 23);
      if (lane == 0) {
        const int64_t e = r / N, n = r % N;
        winv[(e * nch + ci) * N + n] = __uint_as_float((uint32_t)(127 - ex) << 23);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = ci * (kChunkK / 4) + u * 32 + lane;
        if (c < k4) {
          float4 o = v[q][u];
          o.x *= S; o.y *= S; o.z *= S; o.w *= S;
          const uint2 hq = make_uint2(half2_bits(o.x, o.y), half2_bits(o.z, o.w));
          const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&hq.x));
          const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&hq.y));
          __stcs(w16 + base + c, hq);
          __stcs(mid + base + c, make_uint2(half2_bits(o.x - h0.x, o.y - h0.y), half2_bits(o.z - h1.x, o.w - h1.y)));
        }
      }
    }
  }
}

// Both orientations of one weight tensor W [E][A][B] from one DRAM read of W,
// for a layer whose forward and input VJP use the same weights:
//   T, the split for x W  (Kd = A, N = B): planes [E][B][A], winvT [E][ceil(A/256)][B];
//   R, the split for x W^T (N = A, Kd = B): planes [E][A][B], winvR [E][ceil(B/256)][A];
// bit for bit what w16_split_cols_kernel and w16_split_rows_kernel write.  A
// CTA takes 256 x 256 blocks of one expert.  The first sweep reads the block
// for its 256 row maxima (R's scales, chunk = the block's columns) and 256
// column maxima (T's scales, chunk = its rows) and writes nothing; the second
// reads it again, from L2 (two CTAs per SM: about 76 MB of blocks are live),
// in 256-row x 32-column strips, the next strip's loads in flight while the
// current one is written: R's terms go out from the registers and T's through
// a shared-memory transpose, as in the transposing kernel.  Two CTAs per SM
// let one CTA's loads overlap the other's stores.  DRAM traffic: W once, the
// four planes once.
constexpr int kBothThreads = 256, kBothWarps = kBothThreads / 32;
__global__ void __launch_bounds__(kBothThreads, 2) w16_split_both_kernel(const float* __restrict__ w, int E, int A,
                                                                         int B, __half* __restrict__ w16t,
                                                                         float* __restrict__ winvt,
                                                                         __half* __restrict__ w16r,
                                                                         float* __restrict__ winvr) {
  __shared__ uint32_t s_cmax[kChunkK];                     // column maxima (|w| bits)
  __shared__ float s_rs[kChunkK], s_cs[kChunkK];
  __shared__ __align__(16) __half t_hi[32][kChunkK + 2];
  __shared__ __align__(16) __half t_mid[32][kChunkK + 2];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int tx = tid % 8, ty = tid / 8;                   // sweep 2: 4 columns, rows ty + 32 u
  const int nca = (A + kChunkK - 1) / kChunkK, ncb = (B + kChunkK - 1) / kChunkK, b4 = B / 4;
  const int64_t n_blocks = (int64_t)E * nca * ncb;
  const int64_t plane = (int64_t)E * A * B;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr int kRowsPerWarp = kChunkK / kBothWarps, kStripRows = kChunkK / 32;
  if (tid < kChunkK) s_cmax[tid] = 0u;                      // reset again as each block reads it
  __syncthreads();
  for (int64_t t = blockIdx.x; t < n_blocks; t += gridDim.x) {
    const int cb = (int)(t % ncb);
    const int64_t t1 = t / ncb;
    const int ca = (int)(t1 % nca), e = (int)(t1 / nca);
    const int a0 = ca * kChunkK, b0 = cb * kChunkK;
    const float* we = w + (int64_t)e * A * B;
    const int n_strips = min(kChunkK, B - b0 + 31) / 32;   // strips with a column in range
    // sweep 1: warp w takes the block's rows w + 8 i (i < 32), four at a
    // time; lane l holds the float4 columns l and l + 32 of the block's 64
    uint32_t cm[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
#pragma unroll 1
    for (int i0 = 0; i0 < kRowsPerWarp; i0 += 4) {
      float4 v[4][2];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int a = a0 + warp + kBothWarps * (i0 + q);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = b0 / 4 + lane + 32 * u;
          v[q][u] = (a < A && c < b4) ? __ldcg(reinterpret_cast<const float4*>(we + (int64_t)a * B) + c) : zero;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t m = 0;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint32_t x = __float_as_uint(v[q][u].x) & 0x7fffffffu, y = __float_as_uint(v[q][u].y) & 0x7fffffffu;
          const uint32_t z = __float_as_uint(v[q][u].z) & 0x7fffffffu, ww = __float_as_uint(v[q][u].w) & 0x7fffffffu;
          cm[u][0] = max(cm[u][0], x); cm[u][1] = max(cm[u][1], y);
          cm[u][2] = max(cm[u][2], z); cm[u][3] = max(cm[u][3], ww);
          m = max(m, max(max(x, y), max(z, ww)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) {
          const int ar = warp + kBothWarps * (i0 + q), ex = w16_scale_exp(m);
          s_rs[ar] = __uint_as_float((uint32_t)(127 + ex) << 23);
          if (a0 + ar < A) winvr[((int64_t)e * ncb + cb) * A + a0 + ar] = __uint_as_float((uint32_t)(127 - ex) << 23);
        }
      }
    }
    // the first strip's loads go out before the column maxima meet
    float4 v[kStripRows];
    auto load_strip = [&](int sp, float4* dst) {
      const int bc = b0 + 32 * sp + 4 * tx;
      const bool col_ok = bc < B;                          // B % 4 == 0: all four columns
#pragma unroll
      for (int u = 0; u < kStripRows; ++u) {
        const int a = a0 + ty + 32 * u;
        dst[u] = (col_ok && a < A) ? __ldcs(reinterpret_cast<const float4*>(we + (int64_t)a * B + bc)) : zero;
      }
    };
    load_strip(0, v);
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (cm[u][j]) atomicMax(&s_cmax[4 * (lane + 32 * u) + j], cm[u][j]);
    __syncthreads();
    if (tid < kChunkK) {
      const uint32_t mm = s_cmax[tid];
      s_cmax[tid] = 0u;
      const int ex = w16_scale_exp(mm);
      s_cs[tid] = __uint_as_float((uint32_t)(127 + ex) << 23);
      if (b0 + tid < B) winvt[((int64_t)e * nca + ca) * B + b0 + tid] = __uint_as_float((uint32_t)(127 - ex) << 23);
    }
    __syncthreads();
    // sweep 2: strip sp's values in v, strip sp + 1's loads in flight
#pragma unroll 1
    for (int sp = 0; sp < n_strips; ++sp) {
      const int bs = b0 + 32 * sp, bc = bs + 4 * tx;
      const bool col_ok = bc < B;
      float4 vn[kStripRows];
      if (sp + 1 < n_strips) load_strip(sp + 1, vn);
      float cs[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) cs[j] = s_cs[32 * sp + 4 * tx + j];
#pragma unroll
      for (int u = 0; u < kStripRows; ++u) {
        const int ar = ty + 32 * u, a = a0 + ar;
        // R: the row's scale, both terms stored from the registers
        const float S = s_rs[ar];
        float4 o = v[u];
        o.x *= S; o.y *= S; o.z *= S; o.w *= S;
        const uint2 hq = make_uint2(half2_bits(o.x, o.y), half2_bits(o.z, o.w));
        const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&hq.x));
        const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&hq.y));
        if (col_ok && a < A) {
          const int64_t at = ((int64_t)e * A + a) * B + bc;
          __stcs(reinterpret_cast<uint2*>(w16r + at), hq);
          __stcs(reinterpret_cast<uint2*>(w16r + plane + at),
                 make_uint2(half2_bits(o.x - h0.x, o.y - h0.y), half2_bits(o.z - h1.x, o.w - h1.y)));
        }
        // T: the column scales, transposed through shared memory
        const float val[4] = {v[u].x * cs[0], v[u].y * cs[1], v[u].z * cs[2], v[u].w * cs[3]};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half hi = __float2half_rn(val[j]);
          t_hi[4 * tx + j][ar] = hi;
          t_mid[4 * tx + j][ar] = __float2half_rn(val[j] - __half2float(hi));
        }
      }
      __syncthreads();
      // each warp writes four features' 256 values of a as half2 pairs
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int fl = warp * 4 + j, fo = bs + fl;
        if (fo >= B) continue;
        const int64_t row = ((int64_t)e * B + fo) * A;
#pragma unroll
        for (int q = 0; q < kChunkK / 64; ++q) {
          const int kk = 2 * (lane + 32 * q), ao = a0 + kk;
          if (ao < A) {                                       // A % 4 == 0: ao + 1 < A too
            __stcs(reinterpret_cast<__half2*>(w16t + row + ao), *reinterpret_cast<const __half2*>(&t_hi[fl][kk]));
            __stcs(reinterpret_cast<__half2*>(w16t + plane + row + ao),
                   *reinterpret_cast<const __half2*>(&t_mid[fl][kk]));
          }
        }
      }
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kStripRows; ++u) v[u] = vn[u];
    }
  }
}

// ---- the FP16 row split of an activation for a kind::f16 GEMM ---------------
// v = silu(a) (kActSilu) or x silu'(a) (kActDSilu), with the SiLU arithmetic
// of the GEMM epilogues, written as hi and mid binary16 planes
// ([rows][n] each) with one power-of-two scale per row: S_p puts the row's
// largest |v| in [2^14, 2^15), hi = fp16(v S_p), mid = fp16(v S_p - hi),
// row_scale[p] = 1 / S_p.  Rows up to 4096 values stay in the registers of a
// 128-thread block (act_split_blk_kernel); longer ones take one warp and two
// sweeps, the first for the row's maximum, the second recomputing v and
// writing the two terms with loads that find the row in L1 / L2
// (act_split_kernel).  Either way the inputs are read from DRAM once and the
// FP32 v is never stored.
enum ActOp { kActSilu = 1, kActDSilu = 2 };
constexpr int kActU = 4;       // float4 columns per lane in flight per sweep step

template <int kOp, bool kLast>
__device__ __forceinline__ float4 act_value(const float4* __restrict__ x, const float4* __restrict__ a, int64_t i) {
  const float4 av = kLast ? __ldcs(a + i) : __ldg(a + i);
  if (kOp == kActSilu) return make_float4(silu_f(av.x), silu_f(av.y), silu_f(av.z), silu_f(av.w));
  const float4 xv = kLast ? __ldcs(x + i) : __ldg(x + i);
  float4 v;
  float sg;
  sg = sigmoid_fast(av.x); v.x = xv.x * (sg * (1.0f + av.x * (1.0f - sg)));
  sg = sigmoid_fast(av.y); v.y = xv.y * (sg * (1.0f + av.y * (1.0f - sg)));
  sg = sigmoid_fast(av.z); v.z = xv.z * (sg * (1.0f + av.z * (1.0f - sg)));
  sg = sigmoid_fast(av.w); v.w = xv.w * (sg * (1.0f + av.w * (1.0f - sg)));
  return v;
}

template <int kOp>
__global__ void __launch_bounds__(256)
act_split_kernel(const float4* __restrict__ x, const float4* __restrict__ a, int64_t rows, int n4,
                 uint2* __restrict__ rows16, float* __restrict__ row_scale) {
  const int lane = threadIdx.x % 32;
  const int64_t nw = (int64_t)gridDim.x * 8;
  uint2* __restrict__ mid = rows16 + rows * n4;
  for (int64_t p = ((int64_t)blockIdx.x * 256 + threadIdx.x) / 32; p < rows; p += nw) {
    const int64_t base = p * n4;
    uint32_t m = 0;
    for (int c0 = 0; c0 < n4; c0 += 32 * kActU) {
      float4 v[kActU];
#pragma unroll
      for (int u = 0; u < kActU; ++u) {
        const int c = c0 + u * 32 + lane;
        v[u] = c < n4 ? act_value<kOp, false>(x, a, base + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kActU; ++u)
        m = max(m, max(max(__float_as_uint(v[u].x) & 0x7fffffffu, __float_as_uint(v[u].y) & 0x7fffffffu),
                       max(__float_as_uint(v[u].z) & 0x7fffffffu, __float_as_uint(v[u].w) & 0x7fffffffu)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int e = w16_scale_exp(m);
    const float S = __uint_as_float((uint32_t)(127 + e) << 23);
    if (lane == 0) row_scale[p] = __uint_as_float((uint32_t)(127 - e) << 23);
    for (int c0 = 0; c0 < n4; c0 += 32 * kActU) {
#pragma unroll
      for (int u = 0; u < kActU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < n4) {
          float4 o = act_value<kOp, true>(x, a, base + c);
          o.x *= S; o.y *= S; o.z *= S; o.w *= S;
          const uint2 hq = make_uint2(half2_bits(o.x, o.y), half2_bits(o.z, o.w));
          const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&hq.x));
          const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&hq.y));
          __stcs(reinterpret_cast<uint2*>(rows16) + base + c, hq);
          __stcs(mid + base + c, make_uint2(half2_bits(o.x - h0.x, o.y - h0.y), half2_bits(o.z - h1.x, o.w - h1.y)));
        }
      }
    }
  }
}

// Rows of at most 128 * kNU float4 (n <= 4096): a block of 128 threads per
// row keeps it in registers, kNU float4 per thread (a and, for dSiLU, dH all
// in flight at once), so each value is read once and the two terms are
// written from registers; the row maximum goes through shared memory (two
// slots by row parity, so one barrier per row suffices).
constexpr int kActBlk = 128;
template <int kOp, int kNU>
__global__ void __launch_bounds__(kActBlk)
act_split_blk_kernel(const float4* __restrict__ x, const float4* __restrict__ a, int64_t rows, int n4,
                     uint2* __restrict__ rows16, float* __restrict__ row_scale) {
  __shared__ uint32_t red[2][kActBlk / 32];
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  uint2* __restrict__ mid = rows16 + rows * n4;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  int parity = 0;
  for (int64_t p = blockIdx.x; p < rows; p += gridDim.x, parity ^= 1) {
    const int64_t base = p * n4;
    float4 v[kNU];
#pragma unroll
    for (int u = 0; u < kNU; ++u) {
      const int c = u * kActBlk + tid;
      v[u] = c < n4 ? __ldcs(a + base + c) : zero;
    }
    if (kOp == kActDSilu) {
      float4 g[kNU];
#pragma unroll
      for (int u = 0; u < kNU; ++u) {
        const int c = u * kActBlk + tid;
        g[u] = c < n4 ? __ldcs(x + base + c) : zero;
      }
#pragma unroll
      for (int u = 0; u < kNU; ++u) {
        float sg;
        sg = sigmoid_fast(v[u].x); v[u].x = g[u].x * (sg * (1.0f + v[u].x * (1.0f - sg)));
        sg = sigmoid_fast(v[u].y); v[u].y = g[u].y * (sg * (1.0f + v[u].y * (1.0f - sg)));
        sg = sigmoid_fast(v[u].z); v[u].z = g[u].z * (sg * (1.0f + v[u].z * (1.0f - sg)));
        sg = sigmoid_fast(v[u].w); v[u].w = g[u].w * (sg * (1.0f + v[u].w * (1.0f - sg)));
      }
    } else if (kOp == kActSilu) {
#pragma unroll
      for (int u = 0; u < kNU; ++u) v[u] = make_float4(silu_f(v[u].x), silu_f(v[u].y), silu_f(v[u].z), silu_f(v[u].w));
    }
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < kNU; ++u)
      m = max(m, max(max(__float_as_uint(v[u].x) & 0x7fffffffu, __float_as_uint(v[u].y) & 0x7fffffffu),
                     max(__float_as_uint(v[u].z) & 0x7fffffffu, __float_as_uint(v[u].w) & 0x7fffffffu)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[parity][warp] = m;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kActBlk / 32; ++w) m = max(m, red[parity][w]);
    const int e = w16_scale_exp(m);
    const float S = __uint_as_float((uint32_t)(127 + e) << 23);
    if (tid == 0) row_scale[p] = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
    for (int u = 0; u < kNU; ++u) {
      const int c = u * kActBlk + tid;
      if (c < n4) {
        float4 o = v[u];
        o.x *= S; o.y *= S; o.z *= S; o.w *= S;
        const uint2 hq = make_uint2(half2_bits(o.x, o.y), half2_bits(o.z, o.w));
        const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&hq.x));
        const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&hq.y));
        __stcs(rows16 + base + c, hq);
        __stcs(mid + base + c, make_uint2(half2_bits(o.x - h0.x, o.y - h0.y), half2_bits(o.z - h1.x, o.w - h1.y)));
      }
    }
  }
}

template <typename Kernel>
int64_t resident_grid(Kernel k, int64_t rows) {
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k, 256, 0) != cudaSuccess || b < 1) b = 2;
  return std::min<int64_t>((rows + 7) / 8, (int64_t)num_sms() * b);
}

template <int kOp, int kNU>
void launch_act_split_blk(const float* x, const float* a, int64_t rows, int32_t n, uint16_t* rows16, float* row_scale,
                          cudaStream_t stream) {
  static const int per_sm = [] {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, act_split_blk_kernel<kOp, kNU>, kActBlk, 0) != cudaSuccess ||
        b < 1)
      b = 4;
    return b;
  }();
  const int64_t blocks = std::min<int64_t>(rows, (int64_t)num_sms() * per_sm);
  act_split_blk_kernel<kOp, kNU><<<(unsigned)blocks, kActBlk, 0, stream>>>((const float4*)x, (const float4*)a, rows,
                                                                           n / 4, (uint2*)rows16, row_scale);
}

template <int kOp>
janus_status act_split_launch(const float* x, const float* a, int64_t rows, int32_t n, uint16_t* rows16,
                              float* row_scale, cudaStream_t stream) {
  if (rows == 0) return JANUS_OK;
  // float4 per thread for the whole row, 128 threads per row
  switch ((n / 4 + kActBlk - 1) / kActBlk) {
    case 1: launch_act_split_blk<kOp, 1>(x, a, rows, n, rows16, row_scale, stream); break;
    case 2: launch_act_split_blk<kOp, 2>(x, a, rows, n, rows16, row_scale, stream); break;
    case 3: launch_act_split_blk<kOp, 3>(x, a, rows, n, rows16, row_scale, stream); break;
    case 4: launch_act_split_blk<kOp, 4>(x, a, rows, n, rows16, row_scale, stream); break;
    case 5: launch_act_split_blk<kOp, 5>(x, a, rows, n, rows16, row_scale, stream); break;
    case 6: launch_act_split_blk<kOp, 6>(x, a, rows, n, rows16, row_scale, stream); break;
    case 7: launch_act_split_blk<kOp, 7>(x, a, rows, n, rows16, row_scale, stream); break;
    case 8: launch_act_split_blk<kOp, 8>(x, a, rows, n, rows16, row_scale, stream); break;
    default: {
      // longer rows: two sweeps, the second finding the row in L1 / L2
      static const int64_t per_sm_probe = resident_grid(act_split_kernel<kOp>, INT64_MAX / 2);
      const int64_t blocks = std::min<int64_t>((rows + 7) / 8, per_sm_probe);
      act_split_kernel<kOp><<<(unsigned)blocks, 256, 0, stream>>>((const float4*)x, (const float4*)a, rows, n / 4,
                                                                   (uint2*)rows16, row_scale);
    }
  }
  return launch_status();
}

template <int kOp>
janus_status act_split_f16(const float* x, const float* a, int64_t rows, int32_t n, uint16_t* rows16,
                           float* row_scale, cudaStream_t stream) {
  TraceScope trace(kOp == kActSilu ? "act_split silu" : "act_split dsilu", stream);
  return act_split_launch<kOp>(x, a, rows, n, rows16, row_scale, stream);
}

}  // namespace

janus_status split_weights_f16(const float* w, int32_t E, int32_t Kd, int32_t N, bool transposed, uint16_t* w16,
                               float* winv, cudaStream_t stream) {
  TraceScope trace(transposed ? "w16_split transposed" : "w16_split rows", stream);
  if (N % 4 != 0 || Kd % 4 != 0) return JANUS_ERR_MISALIGNED;   // the FFN calls require d, h % 4 == 0
  const int64_t nch = (Kd + kChunkK - 1) / kChunkK;
  if (!transposed) {
    const int64_t items = (int64_t)E * N * nch;
    const int64_t blocks = std::min<int64_t>((items + 7) / 8, (int64_t)num_sms() * 8);
    w16_split_rows_kernel<<<(unsigned)blocks, 256, 0, stream>>>((const float4*)w, (int64_t)E * N, Kd, N,
                                                               (uint2*)w16, winv);
    return launch_status();
  }
  const int64_t tiles = (int64_t)E * nch * ((N + 31) / 32);
  const int64_t blocks = std::min<int64_t>(tiles, (int64_t)num_sms() * 4);
  w16_split_cols_kernel<<<(unsigned)blocks, 256, 0, stream>>>(w, E, Kd, N, reinterpret_cast<__half*>(w16), winv);
  return launch_status();
}

janus_status split_weights_f16_both(const float* w, int32_t E, int32_t A, int32_t B, uint16_t* w16t, float* winvt,
                                    uint16_t* w16r, float* winvr, cudaStream_t stream) {
  TraceScope trace("w16_split both", stream);
  if (A % 4 != 0 || B % 4 != 0) return JANUS_ERR_MISALIGNED;
  const int64_t n_blocks = (int64_t)E * ((A + kChunkK - 1) / kChunkK) * ((B + kChunkK - 1) / kChunkK);
  const int64_t blocks = std::min<int64_t>(n_blocks, (int64_t)num_sms() * 2);   // two CTAs per SM
  w16_split_both_kernel<<<(unsigned)blocks, kBothThreads, 0, stream>>>(
      w, E, A, B, reinterpret_cast<__half*>(w16t), winvt, reinterpret_cast<__half*>(w16r), winvr);
  return launch_status();
}

size_t workspace_extra() { return 0; }

janus_status expert_ffn_fwd(const float* xd, const int32_t* offsets, int32_t E, int64_t R, int32_t d,
                            int32_t h, const float* w1, const float* w2, float* yd, float* act, float* H,
                            int32_t* err, cudaStream_t stream, float* const* yd_rows, bool x_tf32_exact) {
  janus_status st = x_tf32_exact
                        ? launch<kModeNN, kEpiSilu, kBExact>(xd, w1, R, E, d, h, H, act, nullptr, offsets, err, stream)
                        : launch<kModeNN, kEpiSilu>(xd, w1, R, E, d, h, H, act, nullptr, offsets, err, stream);
  if (st != JANUS_OK) return st;
  return launch<kModeNN, kEpiStore>(H, w2, R, E, h, d, yd, nullptr, nullptr, offsets, err, stream, 0, nullptr,
                                    nullptr, yd_rows);
}

namespace {
// The forward behind the FP16 split of W1 (transposed to [E][h][d], K-major):
// the kind::f16 first GEMM on FP16 rows (kBK = kBF16W: the packed payload;
// kBF16S: two-term split rows), then the second GEMM, yd = H W2.  Without
// `second` the first GEMM stores a and H = silu(a) and the second runs on
// 3xTF32.  With it the first GEMM stores only a (into act, else the
// workspace's H), one pass turns a into H's two FP16 terms per row, W2 is
// split per output feature, and the second GEMM runs on the kind::f16 path
// with three products.
template <int kBK>
janus_status fwd_f16(const uint16_t* rows, const float* row_scale, const int32_t* offsets, int32_t E, int64_t R,
                     int32_t d, int32_t h, const float* w1, const float* w2, float* yd, float* act, float* H,
                     uint16_t* w16, float* winv, int32_t* err, cudaStream_t stream, float* const* yd_rows,
                     const F16Second* second, bool presplit) {
  janus_status st = presplit ? JANUS_OK : split_weights_f16(w1, E, d, h, true, w16, winv, stream);
  if (st != JANUS_OK) return st;
  const float* xq = reinterpret_cast<const float*>(rows);
  const float* wq = reinterpret_cast<const float*>(w16);
  if (!second) {
    st = launch<kModeNN, kEpiSilu, kBK>(xq, wq, R, E, d, h, H, act, nullptr, offsets, err, stream, 0, nullptr,
                                        nullptr, nullptr, row_scale, winv);
    if (st != JANUS_OK) return st;
    return launch<kModeNN, kEpiStore>(H, w2, R, E, h, d, yd, nullptr, nullptr, offsets, err, stream, 0, nullptr,
                                      nullptr, yd_rows);
  }
  float* A = act ? act : H;
  st = launch<kModeNN, kEpiStore, kBK>(xq, wq, R, E, d, h, A, nullptr, nullptr, offsets, err, stream, 0, nullptr,
                                       nullptr, nullptr, row_scale, winv);
  if (st != JANUS_OK) return st;
  st = act_split_f16<kActSilu>(nullptr, A, R, h, second->h16, second->hscale, stream);
  if (st != JANUS_OK) return st;
  if (!presplit) st = split_weights_f16(w2, E, h, d, true, second->w16, second->winv, stream);
  if (st != JANUS_OK) return st;
  return launch<kModeNN, kEpiStore, kBF16S>(reinterpret_cast<const float*>(second->h16),
                                            reinterpret_cast<const float*>(second->w16), R, E, h, d, yd, nullptr,
                                            nullptr, offsets, err, stream, 0, nullptr, nullptr, yd_rows,
                                            second->hscale, second->winv);
}
}  // namespace

janus_status expert_ffn_fwd_packed(const uint16_t* payload, const float* row_scale, const int32_t* offsets,
                                   int32_t E, int64_t R, int32_t d, int32_t h, const float* w1, const float* w2,
                                   float* yd, float* act, float* H, uint16_t* w16, float* winv, int32_t* err,
                                   cudaStream_t stream, float* const* yd_rows, const F16Second* second,
                                   bool weights_presplit) {
  return fwd_f16<kBF16W>(payload, row_scale, offsets, E, R, d, h, w1, w2, yd, act, H, w16, winv, err, stream,
                         yd_rows, second, weights_presplit);
}

janus_status expert_ffn_fwd_split(const uint16_t* rows16, const float* row_scale, const int32_t* offsets, int32_t E,
                                  int64_t R, int32_t d, int32_t h, const float* w1, const float* w2, float* yd,
                                  float* act, float* H, uint16_t* w16, float* winv, int32_t* err,
                                  cudaStream_t stream, float* const* yd_rows, const F16Second* second,
                                  bool weights_presplit) {
  return fwd_f16<kBF16S>(rows16, row_scale, offsets, E, R, d, h, w1, w2, yd, act, H, w16, winv, err, stream,
                         yd_rows, second, weights_presplit);
}

janus_status expert_ffn_vjp_split(const uint16_t* gd16, const float* gd_scale, const float* act,
                                  const int32_t* offsets, int32_t E, int64_t R, int32_t d, int32_t h,
                                  const float* w1, const float* w2, float* dxd, float* dA, uint16_t* w16,
                                  float* winv, int32_t* err, cudaStream_t stream, float* const* dxd_rows,
                                  const F16Second* second, bool weights_presplit) {
  // gd W2^T: W2 [E][h][d] is K-major for this product as it stands
  janus_status st = weights_presplit ? JANUS_OK : split_weights_f16(w2, E, d, h, false, w16, winv, stream);
  if (st != JANUS_OK) return st;
  const float* gq = reinterpret_cast<const float*>(gd16);
  const float* wq = reinterpret_cast<const float*>(w16);
  if (!second) {
    // dA = (gd W2^T) * silu'(a) in the epilogue, then dxd = dA W1^T on 3xTF32
    st = launch<kModeNN, kEpiDSilu, kBF16S>(gq, wq, R, E, d, h, dA, nullptr, act, offsets, err, stream, 0, nullptr,
                                             nullptr, nullptr, gd_scale, winv);
    if (st != JANUS_OK) return st;
    return launch<kModeNT, kEpiStore>(dA, w1, R, E, h, d, dxd, nullptr, nullptr, offsets, err, stream, 0, nullptr,
                                      nullptr, dxd_rows);
  }
  // dH = gd W2^T stored plain (in dA's buffer); one pass forms dA = dH *
  // silu'(a) as two FP16 terms per row; W1 [E][d][h] is K-major for dA W1^T
  st = launch<kModeNN, kEpiStore, kBF16S>(gq, wq, R, E, d, h, dA, nullptr, nullptr, offsets, err, stream, 0, nullptr,
                                           nullptr, nullptr, gd_scale, winv);
  if (st != JANUS_OK) return st;
  st = act_split_f16<kActDSilu>(dA, act, R, h, second->h16, second->hscale, stream);
  if (st != JANUS_OK) return st;
  if (!weights_presplit) st = split_weights_f16(w1, E, h, d, false, second->w16, second->winv, stream);
  if (st != JANUS_OK) return st;
  return launch<kModeNN, kEpiStore, kBF16S>(reinterpret_cast<const float*>(second->h16),
                                            reinterpret_cast<const float*>(second->w16), R, E, h, d, dxd, nullptr,
                                            nullptr, offsets, err, stream, 0, nullptr, nullptr, dxd_rows,
                                            second->hscale, second->winv);
}

janus_status expert_ffn_vjp(const float* xd, const float* gd, const float* act_in, float* A,
                            const int32_t* offsets, int32_t E, int64_t R, int32_t d, int32_t h,
                            const float* w1, const float* w2, float* dxd, float* dA, int32_t* err,
                            cudaStream_t stream, float* const* dxd_rows) {
  janus_status st;
  if (!act_in) {
    st = launch<kModeNN, kEpiStore>(xd, w1, R, E, d, h, A, nullptr, nullptr, offsets, err, stream);
    if (st != JANUS_OK) return st;
  }
  st = launch<kModeNT, kEpiDSilu>(gd, w2, R, E, d, h, dA, nullptr, A, offsets, err, stream);
  if (st != JANUS_OK) return st;
  return launch<kModeNT, kEpiStore>(dA, w1, R, E, h, d, dxd, nullptr, nullptr, offsets, err, stream, 0, nullptr,
                                    nullptr, dxd_rows);
}

janus_status expert_ffn_weight_grad(const float* xd, const float* gd, const float* act_in, float* A,
                                    const int32_t* offsets, int32_t E, int64_t R, int32_t d, int32_t h,
                                    const float* w1, const float* w2, float* dw1, float* dw2, float* dA,
                                    float* H, int32_t* err, cudaStream_t stream) {
  janus_status st;
  if (!act_in) {
    st = launch<kModeNN, kEpiStore>(xd, w1, R, E, d, h, A, nullptr, nullptr, offsets, err, stream);
    if (st != JANUS_OK) return st;
  }
  // dA = (gd W2^T) * silu'(a), and H = silu(a)
  st = launch<kModeNT, kEpiDSilu>(gd, w2, R, E, d, h, dA, H, A, offsets, err, stream);
  if (st != JANUS_OK) return st;
  // dW1 = xd^T dA [d][h]: the product dA^T xd, stored transposed
  st = launch<kModeTN, kEpiStore>(dA, xd, R, E, 0, d, dw1, nullptr, nullptr, offsets, err, stream, h);
  if (st != JANUS_OK) return st;
  // dW2 = H^T gd [h][d]
  return launch<kModeTN, kEpiStore>(gd, H, R, E, 0, h, dw2, nullptr, nullptr, offsets, err, stream, d);
}

janus_status expert_ffn_vjp_vjp(const float* xd, const float* gd, const float* vd, const float* act_in, float* A,
                                const int32_t* offsets, int32_t E, int64_t R, int32_t d, int32_t h,
                                const float* w1, const float* w2, float* d_xd, float* d_gd, float* dw1,
                                float* dw2, float* dh, float* t1, float* t2, float* u, int32_t* err,
                                cudaStream_t stream) {
  janus_status st;
  if (!act_in) {
    st = launch<kModeNN, kEpiStore>(xd, w1, R, E, d, h, A, nullptr, nullptr, offsets, err, stream);
    if (st != JANUS_OK) return st;
  }
  // dh = gd W2^T
  st = launch<kModeNT, kEpiStore>(gd, w2, R, E, d, h, dh, nullptr, nullptr, offsets, err, stream);
  if (st != JANUS_OK) return st;
  // ub = vd W1 -> t1 = ub silu'(a), t2 = ub dh silu''(a), u = dh silu'(a)
  st = launch<kModeNN, kEpiD2>(vd, w1, R, E, d, h, t1, t2, A, offsets, err, stream, 0, dh, dw1 ? u : nullptr);
  if (st != JANUS_OK) return st;
  // d_gd = t1 W2, d_xd = t2 W1^T
  st = launch<kModeNN, kEpiStore>(t1, w2, R, E, h, d, d_gd, nullptr, nullptr, offsets, err, stream);
  if (st != JANUS_OK) return st;
  st = launch<kModeNT, kEpiStore>(t2, w1, R, E, h, d, d_xd, nullptr, nullptr, offsets, err, stream);
  if (st != JANUS_OK || !dw1) return st;
  // dW2 = t1^T gd;  dW1 = vd^T u + xd^T t2
  // (each product stored transposed: the first operand's columns index the
  // output's columns)
  st = launch<kModeTN, kEpiStore>(gd, t1, R, E, 0, h, dw2, nullptr, nullptr, offsets, err, stream, d);
  if (st != JANUS_OK) return st;
  st = launch<kModeTN, kEpiStore>(u, vd, R, E, 0, d, dw1, nullptr, nullptr, offsets, err, stream, h);
  if (st != JANUS_OK) return st;
  return launch<kModeTN, kEpiAccum>(t2, xd, R, E, 0, d, dw1, nullptr, nullptr, offsets, err, stream, h);
}

}  // namespace tc
}  // namespace janus
