// Grouped FP32 GEMM on the CUDA cores (FFMA), used by the expert MLP in
// JANUS_FFN_FP32_SIMT mode.  Internal header, included by expert_ffn.cu.
//
//   C[p, :] = epilogue( A[p, :] * B_e )   for rows p in [offsets[e], offsets[e+1])
//
// A is row-major [R, Kd]; B_e is expert e's weight, either stored [Kd][N]
// (kNT = false, "x W") or [N][Kd] (kNT = true, "x W^T").
//
// Tiling: 128x128 output tile, k-step 16, 256 threads, 8x8 outputs per
// thread as two 4x4 quadrants in each direction (conflict-free 128-bit shared
// loads), global->register->shared double buffering with one barrier per
// k-step.  A persistent grid walks a device-side tile list built from
// `offsets` (expert-major, then m-tile, then n-tile), so concurrently running
// CTAs share the same expert's weights and A rows in L2 and the host never
// reads the routing result.
#pragma once

#include "common.cuh"

namespace janus {
namespace simt {

constexpr int BM = 128, BN = 128, BK = 16, kThreads = 256;

enum Epilogue : int {
  kEpiStore = 0,   // C = acc
  kEpiSilu = 1,    // C2 = acc (if C2), C = silu(acc)
  kEpiDSilu = 2,   // C = acc * silu'(aux)
  kEpiD2 = 3       // second-order pass, acc = v W1, aux = a, aux2 = dh:
                   //   C = acc * silu'(a), C2 = acc * dh * silu''(a), C3 = dh * silu'(a) (if C3)
};

struct Args {
  const float* A;
  const float* B;
  int64_t b_expert_stride;   // elements between experts' weights
  float* C;
  float* C2;                 // optional second output (pre-activation)
  const float* aux;          // pre-activation for kEpiDSilu / kEpiD2, [R, N]
  const float* aux2;         // kEpiD2: dh = gd W2^T, [R, N]
  float* C3;                 // kEpiD2: optional third output
  float* const* c_rows;      // kEpiStore: if set, row p is stored at c_rows[p] (not C + p N)
  const int32_t* offsets;
  int E;
  int Kd;                    // reduction length
  int N;                     // output columns
  int64_t rows;              // rows of A and C (offsets[E] <= rows; checked in debug builds)
  int32_t* dbg;              // debug builds: fault word for a bad offsets array
};

__device__ __forceinline__ float silu_f(float a) { return a / (1.0f + expf(-a)); }
__device__ __forceinline__ float dsilu_f(float a) {
  const float s = 1.0f / (1.0f + expf(-a));
  return s * (1.0f + a * (1.0f - s));
}
// silu''(a) = sig (1 - sig) (2 + a (1 - 2 sig))
__device__ __forceinline__ void d2_terms(float acc, float a, float dh, float& t1, float& t2, float& u) {
  const float s = 1.0f / (1.0f + expf(-a));
  const float s1 = s * (1.0f + a * (1.0f - s));
  const float s2 = s * (1.0f - s) * (2.0f + a * (1.0f - 2.0f * s));
  t1 = acc * s1;
  t2 = acc * dh * s2;
  u = dh * s1;
}

// Expert-major tile list: tile_start[e] = sum_{e'<e} ceil(count_e'/BM).
struct TileMap {
  int off[kMaxExperts + 1];
  int start[kMaxExperts + 1];
};

__device__ __forceinline__ void build_tile_map(TileMap& tm, const int32_t* offsets, int E, int64_t rows,
                                               int32_t* dbg) {
  for (int e = threadIdx.x; e <= E; e += blockDim.x) tm.off[e] = offsets[e];
  __syncthreads();
  if (threadIdx.x == 0) {
    if (kDebug) {
      // offsets must be non-decreasing inside [0, rows]; otherwise every
      // expert is treated as empty (no tile touches memory) and the fault recorded
      bool ok = tm.off[0] >= 0 && tm.off[E] <= rows;
      for (int e = 0; e < E; ++e) ok = ok && tm.off[e + 1] >= tm.off[e];
      if (!ok) {
        debug_fault(dbg);
        for (int e = 0; e <= E; ++e) tm.off[e] = 0;
      }
    }
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      tm.start[e] = acc;
      acc += (tm.off[e + 1] - tm.off[e] + BM - 1) / BM;
    }
    tm.start[E] = acc;
  }
  __syncthreads();
}

__device__ __forceinline__ int find_expert(const TileMap& tm, int E, int mt) {
  int lo = 0, hi = E;          // invariant: start[lo] <= mt < start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tm.start[mid] <= mt) lo = mid; else hi = mid;
  }
  return lo;
}

template <bool kNT, int kEpi>
__global__ void __launch_bounds__(kThreads, 2) grouped_gemm_kernel(Args args) {
  __shared__ __align__(16) float As[2][BK][BM];
  __shared__ __align__(16) float Bs[2][BK][BN];
  __shared__ TileMap tm;
  build_tile_map(tm, args.offsets, args.E, args.rows, args.dbg);

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int Kd = args.Kd, N = args.N;
  const int n_tiles_n = (N + BN - 1) / BN;
  const int total = tm.start[args.E] * n_tiles_n;
  const int nk = (Kd + BK - 1) / BK;

  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const int mt = tile / n_tiles_n, nt = tile % n_tiles_n;
    const int e = find_expert(tm, args.E, mt);
    const int m0 = tm.off[e] + (mt - tm.start[e]) * BM;
    const int m_end = tm.off[e + 1];
    const int n0 = nt * BN;
    const float* A = args.A;
    const float* B = args.B + (int64_t)e * args.b_expert_stride;

    float4 ra[2], rb[2];
    // A (and B when kNT): element (row r, k-quad q) at idx = tid + j*256,
    // r = idx % 128, q = idx / 128; consecutive lanes -> consecutive rows, so
    // the transposed shared stores are conflict-free.
    auto load_tile = [&](int kt) {
      const int k0 = kt * BK;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = tid + j * kThreads;
        const int r = idx % BM, q = idx / BM;
        const int kk = k0 + q * 4;
        const bool ok = (m0 + r < m_end) && (kk < Kd);
        ra[j] = ok ? __ldg(reinterpret_cast<const float4*>(A + (int64_t)(m0 + r) * Kd + kk))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = tid + j * kThreads;
        if (kNT) {
          const int n = idx % BN, q = idx / BN;
          const int kk = k0 + q * 4;
          const bool ok = (n0 + n < N) && (kk < Kd);
          rb[j] = ok ? __ldg(reinterpret_cast<const float4*>(B + (int64_t)(n0 + n) * Kd + kk))
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          const int kr = idx / (BN / 4), nq = idx % (BN / 4);
          const bool ok = (k0 + kr < Kd) && (n0 + nq * 4 < N);
          rb[j] = ok ? __ldg(reinterpret_cast<const float4*>(B + (int64_t)(k0 + kr) * N + n0 + nq * 4))
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    };
    auto store_tile = [&](int buf) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = tid + j * kThreads;
        const int r = idx % BM, q = idx / BM;
        As[buf][q * 4 + 0][r] = ra[j].x;
        As[buf][q * 4 + 1][r] = ra[j].y;
        As[buf][q * 4 + 2][r] = ra[j].z;
        As[buf][q * 4 + 3][r] = ra[j].w;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = tid + j * kThreads;
        if (kNT) {
          const int n = idx % BN, q = idx / BN;
          Bs[buf][q * 4 + 0][n] = rb[j].x;
          Bs[buf][q * 4 + 1][n] = rb[j].y;
          Bs[buf][q * 4 + 2][n] = rb[j].z;
          Bs[buf][q * 4 + 3][n] = rb[j].w;
        } else {
          const int kr = idx / (BN / 4), nq = idx % (BN / 4);
          *reinterpret_cast<float4*>(&Bs[buf][kr][nq * 4]) = rb[j];
        }
      }
    };

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    load_tile(0);
    store_tile(0);
    __syncthreads();
    for (int kt = 0; kt < nk; ++kt) {
      const int cur = kt & 1;
      if (kt + 1 < nk) load_tile(kt + 1);
#pragma unroll
      for (int k = 0; k < BK; ++k) {
        const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][k][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][k][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][k][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][k][64 + tx * 4]);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      if (kt + 1 < nk) store_tile(cur ^ 1);
      __syncthreads();
    }

    // epilogue
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
      if (r >= m_end) continue;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int c = n0 + g * 64 + tx * 4;
        if (c >= N) continue;
        float4 v = make_float4(acc[i][g * 4 + 0], acc[i][g * 4 + 1], acc[i][g * 4 + 2], acc[i][g * 4 + 3]);
        const int64_t o = (int64_t)r * N + c;
        if (kEpi == kEpiSilu) {
          if (args.C2) *reinterpret_cast<float4*>(args.C2 + o) = v;
          v = make_float4(silu_f(v.x), silu_f(v.y), silu_f(v.z), silu_f(v.w));
        } else if (kEpi == kEpiDSilu) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(args.aux + o));
          v = make_float4(v.x * dsilu_f(a.x), v.y * dsilu_f(a.y), v.z * dsilu_f(a.z), v.w * dsilu_f(a.w));
          if (args.C2)   // H = silu(a) for the second weight gradient
            *reinterpret_cast<float4*>(args.C2 + o) = make_float4(silu_f(a.x), silu_f(a.y), silu_f(a.z), silu_f(a.w));
        } else if (kEpi == kEpiD2) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(args.aux + o));
          const float4 g = __ldg(reinterpret_cast<const float4*>(args.aux2 + o));
          float4 t2, u;
          d2_terms(v.x, a.x, g.x, v.x, t2.x, u.x);
          d2_terms(v.y, a.y, g.y, v.y, t2.y, u.y);
          d2_terms(v.z, a.z, g.z, v.z, t2.z, u.z);
          d2_terms(v.w, a.w, g.w, v.w, t2.w, u.w);
          *reinterpret_cast<float4*>(args.C2 + o) = t2;
          if (args.C3) *reinterpret_cast<float4*>(args.C3 + o) = u;
        }
        float* dst = (kEpi == kEpiStore && args.c_rows) ? args.c_rows[r] + c : args.C + o;
        *reinterpret_cast<float4*>(dst) = v;
      }
    }
  }
  // rows stored through c_rows may sit in another GPU's memory
  if (kEpi == kEpiStore && args.c_rows) __threadfence_system();
}

// Per-expert weight gradient on the CUDA cores:
//   C[e] [M,N] = sum over rows p of expert e of X[p, :]^T Y[p, :]
// X [R,M] and Y [R,N] row-major; both tiles are loaded along their contiguous
// dimension (k = row), rows past the expert's segment are zero; an expert
// without rows gets a zero matrix.  Same 128x128x16 register tiling.
struct TnArgs {
  const float* X;
  const float* Y;
  float* C;
  const int32_t* offsets;
  int E, M, N;
  int accumulate;   // nonzero: C += X^T Y
  int64_t rows;     // rows of X and Y (offsets[E] <= rows; checked in debug builds)
  int32_t* dbg;     // debug builds: fault word for a bad offsets array
};

__global__ void __launch_bounds__(kThreads, 2) grouped_tn_kernel(TnArgs args) {
  __shared__ __align__(16) float As[2][BK][BM];
  __shared__ __align__(16) float Bs[2][BK][BN];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int M = args.M, N = args.N;
  const int n_tm = (M + BM - 1) / BM, n_tn = (N + BN - 1) / BN;
  const int total = args.E * n_tm * n_tn;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const int e = tile / (n_tm * n_tn);
    const int rem = tile % (n_tm * n_tn);
    const int m0 = (rem / n_tn) * BM, n0 = (rem % n_tn) * BN;
    int p0 = args.offsets[e], p1 = args.offsets[e + 1];
    if (kDebug && !(p0 >= 0 && p1 >= p0 && p1 <= args.rows)) {
      // a bad segment is treated as empty (zero gradient, nothing read)
      if (tid == 0) debug_fault(args.dbg);
      p0 = p1 = 0;
    }
    const int nk = (p1 - p0 + BK - 1) / BK;
    float4 ra[2], rb[2];
    auto load_tile = [&](int kt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = tid + j * kThreads;
        const int kr = idx / (BM / 4), q = idx % (BM / 4);
        const int p = p0 + kt * BK + kr;
        const bool okr = p < p1;
        ra[j] = (okr && m0 + q * 4 < M) ? __ldg(reinterpret_cast<const float4*>(args.X + (int64_t)p * M + m0 + q * 4))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
        rb[j] = (okr && n0 + q * 4 < N) ? __ldg(reinterpret_cast<const float4*>(args.Y + (int64_t)p * N + n0 + q * 4))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    auto store_tile = [&](int buf) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = tid + j * kThreads;
        const int kr = idx / (BM / 4), q = idx % (BM / 4);
        *reinterpret_cast<float4*>(&As[buf][kr][q * 4]) = ra[j];
        *reinterpret_cast<float4*>(&Bs[buf][kr][q * 4]) = rb[j];
      }
    };
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    if (nk > 0) {
      load_tile(0);
      store_tile(0);
    }
    __syncthreads();
    for (int kt = 0; kt < nk; ++kt) {
      const int cur = kt & 1;
      if (kt + 1 < nk) load_tile(kt + 1);
#pragma unroll
      for (int k = 0; k < BK; ++k) {
        const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][k][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][k][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][k][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][k][64 + tx * 4]);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      if (kt + 1 < nk) store_tile(cur ^ 1);
      __syncthreads();
    }
    float* C = args.C + (int64_t)e * M * N;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
      if (r >= M) continue;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int c = n0 + g * 64 + tx * 4;
        if (c >= N) continue;
        float4 v = make_float4(acc[i][g * 4 + 0], acc[i][g * 4 + 1], acc[i][g * 4 + 2], acc[i][g * 4 + 3]);
        float4* dst = reinterpret_cast<float4*>(C + (int64_t)r * N + c);
        if (args.accumulate) {
          const float4 o = *dst;
          v = make_float4(o.x + v.x, o.y + v.y, o.z + v.z, o.w + v.w);
        }
        *dst = v;
      }
    }
  }
}

}  // namespace simt
}  // namespace janus
