// Janus element-routed MoE layer + edge aggregation: plain CPU ORACLE.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
// libjanus.so and its Python binding) may link, load or call this file; only
// the test suite, the package's smoke() check and the benchmark's CPU-baseline
// leg do.  It shares no source, header, table or helper with the CUDA path.
//
// Every function is the plain definition of one step of the hot path, written
// as slow, obviously-correct loops with FP64 accumulation and FP32 outputs.
// Sources (web pages on the method; cited by title and section):
//   [Review]    "Breaking the Training Barrier of Billion-Parameter Universal
//               Machine Learning Interatomic Potentials" (xllm-io paper review)
//   [News]      "11.5B参数、1.2EFLOPS、训练从数周压到数小时" (ScienceAI article)
//   [Blueprint] "MatRIS-MoE与Janus框架：构建百亿参数通用机器学习原子间势"
//               (ksqn.cn post; speculative, used only where the others are silent)
//
// Readings taken where the pages are silent (each pinned by a test under
// tests/ that does not call back into this file's formula):
//   * top-K order: descending logit, ties to the lower expert id;
//   * gate weights: softmax over the K selected logits only;
//   * stable permutation: key = expert, then flat slot s = i*K + k ascending;
//   * per-type FP16 scale: the smallest power of two 2^e with amax <= 65504*2^e,
//     e clamped to [-126, 127]; scale 1 for an all-zero or absent type;
//   * expert = bias-free Linear(d,h) -> SiLU -> Linear(h,d), weights x*W;
//   * combine sums k ascending; edge aggregation is a plain sum.
//
// Parity pins live in tests/test_oracle_*.py.  No part is "parity unpinned".
//
// Build: g++ -O2 -fopenmp -ffp-contract=off -shared -fPIC (see oracle/build.py).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// ---------------------------------------------------------------------------
// IEEE-754 binary16 conversion, round-to-nearest-even, written from the
// format's definition: 1 sign bit, 5 exponent bits (bias 15), 10 fraction
// bits; subnormals are multiples of 2^-24; the largest finite value is 65504.
// ---------------------------------------------------------------------------
uint16_t orc_fp16_from_double(double x) {
  uint16_t sign = std::signbit(x) ? 0x8000u : 0u;
  double a = std::fabs(x);
  if (std::isnan(x)) return (uint16_t)(sign | 0x7E00u);
  if (a == 0.0) return sign;
  int ex;
  std::frexp(a, &ex);          // a = m * 2^ex, m in [0.5, 1)
  int E = ex - 1;              // a = 1.f * 2^E
  if (E < -14) {
    // subnormal range: value = q * 2^-24, q integer in [0, 1024]
    double q = std::nearbyint(std::ldexp(a, 24));  // ties-to-even (default mode)
    // q == 1024 is the smallest normal number 2^-14: bits 0x0400, same encoding
    return (uint16_t)(sign | (uint16_t)q);
  }
  double q = std::nearbyint(std::ldexp(a, 10 - E));  // in [1024, 2048]
  if (q >= 2048.0) { q = 1024.0; E += 1; }
  if (E > 15) return (uint16_t)(sign | 0x7C00u);      // overflow -> inf
  return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(q - 1024.0));
}

double orc_fp16_to_double(uint16_t b) {
  int sign = (b >> 15) & 1;
  int e = (b >> 10) & 0x1F;
  int f = b & 0x3FF;
  double v;
  if (e == 0) v = std::ldexp((double)f, -24);
  else if (e == 31) v = f ? NAN : INFINITY;
  else v = std::ldexp(1024.0 + f, e - 25);
  return sign ? -v : v;
}

// ---------------------------------------------------------------------------
// Routing.  [Review] §3.2 sparse MoE design: each element type activates its
// own top-K experts; [News] "兼顾物理先验与扩展性的模型架构": routing depends
// on the element type, not on coordinates.  JIT planning ([News]
// "兼顾 MoE 稀疏执行与二阶反传的训练框架") counts the per-expert token load.
// Brute force per atom: sort all E logits of the atom's gate row.
// Returns 0, or -1 if a type id lies outside [0, n_types).
// ---------------------------------------------------------------------------
int orc_route(const int32_t* types, int64_t n_atoms, const float* gate,
              int32_t n_types, int32_t n_experts, int32_t top_k,
              int32_t* topk_expert, float* topk_weight, int32_t* counts,
              int32_t* offsets, int32_t* perm, int32_t* slot_of) {
  const int E = n_experts, K = top_k;
  for (int64_t i = 0; i < n_atoms; ++i)
    if (types[i] < 0 || types[i] >= n_types) return -1;

  std::vector<int> order(E);
  for (int64_t i = 0; i < n_atoms; ++i) {
    const float* g = gate + (int64_t)types[i] * E;
    for (int e = 0; e < E; ++e) order[e] = e;
    std::sort(order.begin(), order.end(), [g](int a, int b) {
      if (g[a] != g[b]) return g[a] > g[b];
      return a < b;
    });
    // softmax over the selected logits, shifted by the largest one
    double l0 = (double)g[order[0]];
    double z = 0.0;
    for (int k = 0; k < K; ++k) z += std::exp((double)g[order[k]] - l0);
    for (int k = 0; k < K; ++k) {
      topk_expert[i * K + k] = order[k];
      topk_weight[i * K + k] = (float)(std::exp((double)g[order[k]] - l0) / z);
    }
  }
  const int64_t R = n_atoms * K;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t s = 0; s < R; ++s) counts[topk_expert[s]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  // stable counting sort of the flat slots by expert
  int64_t p = 0;
  for (int e = 0; e < E; ++e)
    for (int64_t s = 0; s < R; ++s)
      if (topk_expert[s] == e) perm[p++] = (int32_t)s;
  for (int64_t q = 0; q < R; ++q) slot_of[perm[q]] = (int32_t)q;
  return 0;
}

// ---------------------------------------------------------------------------
// Dispatch.  [Review] §3.5 (CNIS, MoE dispatch/combine): tokens are copied
// into an expert-grouped buffer.  Xd[p,:] = X[perm[p]/K,:], optionally
// multiplied by the gate weight of slot perm[p] (used by the input VJP).
// ---------------------------------------------------------------------------
void orc_dispatch(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                  const int32_t* perm, const float* topk_weight, float* xd) {
  const int64_t R = n_atoms * top_k;
  for (int64_t p = 0; p < R; ++p) {
    const int64_t s = perm[p];
    const int64_t i = s / top_k;
    for (int j = 0; j < d; ++j) {
      double v = (double)x[i * d + j];
      if (topk_weight) v *= (double)topk_weight[s];
      xd[p * d + j] = (float)v;
    }
  }
}

// ---------------------------------------------------------------------------
// Atom-type-aware FP16 packing.  [Review] §3.5 CNIS "Atom-type-aware FP16压缩":
// after routing, dispatch-buffer tokens are grouped by atom type, quantised
// with one scale per type, sent as FP16 and dequantised afterwards (half the
// FP32 volume).  Reading: per-type absmax, power-of-two scale (see header).
// payload is [R,d] binary16 bits in dispatch order, scale is [T].
// Returns 0, -1 for a bad type id, -2 for a non-finite feature of a present type.
// ---------------------------------------------------------------------------
static int scale_exponent(double amax) {
  if (amax == 0.0) return 0;
  int ex;
  double m = std::frexp(amax, &ex);         // amax = m * 2^ex
  int e = ex - 16 + ((m > 65504.0 / 65536.0) ? 1 : 0);
  if (e < -126) e = -126;
  if (e > 127) e = 127;
  return e;
}

int orc_quant_by_type(const float* x, int64_t n_atoms, int32_t d, int32_t top_k,
                      const int32_t* types, int32_t n_types, const int32_t* perm,
                      uint16_t* payload, float* scale) {
  std::vector<double> amax(n_types, 0.0);
  for (int64_t i = 0; i < n_atoms; ++i) {
    if (types[i] < 0 || types[i] >= n_types) return -1;
    for (int j = 0; j < d; ++j) {
      double a = std::fabs((double)x[i * d + j]);
      if (!std::isfinite(a)) return -2;
      amax[types[i]] = std::max(amax[types[i]], a);
    }
  }
  std::vector<int> ex(n_types);
  for (int t = 0; t < n_types; ++t) {
    ex[t] = scale_exponent(amax[t]);
    scale[t] = (float)std::ldexp(1.0, ex[t]);
  }
  const int64_t R = n_atoms * top_k;
  for (int64_t p = 0; p < R; ++p) {
    const int64_t i = perm[p] / top_k;
    const int t = types[i];
    for (int j = 0; j < d; ++j)
      payload[p * d + j] = orc_fp16_from_double(std::ldexp((double)x[i * d + j], -ex[t]));
  }
  return 0;
}

void orc_dequant_by_type(const uint16_t* payload, int64_t n_atoms, int32_t d,
                         int32_t top_k, const int32_t* types, const int32_t* perm,
                         const float* scale, float* xd) {
  const int64_t R = n_atoms * top_k;
  for (int64_t p = 0; p < R; ++p) {
    const int t = types[perm[p] / top_k];
    for (int j = 0; j < d; ++j)
      xd[p * d + j] = (float)(orc_fp16_to_double(payload[p * d + j]) * (double)scale[t]);
  }
}

// ---------------------------------------------------------------------------
// Expert MLP.  [Review] §3.1 Table II gives the MLP hidden size (= feature
// size); the expert is read as bias-free Linear(d,h) -> SiLU -> Linear(h,d).
// Rows [offsets[e], offsets[e+1]) of the dispatch buffer belong to expert e.
// W1 is [E,d,h], W2 is [E,h,d], row-major; y = silu(x W1) W2.
// rows == NULL: all R rows, outputs [R,*].  Otherwise only the listed rows,
// outputs compacted to [n_sel,*].  act (nullable) receives a = x W1.
// ---------------------------------------------------------------------------
static int expert_of_row(const int32_t* offsets, int32_t n_experts, int64_t p) {
  int e = 0;
  while (e + 1 < n_experts && offsets[e + 1] <= p) ++e;
  return e;
}

static double silu(double a) { return a / (1.0 + std::exp(-a)); }

void orc_expert_ffn_fwd(const float* xd, const int32_t* offsets, int32_t n_experts,
                        int64_t n_rows, int32_t d, int32_t h, const float* w1,
                        const float* w2, const int64_t* rows, int64_t n_sel,
                        float* yd, float* act) {
  const int64_t n_out = rows ? n_sel : n_rows;
#pragma omp parallel
  {
    std::vector<double> a(h), y(d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t q = 0; q < n_out; ++q) {
      const int64_t p = rows ? rows[q] : q;
      const int e = expert_of_row(offsets, n_experts, p);
      const float* W1 = w1 + (int64_t)e * d * h;
      const float* W2 = w2 + (int64_t)e * h * d;
      std::fill(a.begin(), a.end(), 0.0);
      for (int k = 0; k < d; ++k) {
        const double xk = xd[p * d + k];
        for (int j = 0; j < h; ++j) a[j] += xk * (double)W1[(int64_t)k * h + j];
      }
      std::fill(y.begin(), y.end(), 0.0);
      for (int j = 0; j < h; ++j) {
        const double hj = silu(a[j]);
        for (int c = 0; c < d; ++c) y[c] += hj * (double)W2[(int64_t)j * d + c];
      }
      for (int c = 0; c < d; ++c) yd[q * d + c] = (float)y[c];
      if (act)
        for (int j = 0; j < h; ++j) act[q * h + j] = (float)a[j];
    }
  }
}

// ---------------------------------------------------------------------------
// Input VJP of the expert MLP.  [Review] §3.3 and [News]: forces and stress are
// autodiff gradients of the energy (conservative training), so the layer's
// gradient w.r.t. its input is on the path.  For one row with upstream g:
//   dHh = W2 g,  dA = dHh * silu'(a),  dx = W1 dA,
//   silu'(a) = sig(a) (1 + a (1 - sig(a))).   a is recomputed in FP64.
// ---------------------------------------------------------------------------
void orc_expert_ffn_vjp(const float* xd, const float* gd, const int32_t* offsets,
                        int32_t n_experts, int64_t n_rows, int32_t d, int32_t h,
                        const float* w1, const float* w2, const int64_t* rows,
                        int64_t n_sel, float* dxd) {
  const int64_t n_out = rows ? n_sel : n_rows;
#pragma omp parallel
  {
    std::vector<double> a(h), da(h), dx(d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t q = 0; q < n_out; ++q) {
      const int64_t p = rows ? rows[q] : q;
      const int e = expert_of_row(offsets, n_experts, p);
      const float* W1 = w1 + (int64_t)e * d * h;
      const float* W2 = w2 + (int64_t)e * h * d;
      std::fill(a.begin(), a.end(), 0.0);
      for (int k = 0; k < d; ++k) {
        const double xk = xd[p * d + k];
        for (int j = 0; j < h; ++j) a[j] += xk * (double)W1[(int64_t)k * h + j];
      }
      for (int j = 0; j < h; ++j) {
        double dh = 0.0;
        for (int c = 0; c < d; ++c) dh += (double)W2[(int64_t)j * d + c] * (double)gd[p * d + c];
        const double sg = 1.0 / (1.0 + std::exp(-a[j]));
        da[j] = dh * sg * (1.0 + a[j] * (1.0 - sg));
      }
      for (int k = 0; k < d; ++k) {
        double acc = 0.0;
        for (int j = 0; j < h; ++j) acc += (double)W1[(int64_t)k * h + j] * da[j];
        dx[k] = acc;
      }
      for (int k = 0; k < d; ++k) dxd[q * d + k] = (float)dx[k];
    }
  }
}

// ---------------------------------------------------------------------------
// Expert weight gradients (the layer's parameters, needed by force training:
// [Review] section 3.3).  With L = sum_p <Yd[p,:], Gd[p,:]> over the rows of
// expert e and a = x W1, hh = silu(a):
//   dW2[e][j][c] = sum_p hh[p][j] * gd[p][c]
//   dW1[e][k][j] = sum_p x[p][k] * dA[p][j],  dA = (W2 g) * silu'(a)
// An expert with no rows gets zero gradients.  a and dA are recomputed in FP64.
// ---------------------------------------------------------------------------
void orc_expert_ffn_weight_grad(const float* xd, const float* gd, const int32_t* offsets,
                                int32_t n_experts, int32_t d, int32_t h, const float* w1,
                                const float* w2, float* dw1, float* dw2) {
  for (int e = 0; e < n_experts; ++e) {
    const float* W1 = w1 + (int64_t)e * d * h;
    const float* W2 = w2 + (int64_t)e * h * d;
    const int64_t p0 = offsets[e], n = offsets[e + 1] - offsets[e];
    // per row of the expert: hh = silu(a) and dA, in FP64
    std::vector<double> hh((size_t)n * h), da((size_t)n * h);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      const int64_t p = p0 + r;
      std::vector<double> a(h, 0.0);
      for (int k = 0; k < d; ++k) {
        const double xk = xd[p * d + k];
        for (int j = 0; j < h; ++j) a[j] += xk * (double)W1[(int64_t)k * h + j];
      }
      for (int j = 0; j < h; ++j) {
        double dh = 0.0;
        for (int c = 0; c < d; ++c) dh += (double)W2[(int64_t)j * d + c] * (double)gd[p * d + c];
        const double sg = 1.0 / (1.0 + std::exp(-a[j]));
        hh[(size_t)r * h + j] = a[j] * sg;
        da[(size_t)r * h + j] = dh * sg * (1.0 + a[j] * (1.0 - sg));
      }
    }
    // sums over the expert's rows in row order
#pragma omp parallel for schedule(dynamic, 4)
    for (int k = 0; k < d; ++k) {
      std::vector<double> acc(h, 0.0);
      for (int64_t r = 0; r < n; ++r) {
        const double xk = xd[(p0 + r) * d + k];
        for (int j = 0; j < h; ++j) acc[j] += xk * da[(size_t)r * h + j];
      }
      for (int j = 0; j < h; ++j) dw1[(int64_t)e * d * h + (int64_t)k * h + j] = (float)acc[j];
    }
#pragma omp parallel for schedule(dynamic, 4)
    for (int j = 0; j < h; ++j) {
      std::vector<double> acc(d, 0.0);
      for (int64_t r = 0; r < n; ++r) {
        const double hj = hh[(size_t)r * h + j];
        for (int c = 0; c < d; ++c) acc[c] += hj * (double)gd[(p0 + r) * d + c];
      }
      for (int c = 0; c < d; ++c) dw2[(int64_t)e * h * d + (int64_t)j * d + c] = (float)acc[c];
    }
  }
}

// ---------------------------------------------------------------------------
// Second-order pass: the VJP of the input VJP.  Force training ([Review]
// section 3.3: forces are -dE/dx, fitted by a loss) differentiates the forces,
// so the gradient of a loss on the layer's input VJP is on the path.  Per row,
// with a = x W1, sig = sigmoid(a):
//   s1 = silu'(a)  = sig (1 + a (1 - sig))
//   s2 = silu''(a) = sig (1 - sig) (2 + a (1 - 2 sig))
//   dh = W2 g,  u = dh * s1,  dx = W1 u                (the input VJP)
// and for L = <dx, v> with v the cotangent of dx:
//   ub = W1^T v,  t1 = ub * s1,  t2 = ub * dh * s2
//   dL/dx = W1 t2,  dL/dg = W2^T t1
//   dL/dW1[k][j] = sum_p v[k] u[j] + x[k] t2[j],  dL/dW2[j][c] = sum_p t1[j] g[c]
// Everything per row in FP64 (a recomputed), outputs rounded once to FP32.
// ---------------------------------------------------------------------------
namespace {
struct RowTerms {
  std::vector<double> a, dh, s1, s2, u, t1, t2;
  explicit RowTerms(int h) : a(h), dh(h), s1(h), s2(h), u(h), t1(h), t2(h) {}
  void compute(const float* x, const float* g, const float* v, const float* W1, const float* W2, int d,
               int h) {
    std::fill(a.begin(), a.end(), 0.0);
    for (int k = 0; k < d; ++k) {
      const double xk = x[k];
      for (int j = 0; j < h; ++j) a[j] += xk * (double)W1[(int64_t)k * h + j];
    }
    for (int j = 0; j < h; ++j) {
      double acc = 0.0, ub = 0.0;
      for (int c = 0; c < d; ++c) acc += (double)W2[(int64_t)j * d + c] * (double)g[c];
      for (int k = 0; k < d; ++k) ub += (double)W1[(int64_t)k * h + j] * (double)v[k];
      const double sg = 1.0 / (1.0 + std::exp(-a[j]));
      dh[j] = acc;
      s1[j] = sg * (1.0 + a[j] * (1.0 - sg));
      s2[j] = sg * (1.0 - sg) * (2.0 + a[j] * (1.0 - 2.0 * sg));
      u[j] = dh[j] * s1[j];
      t1[j] = ub * s1[j];
      t2[j] = ub * dh[j] * s2[j];
    }
  }
};
}  // namespace

void orc_expert_ffn_vjp_vjp(const float* xd, const float* gd, const float* vd, const int32_t* offsets,
                            int32_t n_experts, int64_t n_rows, int32_t d, int32_t h, const float* w1,
                            const float* w2, const int64_t* rows, int64_t n_sel, float* d_xd, float* d_gd) {
  const int64_t n_out = rows ? n_sel : n_rows;
#pragma omp parallel
  {
    RowTerms t(h);
#pragma omp for schedule(dynamic, 1)
    for (int64_t q = 0; q < n_out; ++q) {
      const int64_t p = rows ? rows[q] : q;
      const int e = expert_of_row(offsets, n_experts, p);
      const float* W1 = w1 + (int64_t)e * d * h;
      const float* W2 = w2 + (int64_t)e * h * d;
      t.compute(xd + p * d, gd + p * d, vd + p * d, W1, W2, d, h);
      for (int k = 0; k < d; ++k) {
        double acc = 0.0;
        for (int j = 0; j < h; ++j) acc += (double)W1[(int64_t)k * h + j] * t.t2[j];
        d_xd[q * d + k] = (float)acc;
      }
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int j = 0; j < h; ++j) acc += (double)W2[(int64_t)j * d + c] * t.t1[j];
        d_gd[q * d + c] = (float)acc;
      }
    }
  }
}

// Weight part of the second-order pass (sums over each expert's rows, in row
// order); an expert with no rows gets zeros.
void orc_expert_ffn_vjp_vjp_weight_grad(const float* xd, const float* gd, const float* vd,
                                        const int32_t* offsets, int32_t n_experts, int32_t d, int32_t h,
                                        const float* w1, const float* w2, float* dw1, float* dw2) {
  for (int e = 0; e < n_experts; ++e) {
    const float* W1 = w1 + (int64_t)e * d * h;
    const float* W2 = w2 + (int64_t)e * h * d;
    const int64_t p0 = offsets[e], n = offsets[e + 1] - offsets[e];
    std::vector<double> u((size_t)n * h), t1((size_t)n * h), t2((size_t)n * h);
#pragma omp parallel
    {
      RowTerms t(h);
#pragma omp for schedule(dynamic, 1)
      for (int64_t r = 0; r < n; ++r) {
        const int64_t p = p0 + r;
        t.compute(xd + p * d, gd + p * d, vd + p * d, W1, W2, d, h);
        for (int j = 0; j < h; ++j) {
          u[(size_t)r * h + j] = t.u[j];
          t1[(size_t)r * h + j] = t.t1[j];
          t2[(size_t)r * h + j] = t.t2[j];
        }
      }
    }
#pragma omp parallel for schedule(dynamic, 4)
    for (int k = 0; k < d; ++k) {
      std::vector<double> acc(h, 0.0);
      for (int64_t r = 0; r < n; ++r) {
        const double vk = vd[(p0 + r) * d + k], xk = xd[(p0 + r) * d + k];
        for (int j = 0; j < h; ++j) acc[j] += vk * u[(size_t)r * h + j] + xk * t2[(size_t)r * h + j];
      }
      for (int j = 0; j < h; ++j) dw1[(int64_t)e * d * h + (int64_t)k * h + j] = (float)acc[j];
    }
#pragma omp parallel for schedule(dynamic, 4)
    for (int j = 0; j < h; ++j) {
      std::vector<double> acc(d, 0.0);
      for (int64_t r = 0; r < n; ++r) {
        const double tj = t1[(size_t)r * h + j];
        for (int c = 0; c < d; ++c) acc[c] += tj * (double)gd[(p0 + r) * d + c];
      }
      for (int c = 0; c < d; ++c) dw2[(int64_t)e * h * d + (int64_t)j * d + c] = (float)acc[c];
    }
  }
}

// ---------------------------------------------------------------------------
// Expert-parallel exchange layout.  [Review] section 3.4 (FSEP: experts are
// sharded over ranks) and section 3.5 (the dispatch all-to-all of the packed
// rows).  P ranks; rank o owns experts [o*E/P, (o+1)*E/P) (E divisible by P).
// counts_all[s][e] = rows rank s routed to expert e.  Definitions:
//   src_off[s][e]  = sum_{e' < e} counts_all[s][e']        (sender's local dispatch
//                    order is expert-major; src_off[s][E] = its row count)
//   recv_off[o][j] = sum_{local experts j' < j of o} sum_s counts_all[s][o*E/P + j']
//                    (the owner groups received rows by local expert, then sender)
//   dst_off[s][e]  = recv_off[owner(e)][e - owner(e)*E/P] + sum_{s' < s} counts_all[s'][e]
// Row i of (s, e) travels from sender row src_off[s][e] + i to owner row
// dst_off[s][e] + i.  Returns 0, or -1 if E is not a multiple of P.
// ---------------------------------------------------------------------------
int orc_ep_layout(const int32_t* counts_all, int32_t P, int32_t E, int32_t* src_off, int32_t* dst_off,
                  int32_t* recv_off) {
  if (P < 1 || E < P || E % P != 0) return -1;
  const int El = E / P;
  for (int s = 0; s < P; ++s) {
    int64_t acc = 0;
    for (int e = 0; e < E; ++e) {
      src_off[s * (E + 1) + e] = (int32_t)acc;
      acc += counts_all[s * E + e];
    }
    src_off[s * (E + 1) + E] = (int32_t)acc;
  }
  for (int o = 0; o < P; ++o) {
    int64_t acc = 0;
    for (int j = 0; j < El; ++j) {
      recv_off[o * (El + 1) + j] = (int32_t)acc;
      for (int s = 0; s < P; ++s) acc += counts_all[s * E + o * El + j];
    }
    recv_off[o * (El + 1) + El] = (int32_t)acc;
  }
  for (int e = 0; e < E; ++e) {
    const int o = e / El, j = e - o * El;
    int64_t acc = recv_off[o * (El + 1) + j];
    for (int s = 0; s < P; ++s) {
      dst_off[s * E + e] = (int32_t)acc;
      acc += counts_all[s * E + e];
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Combine.  [Blueprint] §3.2: the activated experts' outputs are summed with
// the gate weights.  Gather form: Y[i,:] = sum_{k ascending} w[i,k] *
// Yd[slot_of[i*K+k],:]; topk_weight == NULL means weight 1 (the VJP combine).
// ---------------------------------------------------------------------------
void orc_combine(const float* yd, const int32_t* slot_of, const float* topk_weight,
                 int64_t n_atoms, int32_t top_k, int32_t d, float* y) {
  std::vector<double> acc(d);
  for (int64_t i = 0; i < n_atoms; ++i) {
    std::fill(acc.begin(), acc.end(), 0.0);
    for (int k = 0; k < top_k; ++k) {
      const int64_t s = i * top_k + k;
      const int64_t p = slot_of[s];
      const double w = topk_weight ? (double)topk_weight[s] : 1.0;
      for (int j = 0; j < d; ++j) acc[j] += w * (double)yd[p * d + j];
    }
    for (int j = 0; j < d; ++j) y[i * d + j] = (float)acc[j];
  }
}

// ---------------------------------------------------------------------------
// Edge -> atom aggregation.  [Review] §3.5 CNIS high-performance kernels
// (neighbour aggregation, edge aggregation): edge messages are reduced into
// their receiver atoms.  Reading: plain sum over a receiver-sorted CSR,
// X[i,:] = sum_{e in [row_ptr[i], row_ptr[i+1])} msg[e,:]; zero degree -> 0.
// ---------------------------------------------------------------------------
void orc_edge_aggregate(const float* msg, const int64_t* row_ptr, int64_t n_atoms,
                        int32_t d, float* out) {
  std::vector<double> acc(d);
  for (int64_t i = 0; i < n_atoms; ++i) {
    std::fill(acc.begin(), acc.end(), 0.0);
    for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e)
      for (int j = 0; j < d; ++j) acc[j] += (double)msg[e * d + j];
    for (int j = 0; j < d; ++j) out[i * d + j] = (float)acc[j];
  }
}

// ---------------------------------------------------------------------------
// Edge-side neighbour operations ([Review] §3.5, CNIS kernels: neighbour
// aggregation with fused indexing).  Reading: with the receiver-sorted CSR
// (row_ptr, senders),
//   gradient of the edge aggregation:  dmsg[e,:] = dX[i,:] for e in row i;
//   neighbour aggregation by sender:   out[i,:] = sum_{e in row i} x[senders[e],:].
// ---------------------------------------------------------------------------
void orc_edge_broadcast(const float* dx, const int64_t* row_ptr, int64_t n_atoms, int32_t d,
                        float* dmsg) {
  for (int64_t i = 0; i < n_atoms; ++i)
    for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e)
      for (int j = 0; j < d; ++j) dmsg[e * d + j] = dx[i * d + j];
}

int orc_neighbor_aggregate(const float* x, const int64_t* row_ptr, const int32_t* senders,
                           int64_t n_atoms, int32_t d, float* out) {
  std::vector<double> acc(d);
  for (int64_t i = 0; i < n_atoms; ++i) {
    std::fill(acc.begin(), acc.end(), 0.0);
    for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
      const int64_t s = senders[e];
      if (s < 0 || s >= n_atoms) return -1;
      for (int j = 0; j < d; ++j) acc[j] += (double)x[s * d + j];
    }
    for (int j = 0; j < d; ++j) out[i * d + j] = (float)acc[j];
  }
  return 0;
}

}  // extern "C"
