// oracle_core.cpp -- TEST INFRASTRUCTURE ONLY.
//
// The heavy loops of the CPU oracle for the sparse MoE layer, in plain fp64.
// Nothing in the product library calls this file, links it or shares code
// with it; only the test suite, the smoke check and the CPU-baseline leg of
// the benchmark use it (through oracle/__init__.py).
//
// What it computes, from "Inkling, Dissected" (§02 "Anatomy of one MoE layer",
// §02b "Sigmoid, not softmax"):
//   * router logits z[t,i] = x_t . w_i for every expert i (the argument of the
//     sigmoid in the router formula of §02b);
//   * one expert applied to token rows: the pages define an expert as an MLP,
//     "two matrix multiplies with a nonlinearity between them" (§02); the
//     nonlinearity is GELU with the tanh form (Hendrycks & Gimpel, 2016),
//         gelu(u) = u/2 * (1 + tanh(sqrt(2/pi) * (u + 0.044715 u^3))),
//     so y = W2 . gelu(W1 . x) with W1 [d_ff, d] and W2 [d, d_ff];
//   * the gated expert of the released Inkling configuration ("Under the hood",
//     "MoE: the expert configuration": each routed expert is a SwiGLU FFN),
//     SwiGLU as defined by Shazeer (2020, "GLU Variants Improve Transformer"):
//         y = W2 . (silu(Wg . x) * (Wu . x)),  silu(u) = u / (1 + e^-u),
//     with Wg, Wu [d_ff, d] stacked as W1 [2 d_ff, d] (gate rows first).
// Inputs are bf16 bit patterns, widened exactly to double; every sum runs in
// index order in double precision (compiled without FP contraction).
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <thread>
#include <vector>

namespace {

inline double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof(f));
  return (double)f;
}

inline double gelu_tanh(double u) {
  const double c = std::sqrt(2.0 / M_PI);
  return 0.5 * u * (1.0 + std::tanh(c * (u + 0.044715 * u * u * u)));
}

inline double silu(double u) { return u / (1.0 + std::exp(-u)); }

template <class F>
void parallel_rows(int64_t n, int nthreads, F f) {
  if (nthreads <= 0) nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
  if ((int64_t)nthreads > n) nthreads = (int)std::max<int64_t>(1, n);
  if (nthreads == 1) {
    for (int64_t i = 0; i < n; ++i) f(i);
    return;
  }
  std::vector<std::thread> ts;
  for (int t = 0; t < nthreads; ++t)
    ts.emplace_back([=] {
      for (int64_t i = t; i < n; i += nthreads) f(i);
    });
  for (auto& t : ts) t.join();
}

std::vector<double> widen(const uint16_t* p, int64_t n, int nthreads) {
  std::vector<double> out((size_t)n);
  const int64_t chunk = 1 << 16;
  int64_t nchunks = (n + chunk - 1) / chunk;
  parallel_rows(nchunks, nthreads, [&](int64_t c) {
    int64_t b = c * chunk, e = std::min(n, b + chunk);
    for (int64_t i = b; i < e; ++i) out[(size_t)i] = bf16_to_double(p[i]);
  });
  return out;
}

}  // namespace

extern "C" {

// z[t, i] = sum_c x[t, c] * w[i, c]; x [T, d], w [E, d] bf16; z [T, E] fp64.
void or_logits(const uint16_t* x, const uint16_t* w, int64_t T, int64_t d, int64_t E, double* z,
               int nthreads) {
  std::vector<double> wd = widen(w, E * d, nthreads);
  parallel_rows(T, nthreads, [&](int64_t t) {
    std::vector<double> xr((size_t)d);
    for (int64_t c = 0; c < d; ++c) xr[(size_t)c] = bf16_to_double(x[t * d + c]);
    for (int64_t i = 0; i < E; ++i) {
      const double* wi = wd.data() + i * d;
      double acc = 0.0;
      for (int64_t c = 0; c < d; ++c) acc += xr[(size_t)c] * wi[c];
      z[t * E + i] = acc;
    }
  });
}

// Elementwise GELU (tanh form) in fp64, exposed so tests can pin it.
void or_gelu_tanh(const double* u, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = gelu_tanh(u[i]);
}

// One expert on n token rows: y[r] = W2 . gelu(W1 . x[r]).
// xrows [n, d] bf16, w1 [f, d] bf16, w2 [d, f] bf16, y [n, d] fp64.
void or_expert_mlp(const uint16_t* xrows, int64_t n, const uint16_t* w1, const uint16_t* w2, int64_t d,
                   int64_t f, double* y, int nthreads) {
  if (n <= 0) return;
  std::vector<double> w1d = widen(w1, f * d, nthreads);
  std::vector<double> w2d = widen(w2, d * f, nthreads);
  parallel_rows(n, nthreads, [&](int64_t r) {
    std::vector<double> xr((size_t)d), h((size_t)f);
    for (int64_t c = 0; c < d; ++c) xr[(size_t)c] = bf16_to_double(xrows[r * d + c]);
    for (int64_t j = 0; j < f; ++j) {
      const double* wj = w1d.data() + j * d;
      double acc = 0.0;
      for (int64_t c = 0; c < d; ++c) acc += wj[c] * xr[(size_t)c];
      h[(size_t)j] = gelu_tanh(acc);
    }
    for (int64_t i = 0; i < d; ++i) {
      const double* wi = w2d.data() + i * f;
      double acc = 0.0;
      for (int64_t j = 0; j < f; ++j) acc += wi[j] * h[(size_t)j];
      y[r * d + i] = acc;
    }
  });
}

// Elementwise SiLU in fp64, exposed so tests can pin it.
void or_silu(const double* u, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = silu(u[i]);
}

// One gated expert on n token rows: y[r] = W2 . (silu(Wg . x[r]) * (Wu . x[r])).
// xrows [n, d] bf16, w1 [2f, d] bf16 (rows 0..f-1 = Wg, f..2f-1 = Wu), w2 [d, f] bf16, y [n, d] fp64.
void or_expert_swiglu(const uint16_t* xrows, int64_t n, const uint16_t* w1, const uint16_t* w2, int64_t d,
                      int64_t f, double* y, int nthreads) {
  if (n <= 0) return;
  std::vector<double> w1d = widen(w1, 2 * f * d, nthreads);
  std::vector<double> w2d = widen(w2, d * f, nthreads);
  parallel_rows(n, nthreads, [&](int64_t r) {
    std::vector<double> xr((size_t)d), h((size_t)f);
    for (int64_t c = 0; c < d; ++c) xr[(size_t)c] = bf16_to_double(xrows[r * d + c]);
    for (int64_t j = 0; j < f; ++j) {
      const double* wg = w1d.data() + j * d;
      const double* wu = w1d.data() + (f + j) * d;
      double g = 0.0, u = 0.0;
      for (int64_t c = 0; c < d; ++c) {
        g += wg[c] * xr[(size_t)c];
        u += wu[c] * xr[(size_t)c];
      }
      h[(size_t)j] = silu(g) * u;
    }
    for (int64_t i = 0; i < d; ++i) {
      const double* wi = w2d.data() + i * f;
      double acc = 0.0;
      for (int64_t j = 0; j < f; ++j) acc += wi[j] * h[(size_t)j];
      y[r * d + i] = acc;
    }
  });
}

// The gated expert on fp64 rows and weights (for pins with exact inputs).
void or_expert_swiglu_f64(const double* xrows, int64_t n, const double* w1, const double* w2, int64_t d,
                          int64_t f, double* y, int nthreads) {
  parallel_rows(n, nthreads, [&](int64_t r) {
    std::vector<double> h((size_t)f);
    const double* xr = xrows + r * d;
    for (int64_t j = 0; j < f; ++j) {
      double g = 0.0, u = 0.0;
      for (int64_t c = 0; c < d; ++c) {
        g += w1[j * d + c] * xr[c];
        u += w1[(f + j) * d + c] * xr[c];
      }
      h[(size_t)j] = silu(g) * u;
    }
    for (int64_t i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < f; ++j) acc += w2[i * f + j] * h[(size_t)j];
      y[r * d + i] = acc;
    }
  });
}

// The same expert on fp64 rows (used by the pins that feed exact values).
void or_expert_mlp_f64(const double* xrows, int64_t n, const double* w1, const double* w2, int64_t d,
                       int64_t f, double* y, int nthreads) {
  parallel_rows(n, nthreads, [&](int64_t r) {
    std::vector<double> h((size_t)f);
    const double* xr = xrows + r * d;
    for (int64_t j = 0; j < f; ++j) {
      double acc = 0.0;
      for (int64_t c = 0; c < d; ++c) acc += w1[j * d + c] * xr[c];
      h[(size_t)j] = gelu_tanh(acc);
    }
    for (int64_t i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < f; ++j) acc += w2[i * f + j] * h[(size_t)j];
      y[r * d + i] = acc;
    }
  });
}

}  // extern "C"
