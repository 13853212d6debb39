// nc_oracle.cpp -- CPU oracle for the nanochat base-pretraining step.
//
// TEST INFRASTRUCTURE ONLY (see nc_oracle.h): loaded by tests/, by
// __graft_entry__.smoke() and by bench.py's CPU-baseline leg, never by the
// product library.  Every quantity is computed in double precision with
// plain loops in the order the definitions state; rows are spread over
// OpenMP threads, each output element is summed by one thread in index
// order, so results do not depend on the thread count.
//
// Sources followed (dev.to guide "Como treinar seu proprio ChatGPT por 50
// dolares"):
//   section "1. Modelo GPT (nanochat/gpt.py)"         -- the block structure
//   section "2. Otimizador Muon (nanochat/optim.py)"  -- momentum + Newton-Schulz
//   section "Filosofia: Um Unico Seletor ..."         -- --depth sets the shapes
//   table "O Que o nanochat Abrange"                  -- BPE vocabulary 32768

#include "nc_oracle.h"

#include <omp.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

constexpr double kNormEps = 1e-6;    // RMSNorm eps (pages silent; reading: 1e-6)
constexpr double kRopeBase = 10000;  // RoPE base (pages silent; reading: 10000)
constexpr double kNsA = 3.4445, kNsB = -4.7750, kNsC = 2.0315;
constexpr int kNsSteps = 5;
constexpr double kNsEps = 1e-7;      // Frobenius-normalisation eps (reading)

struct Dims {
  int L, d, H, hd, F, V, Hkv;
};

bool make_dims(int depth, int vocab, Dims* s) {
  if (depth < 1 || depth > 64 || vocab < 1) return false;
  s->L = depth;
  s->d = 64 * depth;
  s->hd = s->d < 128 ? s->d : 128;
  if (s->d % s->hd) return false;
  s->H = s->d / s->hd;
  s->F = 4 * s->d;
  s->V = vocab;
  s->Hkv = s->H;
  return true;
}

// Grouped KV heads (guide, section "1. Modelo GPT": "GQA: atencao com menos
// heads KV"): n_kv_head <= 0 keeps one KV head per query head; otherwise it
// must divide n_head.  wk and wv then have n_kv_head * head_dim rows.
bool make_dims_kv(int depth, int vocab, int n_kv_head, Dims* s) {
  if (!make_dims(depth, vocab, s)) return false;
  if (n_kv_head > 0) {
    if (n_kv_head > s->H || s->H % n_kv_head) return false;
    s->Hkv = n_kv_head;
  }
  return true;
}

int64_t numel_of(const Dims& s, int idx) {
  const int n = 6 * s.L + 2;
  if (idx < 0 || idx >= n) return -1;
  if (idx == 0 || idx == n - 1) return (int64_t)s.V * s.d;
  const int j = (idx - 1) % 6;
  if (j == 4 || j == 5) return (int64_t)s.F * s.d;
  if (j == 1 || j == 2) return (int64_t)s.Hkv * s.hd * s.d;
  return (int64_t)s.d * s.d;
}

// fan_in (in-features) of tensor idx; the embedding's one-hot input has fan_in 1.
int64_t fan_in_of(const Dims& s, int idx) {
  const int n = 6 * s.L + 2;
  if (idx == 0) return 1;
  if (idx == n - 1) return s.d;
  return ((idx - 1) % 6 == 5) ? s.F : s.d;
}

uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// ---------------------------------------------------------------- matmuls
// y[r, o] = sum_k x[r, k] * w[o, k]        (y = x W^T)
template <class TW>
void mm_nt(const double* x, const TW* w, int64_t rows, int64_t n, int64_t k, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const double* xr = x + r * k;
    for (int64_t o = 0; o < n; ++o) {
      const TW* wo = w + o * k;
      double acc = 0;
      for (int64_t i = 0; i < k; ++i) acc += xr[i] * (double)wo[i];
      y[r * n + o] = acc;
    }
  }
}

// dx[r, i] (+)= sum_o dy[r, o] * w[o, i]   (dx = dy W)
template <class TW>
void mm_nn_acc(const double* dy, const TW* w, int64_t rows, int64_t n, int64_t k, double* dx,
               bool accumulate) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    double* dxr = dx + r * k;
    if (!accumulate) std::memset(dxr, 0, sizeof(double) * k);
    for (int64_t o = 0; o < n; ++o) {
      const double g = dy[r * n + o];
      const TW* wo = w + o * k;
      for (int64_t i = 0; i < k; ++i) dxr[i] += g * (double)wo[i];
    }
  }
}

// dw[o, i] = sum_r dy[r, o] * x[r, i]      (dW = dy^T x)
void mm_tn(const double* dy, const double* x, int64_t rows, int64_t n, int64_t k, double* dw) {
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < n; ++o) {
    double* dwo = dw + o * k;
    std::memset(dwo, 0, sizeof(double) * k);
    for (int64_t r = 0; r < rows; ++r) {
      const double g = dy[r * n + o];
      const double* xr = x + r * k;
      for (int64_t i = 0; i < k; ++i) dwo[i] += g * xr[i];
    }
  }
}

// ---------------------------------------------------------------- RMSNorm
// y = x * rstd, rstd = 1 / sqrt(mean(x^2) + eps), one row of `cols`.
void rms_row(const double* x, int cols, double* y, double* rstd) {
  double ss = 0;
  for (int i = 0; i < cols; ++i) ss += x[i] * x[i];
  const double r = 1.0 / std::sqrt(ss / cols + kNormEps);
  for (int i = 0; i < cols; ++i) y[i] = x[i] * r;
  if (rstd) *rstd = r;
}

// Reverse of rms_row: with y = x*r, dx = r * (dy - y * mean(dy*y)).  Adds into dx.
void rms_row_bwd_acc(const double* dy, const double* x, double r, int cols, double* dx) {
  double dot = 0;
  for (int i = 0; i < cols; ++i) dot += dy[i] * x[i] * r;
  const double m = dot / cols;
  for (int i = 0; i < cols; ++i) dx[i] += r * (dy[i] - x[i] * r * m);
}

// ---------------------------------------------------------------- RoPE
// Pairs (i, i + hd/2) rotate by theta_i = pos * base^(-2i/hd).
void rope_row(double* v, int hd, int64_t pos, double base, int sign) {
  const int h = hd / 2;
  for (int i = 0; i < h; ++i) {
    const double th = (double)pos * std::pow(base, -2.0 * i / hd);
    const double c = std::cos(th), s = sign * std::sin(th);
    const double a = v[i], b = v[i + h];
    v[i] = a * c - b * s;
    v[i + h] = a * s + b * c;
  }
}

// ---------------------------------------------------------------- attention
// Causal softmax attention per (b, h).  Tensors are [B, T, H, hd].
void attention_fwd(const double* q, const double* k, const double* v, int B, int T, int H, int hd,
                   double* o, double* lse, double* probs) {
  const double scale = 1.0 / std::sqrt((double)hd);
  const int64_t rs = (int64_t)H * hd;  // row stride
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int hh = 0; hh < H; ++hh) {
      std::vector<double> s(T);
      for (int t = 0; t < T; ++t) {
        const double* qt = q + ((int64_t)b * T + t) * rs + (int64_t)hh * hd;
        double m = -INFINITY;
        for (int j = 0; j <= t; ++j) {
          const double* kj = k + ((int64_t)b * T + j) * rs + (int64_t)hh * hd;
          double acc = 0;
          for (int i = 0; i < hd; ++i) acc += qt[i] * kj[i];
          s[j] = acc * scale;
          if (s[j] > m) m = s[j];
        }
        double l = 0;
        for (int j = 0; j <= t; ++j) l += std::exp(s[j] - m);
        const double ls = m + std::log(l);
        lse[((int64_t)b * H + hh) * T + t] = ls;
        double* ot = o + ((int64_t)b * T + t) * rs + (int64_t)hh * hd;
        for (int i = 0; i < hd; ++i) ot[i] = 0;
        for (int j = 0; j <= t; ++j) {
          const double p = std::exp(s[j] - ls);
          const double* vj = v + ((int64_t)b * T + j) * rs + (int64_t)hh * hd;
          for (int i = 0; i < hd; ++i) ot[i] += p * vj[i];
          if (probs) probs[(((int64_t)b * H + hh) * T + t) * T + j] = p;
        }
        if (probs)
          for (int j = t + 1; j < T; ++j) probs[(((int64_t)b * H + hh) * T + t) * T + j] = 0;
      }
    }
}

// Reverse mode of attention_fwd.  P is recomputed from lse.
//   dP_j = dO . v_j;  D = sum_j P_j dP_j;  dS_j = P_j (dP_j - D)
//   dq += scale * sum_j dS_j k_j;  dk_j += scale * dS_j q;  dv_j += P_j dO
void attention_bwd(const double* q, const double* k, const double* v, const double* lse,
                   const double* dout, int B, int T, int H, int hd, double* dq, double* dk,
                   double* dv) {
  const double scale = 1.0 / std::sqrt((double)hd);
  const int64_t rs = (int64_t)H * hd;
  const int64_t n = (int64_t)B * T * rs;
  std::memset(dq, 0, sizeof(double) * n);
  std::memset(dk, 0, sizeof(double) * n);
  std::memset(dv, 0, sizeof(double) * n);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int hh = 0; hh < H; ++hh) {
      std::vector<double> p(T), dp(T);
      for (int t = 0; t < T; ++t) {
        const int64_t rt = ((int64_t)b * T + t) * rs + (int64_t)hh * hd;
        const double ls = lse[((int64_t)b * H + hh) * T + t];
        double D = 0;
        for (int j = 0; j <= t; ++j) {
          const int64_t rj = ((int64_t)b * T + j) * rs + (int64_t)hh * hd;
          double s = 0, g = 0;
          for (int i = 0; i < hd; ++i) {
            s += q[rt + i] * k[rj + i];
            g += dout[rt + i] * v[rj + i];
          }
          p[j] = std::exp(s * scale - ls);
          dp[j] = g;
          D += p[j] * g;
        }
        for (int j = 0; j <= t; ++j) {
          const int64_t rj = ((int64_t)b * T + j) * rs + (int64_t)hh * hd;
          const double ds = p[j] * (dp[j] - D);
          for (int i = 0; i < hd; ++i) {
            dq[rt + i] += scale * ds * k[rj + i];
            dk[rj + i] += scale * ds * q[rt + i];
            dv[rj + i] += p[j] * dout[rt + i];
          }
        }
      }
    }
}

// Causal attention with grouped KV heads and a left window (guide, section
// "1. Modelo GPT": "GQA: atencao com menos heads KV", "atencao de janela ...
// 'SSSL'", and the flash-attention call with causal=True, window_size):
// query head hh reads KV head hh / (H / Hkv); query t sees keys
// j in [t - window, t] (window < 0: no lower bound).  q, o: [B, T, H, hd];
// k, v: [B, T, Hkv, hd]; lse [B, H, T].
void attention_fwd_gw(const double* q, const double* k, const double* v, int B, int T, int H,
                      int Hkv, int hd, int window, double* o, double* lse) {
  const double scale = 1.0 / std::sqrt((double)hd);
  const int64_t rq = (int64_t)H * hd, rk = (int64_t)Hkv * hd;
  const int group = H / Hkv;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int hh = 0; hh < H; ++hh) {
      const int hk = hh / group;
      std::vector<double> s(T);
      for (int t = 0; t < T; ++t) {
        const int j0 = window < 0 ? 0 : std::max(0, t - window);
        const double* qt = q + ((int64_t)b * T + t) * rq + (int64_t)hh * hd;
        double m = -INFINITY;
        for (int j = j0; j <= t; ++j) {
          const double* kj = k + ((int64_t)b * T + j) * rk + (int64_t)hk * hd;
          double acc = 0;
          for (int i = 0; i < hd; ++i) acc += qt[i] * kj[i];
          s[j] = acc * scale;
          if (s[j] > m) m = s[j];
        }
        double l = 0;
        for (int j = j0; j <= t; ++j) l += std::exp(s[j] - m);
        const double ls = m + std::log(l);
        lse[((int64_t)b * H + hh) * T + t] = ls;
        double* ot = o + ((int64_t)b * T + t) * rq + (int64_t)hh * hd;
        for (int i = 0; i < hd; ++i) ot[i] = 0;
        for (int j = j0; j <= t; ++j) {
          const double p = std::exp(s[j] - ls);
          const double* vj = v + ((int64_t)b * T + j) * rk + (int64_t)hk * hd;
          for (int i = 0; i < hd; ++i) ot[i] += p * vj[i];
        }
      }
    }
}

// Reverse mode of attention_fwd_gw (same formulas as attention_bwd).  The
// query heads of one KV head run in one thread, in head order, because they
// all add into that KV head's dk and dv.
void attention_bwd_gw(const double* q, const double* k, const double* v, const double* lse,
                      const double* dout, int B, int T, int H, int Hkv, int hd, int window,
                      double* dq, double* dk, double* dv) {
  const double scale = 1.0 / std::sqrt((double)hd);
  const int64_t rq = (int64_t)H * hd, rk = (int64_t)Hkv * hd;
  const int group = H / Hkv;
  std::memset(dq, 0, sizeof(double) * B * T * rq);
  std::memset(dk, 0, sizeof(double) * B * T * rk);
  std::memset(dv, 0, sizeof(double) * B * T * rk);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int hk = 0; hk < Hkv; ++hk) {
      std::vector<double> p(T), dp(T);
      for (int hh = hk * group; hh < (hk + 1) * group; ++hh)
        for (int t = 0; t < T; ++t) {
          const int j0 = window < 0 ? 0 : std::max(0, t - window);
          const int64_t rt = ((int64_t)b * T + t) * rq + (int64_t)hh * hd;
          const double ls = lse[((int64_t)b * H + hh) * T + t];
          double D = 0;
          for (int j = j0; j <= t; ++j) {
            const int64_t rj = ((int64_t)b * T + j) * rk + (int64_t)hk * hd;
            double sc = 0, g = 0;
            for (int i = 0; i < hd; ++i) {
              sc += q[rt + i] * k[rj + i];
              g += dout[rt + i] * v[rj + i];
            }
            p[j] = std::exp(sc * scale - ls);
            dp[j] = g;
            D += p[j] * g;
          }
          for (int j = j0; j <= t; ++j) {
            const int64_t rj = ((int64_t)b * T + j) * rk + (int64_t)hk * hd;
            const double ds = p[j] * (dp[j] - D);
            for (int i = 0; i < hd; ++i) {
              dq[rt + i] += scale * ds * k[rj + i];
              dk[rj + i] += scale * ds * q[rt + i];
              dv[rj + i] += p[j] * dout[rt + i];
            }
          }
        }
    }
}

// ---------------------------------------------------------------- Newton-Schulz
// Plain product c[m, n] = a[m, k] * b[k, n].
void mm_plain(const double* a, const double* b, int m, int k, int n, double* c) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < m; ++i) {
    double* ci = c + (int64_t)i * n;
    for (int j = 0; j < n; ++j) ci[j] = 0;
    for (int p = 0; p < k; ++p) {
      const double aip = a[(int64_t)i * k + p];
      const double* bp = b + (int64_t)p * n;
      for (int j = 0; j < n; ++j) ci[j] += aip * bp[j];
    }
  }
}

void transpose(const double* x, int rows, int cols, double* y) {
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < cols; ++j) y[(int64_t)j * rows + i] = x[(int64_t)i * cols + j];
}

// The guide's iteration, right-hand form, on a tall X [m, n] (m >= n):
//   A = X^T X;  B = b*A + c*A*A;  X = a*X + X*B.
void ns_tall(double* X, int m, int n, int steps, double a, double b, double c) {
  std::vector<double> Xt((int64_t)n * m), A((int64_t)n * n), AA((int64_t)n * n),
      Bm((int64_t)n * n), XB((int64_t)m * n);
  for (int it = 0; it < steps; ++it) {
    transpose(X, m, n, Xt.data());
    mm_plain(Xt.data(), X, n, m, n, A.data());
    mm_plain(A.data(), A.data(), n, n, n, AA.data());
    for (int64_t i = 0; i < (int64_t)n * n; ++i) Bm[i] = b * A[i] + c * AA[i];
    mm_plain(X, Bm.data(), m, n, n, XB.data());
    for (int64_t i = 0; i < (int64_t)m * n; ++i) X[i] = a * X[i] + XB[i];
  }
}

void newton_schulz(const double* G, int rows, int cols, int steps, double a, double b, double c,
                   double eps, double* out) {
  const int64_t n = (int64_t)rows * cols;
  double ss = 0;
  for (int64_t i = 0; i < n; ++i) ss += G[i] * G[i];
  const double inv = 1.0 / (std::sqrt(ss) + eps);
  if (rows >= cols) {
    for (int64_t i = 0; i < n; ++i) out[i] = G[i] * inv;
    ns_tall(out, rows, cols, steps, a, b, c);
  } else {
    std::vector<double> Xt(n);
    transpose(G, rows, cols, Xt.data());  // [cols, rows], tall
    for (int64_t i = 0; i < n; ++i) Xt[i] *= inv;
    ns_tall(Xt.data(), cols, rows, steps, a, b, c);
    transpose(Xt.data(), cols, rows, out);
  }
}

// ---------------------------------------------------------------- FP8
// "Treinamento FP8 disponivel via --fp8" (guide, section "1. Modelo GPT",
// and the d26 run of its results table) with no recipe given.  Reading: the
// GEMMs of the block projections take operands in the OCP 8-bit format
// E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
// infinities, largest finite 448 = 1.75 * 2^8, smallest normal 2^-6,
// subnormals k * 2^-9), each operand tensor with one dynamic scale.

// Nearest E4M3 value of a (ties to the even mantissa), saturating to +-448
// ("satfinite": magnitudes above 448, infinities included, become 448).
double e4m3_round(double a) {
  if (std::isnan(a)) return a;
  const double mag = std::fabs(a);
  double q;
  if (mag >= 448.0) {
    q = 448.0;
  } else {
    int e2;
    std::frexp(mag, &e2);  // mag = f * 2^e2, f in [0.5, 1): leading bit 2^(e2 - 1)
    // Spacing of the grid around mag: 2^(e - 3) in the binade [2^e, 2^(e+1)),
    // and the subnormal spacing 2^-9 below 2^-6.
    const int e = mag < 0x1.0p-6 ? -6 : e2 - 1;
    const double step = std::ldexp(1.0, e - 3);
    q = std::nearbyint(mag / step) * step;  // default rounding: to nearest, ties to even
  }
  return std::signbit(a) ? -q : q;
}

// Nearest bfloat16 value of the fp32 value v, ties to even: the storage
// format of activations and their gradients, from which a kernel quantises.
float bf16_round(float v) {
  if (std::isnan(v)) return v;
  uint32_t u;
  std::memcpy(&u, &v, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  float r;
  std::memcpy(&r, &u, 4);
  return r;
}

// The value a tensor is quantised from: fp32(x), rounded on to bf16 for an
// activation or gradient (bf16 in memory) in E4M3 mode; weights quantise
// from their fp32 masters.  Scaling alone (fmt 0) keeps fp32 everywhere.
inline float fp8_source(double x, int fmt, bool act) {
  return (fmt && act) ? bf16_round((float)x) : (float)x;
}

// Scale of one operand tensor: s = 448 / amax, in fp32 arithmetic as a
// kernel computes it (amax over the source values; 1 when all are zero).
float fp8_scale(const double* x, int64_t n, int fmt = 1, bool act = false) {
  float amax = 0.f;
  for (int64_t i = 0; i < n; ++i) amax = std::max(amax, std::fabs(fp8_source(x[i], fmt, act)));
  return amax > 0.f ? 448.0f / amax : 1.0f;
}

// q_i = e4m3(v_i * s) with the fp32 product of the source value v_i; fmt 0
// keeps the scaled fp32 value (scaling without rounding, a check of the
// surrounding steps).
float fp8_quantize(const double* x, int64_t n, int fmt, bool act, double* q) {
  const float sc = fp8_scale(x, n, fmt, act);
  for (int64_t i = 0; i < n; ++i) {
    const float y = fp8_source(x[i], fmt, act) * sc;
    q[i] = fmt ? e4m3_round((double)y) : (double)y;
  }
  return sc;
}

template <class TW>
std::vector<double> as_f64(const TW* w, int64_t n) {
  return std::vector<double>(w, w + n);
}

// y = x W^T on quantised operands: (Q(x) Q(W)^T) / (s_x s_W); x is an
// activation, W a weight.
void fp8_mm_nt(const double* x, const double* w, int64_t rows, int64_t n, int64_t k, int fmt,
               double* y) {
  std::vector<double> qx(rows * k), qw(n * k);
  const double sx = fp8_quantize(x, rows * k, fmt, true, qx.data());
  const double sw = fp8_quantize(w, n * k, fmt, false, qw.data());
  mm_nt(qx.data(), qw.data(), rows, n, k, y);
  const double inv = 1.0 / (sx * sw);
  for (int64_t i = 0; i < rows * n; ++i) y[i] *= inv;
}

// dx (+)= dy W on quantised operands (dy a gradient, W a weight).
void fp8_mm_nn(const double* dy, const double* w, int64_t rows, int64_t n, int64_t k, int fmt,
               double* dx, bool accumulate) {
  std::vector<double> qd(rows * n), qw(n * k), t(rows * k);
  const double sd = fp8_quantize(dy, rows * n, fmt, true, qd.data());
  const double sw = fp8_quantize(w, n * k, fmt, false, qw.data());
  mm_nn_acc(qd.data(), qw.data(), rows, n, k, t.data(), false);
  const double inv = 1.0 / (sd * sw);
  for (int64_t i = 0; i < rows * k; ++i) dx[i] = (accumulate ? dx[i] : 0.0) + t[i] * inv;
}

// dW = dy^T x on quantised operands (both activations or gradients).
void fp8_mm_tn(const double* dy, const double* x, int64_t rows, int64_t n, int64_t k, int fmt,
               double* dw) {
  std::vector<double> qd(rows * n), qx(rows * k);
  const double sd = fp8_quantize(dy, rows * n, fmt, true, qd.data());
  const double sx = fp8_quantize(x, rows * k, fmt, true, qx.data());
  mm_tn(qd.data(), qx.data(), rows, n, k, dw);
  const double inv = 1.0 / (sd * sx);
  for (int64_t i = 0; i < n * k; ++i) dw[i] *= inv;
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

int oc_dims(int depth, int vocab, int64_t* out) {
  Dims s;
  if (!out || !make_dims(depth, vocab, &s)) return -1;
  out[0] = s.d;
  out[1] = s.H;
  out[2] = s.hd;
  out[3] = s.F;
  out[4] = 6 * s.L + 2;
  out[5] = 6 * s.L;
  return 0;
}

int oc_dims_ex(int depth, int vocab, int n_kv_head, int64_t* out) {
  Dims s;
  if (!out || !make_dims_kv(depth, vocab, n_kv_head, &s)) return -1;
  oc_dims(depth, vocab, out);
  out[6] = s.Hkv;
  return 0;
}

int64_t oc_param_numel(int depth, int vocab, int idx) {
  return oc_param_numel_ex(depth, vocab, 0, idx);
}

int64_t oc_param_numel_ex(int depth, int vocab, int n_kv_head, int idx) {
  Dims s;
  if (!make_dims_kv(depth, vocab, n_kv_head, &s)) return -1;
  return numel_of(s, idx);
}

uint64_t oc_splitmix64(uint64_t x) { return splitmix64(x); }

int oc_init_params(int depth, int vocab, uint64_t seed, int spec_zero, float* const* params) {
  return oc_init_params_ex(depth, vocab, 0, seed, spec_zero, params);
}

int oc_init_params_ex(int depth, int vocab, int n_kv_head, uint64_t seed, int spec_zero,
                      float* const* params) {
  Dims s;
  if (!params || !make_dims_kv(depth, vocab, n_kv_head, &s)) return -1;
  const int n_t = 6 * s.L + 2;
  const double two_pi = 6.283185307179586476925286766559;
  for (int t = 0; t < n_t; ++t) {
    float* p = params[t];
    if (!p) return -1;
    const int64_t n = numel_of(s, t);
    const bool is_out_proj = (t > 0 && t < n_t - 1) && ((t - 1) % 6 == 3 || (t - 1) % 6 == 5);
    const bool is_head = (t == n_t - 1);
    if (spec_zero && (is_out_proj || is_head)) {
      for (int64_t i = 0; i < n; ++i) p[i] = 0.0f;
      continue;
    }
    const double stdv = 1.0 / std::sqrt((double)fan_in_of(s, t));
    const uint64_t key = splitmix64(seed ^ splitmix64((uint64_t)t + 1));
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
      const uint64_t w1 = splitmix64(key + 2 * (uint64_t)i);
      const uint64_t w2 = splitmix64(key + 2 * (uint64_t)i + 1);
      const double u1 = (double)(w1 >> 11) * 0x1.0p-53;
      const double u2 = (double)(w2 >> 11) * 0x1.0p-53;
      const double z = std::sqrt(-2.0 * std::log(1.0 - u1)) * std::cos(two_pi * u2);
      p[i] = (float)(z * stdv);
    }
  }
  return 0;
}

int oc_rmsnorm(const double* x, int64_t rows, int cols, double eps, double* y, double* rstd) {
  if (!x || !y || rows < 0 || cols < 1) return -1;
  for (int64_t r = 0; r < rows; ++r) {
    double ss = 0;
    for (int i = 0; i < cols; ++i) ss += x[r * cols + i] * x[r * cols + i];
    const double rs = 1.0 / std::sqrt(ss / cols + eps);
    for (int i = 0; i < cols; ++i) y[r * cols + i] = x[r * cols + i] * rs;
    if (rstd) rstd[r] = rs;
  }
  return 0;
}

int oc_rope_row(double* v, int hd, int64_t pos, double base) {
  if (!v || hd < 2 || (hd & 1)) return -1;
  rope_row(v, hd, pos, base, +1);
  return 0;
}

int oc_attention(const double* q, const double* k, const double* v, int B, int T, int H, int hd,
                 double* o, double* lse, double* probs) {
  if (!q || !k || !v || !o || !lse || B < 0 || T < 0 || H < 1 || hd < 1) return -1;
  attention_fwd(q, k, v, B, T, H, hd, o, lse, probs);
  return 0;
}

int oc_attention_bwd(const double* q, const double* k, const double* v, const double* lse,
                     const double* dout, int B, int T, int H, int hd, double* dq, double* dk,
                     double* dv) {
  if (!q || !k || !v || !lse || !dout || !dq || !dk || !dv || B < 0 || T < 0 || H < 1 || hd < 1)
    return -1;
  attention_bwd(q, k, v, lse, dout, B, T, H, hd, dq, dk, dv);
  return 0;
}

int oc_attention_ex(const double* q, const double* k, const double* v, int B, int T, int H, int Hkv,
                    int hd, int window, double* o, double* lse) {
  if (!q || !k || !v || !o || !lse || B < 0 || T < 0 || H < 1 || hd < 1 || Hkv < 1 || H % Hkv)
    return -1;
  attention_fwd_gw(q, k, v, B, T, H, Hkv, hd, window, o, lse);
  return 0;
}

int oc_attention_bwd_ex(const double* q, const double* k, const double* v, const double* lse,
                        const double* dout, int B, int T, int H, int Hkv, int hd, int window,
                        double* dq, double* dk, double* dv) {
  if (!q || !k || !v || !lse || !dout || !dq || !dk || !dv || B < 0 || T < 0 || H < 1 || hd < 1 ||
      Hkv < 1 || H % Hkv)
    return -1;
  attention_bwd_gw(q, k, v, lse, dout, B, T, H, Hkv, hd, window, dq, dk, dv);
  return 0;
}

int oc_matmul_nt(const double* x, const double* w, int64_t rows, int64_t n, int64_t k, double* y) {
  if (!x || !w || !y || rows < 0 || n < 0 || k < 0) return -1;
  mm_nt(x, w, rows, n, k, y);
  return 0;
}

static int gpt_impl(int depth, int vocab, int n_kv_head, const int32_t* window, int fp8,
                    const float* const* params, const int32_t* tokens, const int32_t* targets,
                    int B, int T, double* loss, double* const* grads, double* logits);

int oc_gpt_fwd_bwd(int depth, int vocab, const float* const* params, const int32_t* tokens,
                   const int32_t* targets, int B, int T, double* loss, double* const* grads,
                   double* logits) {
  return oc_gpt_fwd_bwd_ex(depth, vocab, 0, nullptr, params, tokens, targets, B, T, loss, grads,
                           logits);
}

int oc_gpt_fwd_bwd_ex(int depth, int vocab, int n_kv_head, const int32_t* window,
                      const float* const* params, const int32_t* tokens, const int32_t* targets,
                      int B, int T, double* loss, double* const* grads, double* logits) {
  return gpt_impl(depth, vocab, n_kv_head, window, -1, params, tokens, targets, B, T, loss, grads,
                  logits);
}

int oc_gpt_fwd_bwd_fp8(int depth, int vocab, int n_kv_head, const int32_t* window, int fmt,
                       const float* const* params, const int32_t* tokens, const int32_t* targets,
                       int B, int T, double* loss, double* const* grads, double* logits) {
  if (fmt != 0 && fmt != 1) return -1;
  return gpt_impl(depth, vocab, n_kv_head, window, fmt, params, tokens, targets, B, T, loss, grads,
                  logits);
}

double oc_e4m3_round(double x) { return e4m3_round(x); }

int oc_threads(int n) {
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
}

float oc_fp8_scale(const double* x, int64_t n, int act) {
  return (x && n > 0) ? fp8_scale(x, n, 1, act != 0) : -1.0f;
}

int oc_fp8_matmul_nt(const double* x, const double* w, int64_t rows, int64_t n, int64_t k,
                     int fmt, double* y) {
  if (!x || !w || !y || rows < 1 || n < 1 || k < 1 || (fmt != 0 && fmt != 1)) return -1;
  fp8_mm_nt(x, w, rows, n, k, fmt, y);
  return 0;
}

// The model of oc_gpt_fwd_bwd_ex; fp8 < 0: exact GEMMs, fp8 >= 0: the block
// projections' GEMMs on quantised operands (fp8_mm_*, format fp8), the q|k|v
// projection as one [d + 2 dkv, d] tensor with one scale (its weights and its
// output gradient each quantised as a whole).
static int gpt_impl(int depth, int vocab, int n_kv_head, const int32_t* window, int fp8,
                    const float* const* params, const int32_t* tokens, const int32_t* targets,
                    int B, int T, double* loss, double* const* grads, double* logits) {
  Dims s;
  if (!params || !tokens || !targets || !loss || B < 1 || T < 1 ||
      !make_dims_kv(depth, vocab, n_kv_head, &s))
    return -1;
  const int L = s.L, d = s.d, H = s.H, hd = s.hd, F = s.F, V = s.V, Hkv = s.Hkv;
  const int dkv = Hkv * hd;  // width of k and v
  const int64_t N = (int64_t)B * T;
  // Window of layer l: keys t - win(l) .. t (negative: every key up to t).
  auto win = [&](int l) { return window ? window[l] : -1; };
  for (int64_t n = 0; n < N; ++n)
    if (tokens[n] < 0 || tokens[n] >= V || targets[n] < 0 || targets[n] >= V) return -2;
  const float* wte = params[0];
  const float* wlm = params[6 * L + 1];
  auto W = [&](int l, int j) { return params[1 + 6 * l + j]; };

  typedef std::vector<double> vec;
  // Projections y = x W^T, dx (+)= dy W, dW = dy^T x: exact, or on fp8 operands.
  auto lin_nt = [&](const double* xx, const float* w, int64_t rows, int64_t n, int64_t k,
                    double* y) {
    if (fp8 < 0) mm_nt(xx, w, rows, n, k, y);
    else fp8_mm_nt(xx, as_f64(w, n * k).data(), rows, n, k, fp8, y);
  };
  auto lin_nn = [&](const double* dy, const float* w, int64_t rows, int64_t n, int64_t k,
                    double* dx, bool accumulate) {
    if (fp8 < 0) mm_nn_acc(dy, w, rows, n, k, dx, accumulate);
    else fp8_mm_nn(dy, as_f64(w, n * k).data(), rows, n, k, fp8, dx, accumulate);
  };
  auto lin_tn = [&](const double* dy, const double* xx, int64_t rows, int64_t n, int64_t k,
                    double* dw) {
    if (fp8 < 0) mm_tn(dy, xx, rows, n, k, dw);
    else fp8_mm_tn(dy, xx, rows, n, k, fp8, dw);
  };
  const int Qw = d + 2 * dkv;  // width of the fused q|k|v projection
  // [wq; wk; wv] of layer l as one row-major [Qw, d] matrix (fp8 only).
  auto wqkv = [&](int l) {
    vec w((int64_t)Qw * d);
    std::copy(W(l, 0), W(l, 0) + (int64_t)d * d, w.begin());
    std::copy(W(l, 1), W(l, 1) + (int64_t)dkv * d, w.begin() + (int64_t)d * d);
    std::copy(W(l, 2), W(l, 2) + (int64_t)dkv * d, w.begin() + (int64_t)(d + dkv) * d);
    return w;
  };
  const int64_t Nd = N * d, NF = N * F, NH = N * H, Nkv = N * dkv, NHkv = N * Hkv;
  // Saved forward state per layer.
  std::vector<vec> xin(L, vec(Nd)), h1(L, vec(Nd)), r1(L, vec(N)), qr(L, vec(Nd)),
      kr(L, vec(Nkv)), rq(L, vec(NH)), rk(L, vec(NHkv)), qn(L, vec(Nd)), kn(L, vec(Nkv)),
      vv(L, vec(Nkv)), ao(L, vec(Nd)), lse(L, vec(NH)), xmid(L, vec(Nd)), h2(L, vec(Nd)),
      r2(L, vec(N)), uu(L, vec(NF)), aa(L, vec(NF));
  vec x(Nd), tmp(Nd);

  // x0 = wte[token]
  for (int64_t n = 0; n < N; ++n)
    for (int i = 0; i < d; ++i) x[n * d + i] = wte[(int64_t)tokens[n] * d + i];

  for (int l = 0; l < L; ++l) {
    xin[l] = x;
    for (int64_t n = 0; n < N; ++n) rms_row(&x[n * d], d, &h1[l][n * d], &r1[l][n]);
    if (fp8 < 0) {
      mm_nt(h1[l].data(), W(l, 0), N, d, d, qr[l].data());
      mm_nt(h1[l].data(), W(l, 1), N, dkv, d, kr[l].data());
      mm_nt(h1[l].data(), W(l, 2), N, dkv, d, vv[l].data());
    } else {
      vec y(N * Qw);
      fp8_mm_nt(h1[l].data(), wqkv(l).data(), N, Qw, d, fp8, y.data());
      for (int64_t n = 0; n < N; ++n) {
        std::copy(&y[n * Qw], &y[n * Qw] + d, &qr[l][n * d]);
        std::copy(&y[n * Qw] + d, &y[n * Qw] + d + dkv, &kr[l][n * dkv]);
        std::copy(&y[n * Qw] + d + dkv, &y[n * Qw] + Qw, &vv[l][n * dkv]);
      }
    }
    // RoPE, then RMSNorm over each head (QK normalisation).
    for (int64_t n = 0; n < N; ++n) {
      const int64_t pos = n % T;
      for (int hh = 0; hh < H; ++hh) {
        const int64_t off = n * d + (int64_t)hh * hd;
        rope_row(&qr[l][off], hd, pos, kRopeBase, +1);
        rms_row(&qr[l][off], hd, &qn[l][off], &rq[l][n * H + hh]);
      }
      for (int hh = 0; hh < Hkv; ++hh) {
        const int64_t off = n * dkv + (int64_t)hh * hd;
        rope_row(&kr[l][off], hd, pos, kRopeBase, +1);
        rms_row(&kr[l][off], hd, &kn[l][off], &rk[l][n * Hkv + hh]);
      }
    }
    attention_fwd_gw(qn[l].data(), kn[l].data(), vv[l].data(), B, T, H, Hkv, hd, win(l),
                     ao[l].data(), lse[l].data());
    lin_nt(ao[l].data(), W(l, 3), N, d, d, tmp.data());
    for (int64_t i = 0; i < Nd; ++i) x[i] += tmp[i];
    xmid[l] = x;
    for (int64_t n = 0; n < N; ++n) rms_row(&x[n * d], d, &h2[l][n * d], &r2[l][n]);
    lin_nt(h2[l].data(), W(l, 4), N, F, d, uu[l].data());
    for (int64_t i = 0; i < NF; ++i) {
      const double r = uu[l][i] > 0 ? uu[l][i] : 0.0;
      aa[l][i] = r * r;
    }
    lin_nt(aa[l].data(), W(l, 5), N, d, F, tmp.data());
    for (int64_t i = 0; i < Nd; ++i) x[i] += tmp[i];
  }

  vec hf(Nd), rf(N);
  for (int64_t n = 0; n < N; ++n) rms_row(&x[n * d], d, &hf[n * d], &rf[n]);
  vec z(N * (int64_t)V);
  mm_nt(hf.data(), wlm, N, V, d, z.data());

  // loss = mean_n [ logsumexp(z_n) - z_n[target_n] ];  dz = (softmax(z) - onehot) / N
  double total = 0;
  vec dz(grads ? N * (int64_t)V : 0);
#pragma omp parallel for reduction(+ : total) schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const double* zn = &z[n * V];
    double m = -INFINITY;
    for (int j = 0; j < V; ++j) m = zn[j] > m ? zn[j] : m;
    double se = 0;
    for (int j = 0; j < V; ++j) se += std::exp(zn[j] - m);
    const double ls = m + std::log(se);
    total += ls - zn[targets[n]];
    if (grads) {
      for (int j = 0; j < V; ++j) dz[n * V + j] = std::exp(zn[j] - ls) / (double)N;
      dz[n * V + targets[n]] -= 1.0 / (double)N;
    }
  }
  *loss = total / (double)N;
  if (logits) std::memcpy(logits, z.data(), sizeof(double) * N * V);
  if (!grads) return 0;

  // ---------------- backward
  mm_tn(dz.data(), hf.data(), N, V, d, grads[6 * L + 1]);
  vec dhf(Nd), dx(Nd, 0.0);
  mm_nn_acc(dz.data(), wlm, N, V, d, dhf.data(), false);
  for (int64_t n = 0; n < N; ++n) rms_row_bwd_acc(&dhf[n * d], &x[n * d], rf[n], d, &dx[n * d]);

  vec da(NF), du(NF), dh(Nd), dxm(Nd), dao(Nd), dqn(Nd), dkn(Nkv), dvv(Nkv), dq(Nd), dk(Nkv);
  for (int l = L - 1; l >= 0; --l) {
    // x_out = xmid + a W_down^T
    lin_tn(dx.data(), aa[l].data(), N, d, F, grads[1 + 6 * l + 5]);
    lin_nn(dx.data(), W(l, 5), N, d, F, da.data(), false);
    for (int64_t i = 0; i < NF; ++i) du[i] = uu[l][i] > 0 ? 2.0 * uu[l][i] * da[i] : 0.0;
    lin_tn(du.data(), h2[l].data(), N, F, d, grads[1 + 6 * l + 4]);
    lin_nn(du.data(), W(l, 4), N, F, d, dh.data(), false);
    dxm = dx;
    for (int64_t n = 0; n < N; ++n)
      rms_row_bwd_acc(&dh[n * d], &xmid[l][n * d], r2[l][n], d, &dxm[n * d]);
    // xmid = xin + o W_o^T
    lin_tn(dxm.data(), ao[l].data(), N, d, d, grads[1 + 6 * l + 3]);
    lin_nn(dxm.data(), W(l, 3), N, d, d, dao.data(), false);
    attention_bwd_gw(qn[l].data(), kn[l].data(), vv[l].data(), lse[l].data(), dao.data(), B, T,
                     H, Hkv, hd, win(l), dqn.data(), dkn.data(), dvv.data());
    // Through QK-norm, then RoPE (its transpose is the rotation by -theta).
    std::fill(dq.begin(), dq.end(), 0.0);
    std::fill(dk.begin(), dk.end(), 0.0);
    for (int64_t n = 0; n < N; ++n) {
      const int64_t pos = n % T;
      for (int hh = 0; hh < H; ++hh) {
        const int64_t off = n * d + (int64_t)hh * hd;
        rms_row_bwd_acc(&dqn[off], &qr[l][off], rq[l][n * H + hh], hd, &dq[off]);
        rope_row(&dq[off], hd, pos, kRopeBase, -1);
      }
      for (int hh = 0; hh < Hkv; ++hh) {
        const int64_t off = n * dkv + (int64_t)hh * hd;
        rms_row_bwd_acc(&dkn[off], &kr[l][off], rk[l][n * Hkv + hh], hd, &dk[off]);
        rope_row(&dk[off], hd, pos, kRopeBase, -1);
      }
    }
    if (fp8 < 0) {
      mm_tn(dq.data(), h1[l].data(), N, d, d, grads[1 + 6 * l + 0]);
      mm_tn(dk.data(), h1[l].data(), N, dkv, d, grads[1 + 6 * l + 1]);
      mm_tn(dvv.data(), h1[l].data(), N, dkv, d, grads[1 + 6 * l + 2]);
      mm_nn_acc(dq.data(), W(l, 0), N, d, d, dh.data(), false);
      mm_nn_acc(dk.data(), W(l, 1), N, dkv, d, dh.data(), true);
      mm_nn_acc(dvv.data(), W(l, 2), N, dkv, d, dh.data(), true);
    } else {
      vec g(N * Qw), gw((int64_t)Qw * d);
      for (int64_t n = 0; n < N; ++n) {
        std::copy(&dq[n * d], &dq[n * d] + d, &g[n * Qw]);
        std::copy(&dk[n * dkv], &dk[n * dkv] + dkv, &g[n * Qw] + d);
        std::copy(&dvv[n * dkv], &dvv[n * dkv] + dkv, &g[n * Qw] + d + dkv);
      }
      fp8_mm_tn(g.data(), h1[l].data(), N, Qw, d, fp8, gw.data());
      std::copy(gw.begin(), gw.begin() + (int64_t)d * d, grads[1 + 6 * l + 0]);
      std::copy(gw.begin() + (int64_t)d * d, gw.begin() + (int64_t)(d + dkv) * d,
                grads[1 + 6 * l + 1]);
      std::copy(gw.begin() + (int64_t)(d + dkv) * d, gw.end(), grads[1 + 6 * l + 2]);
      fp8_mm_nn(g.data(), wqkv(l).data(), N, Qw, d, fp8, dh.data(), false);
    }
    dx = dxm;
    for (int64_t n = 0; n < N; ++n)
      rms_row_bwd_acc(&dh[n * d], &xin[l][n * d], r1[l][n], d, &dx[n * d]);
  }
  // Embedding: scatter-add of dx0 into the rows the tokens selected.
  double* gE = grads[0];
  std::memset(gE, 0, sizeof(double) * (int64_t)V * d);
  for (int64_t n = 0; n < N; ++n)
    for (int i = 0; i < d; ++i) gE[(int64_t)tokens[n] * d + i] += dx[n * d + i];
  return 0;
}

int oc_newton_schulz(const double* G, int rows, int cols, int steps, double a, double b, double c,
                     double eps_norm, double* out) {
  if (!G || !out || rows < 1 || cols < 1 || steps < 0) return -1;
  newton_schulz(G, rows, cols, steps, a, b, c, eps_norm, out);
  return 0;
}

int oc_muon_update(double* W, double* M, const double* G, int rows, int cols, double lr,
                   double mu) {
  if (!W || !M || !G || rows < 1 || cols < 1) return -1;
  const int64_t n = (int64_t)rows * cols;
  for (int64_t i = 0; i < n; ++i) M[i] = mu * M[i] + G[i];
  std::vector<double> O(n);
  newton_schulz(M, rows, cols, kNsSteps, kNsA, kNsB, kNsC, kNsEps, O.data());
  for (int64_t i = 0; i < n; ++i) W[i] -= lr * O[i];
  return 0;
}

int oc_adamw_update(double* W, double* m, double* v, const double* g, int64_t n, double lr,
                    double b1, double b2, double eps, double wd, int t) {
  if (!W || !m || !v || !g || n < 1 || t < 1) return -1;
  const double c1 = 1.0 - std::pow(b1, t), c2 = 1.0 - std::pow(b2, t);
  for (int64_t i = 0; i < n; ++i) {
    m[i] = b1 * m[i] + (1.0 - b1) * g[i];
    v[i] = b2 * v[i] + (1.0 - b2) * g[i] * g[i];
    const double mhat = m[i] / c1, vhat = v[i] / c2;
    W[i] -= lr * (mhat / (std::sqrt(vhat) + eps) + wd * W[i]);
  }
  return 0;
}

}  // extern "C"
