// Oracle for the looped weight-shared decoder: TEST INFRASTRUCTURE ONLY.
//
// A plain CPU forward pass written from the method's description (see
// oracle.h for the pages it follows).  Every dot product, norm, softmax and
// Sinkhorn step is computed in fp64; weights are stored as fp32 values (already
// rounded to bf16 in the bf16 configuration).  In the bf16 configuration the
// activations that enter a matrix product (the normalised layer input x-hat,
// q/k/v, the attention or linear-attention output, and the SwiGLU product) are
// rounded to bf16, because that is the precision in which a bf16 model feeds
// its matrix products; nothing else is rounded.
//
// No blocking, fusion or reordering: linear attention runs in its recurrent
// form, full attention as a naive masked softmax, one token at a time.
// OpenMP only splits independent output elements across threads, so results do
// not depend on the thread count.
//
// Only tests/, the smoke entry and the bench's CPU-baseline leg may load this
// library.  It shares no code with the CUDA library.

#include "oracle.h"

#include <cmath>
#include <cstdint>
#include <cstring>
#include <memory>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Generator: SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) as a counter stream.
// ---------------------------------------------------------------------------
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t stream_key(uint64_t seed, uint64_t stream) { return mix64(mix64(seed) + stream); }

uint64_t draw(uint64_t key, uint64_t j) { return mix64(key + (j + 1) * kGamma); }

// Box-Muller on the pair containing element i (even: cosine, odd: sine).
double normal_at(uint64_t key, uint64_t i) {
  const uint64_t p = i >> 1;
  const double u1 = (double)((draw(key, 2 * p) >> 11) + 1) * 0x1.0p-53;
  const double u2 = (double)(draw(key, 2 * p + 1) >> 11) * 0x1.0p-53;
  const double r = std::sqrt(-2.0 * std::log(u1));
  const double t = 2.0 * M_PI * u2;
  return (i & 1) ? r * std::sin(t) : r * std::cos(t);
}

// Round an fp32 value to the nearest bf16 (ties to even), kept as fp32.
float round_bf16(float x) {
  uint32_t b;
  std::memcpy(&b, &x, 4);
  b = (b + 0x7FFFu + ((b >> 16) & 1u)) & 0xFFFF0000u;
  float y;
  std::memcpy(&y, &b, 4);
  return y;
}

double round_act(double x, bool bf16) { return bf16 ? (double)round_bf16((float)x) : x; }

// Tensor streams.
uint64_t layer_stream(int layer, int kind) { return 1000 + 100 * (uint64_t)layer + kind; }
uint64_t site_stream(int site) { return 100000 + 10 * (uint64_t)site + 1; }
constexpr uint64_t kStreamEmbed = 1;

// ---------------------------------------------------------------------------
// The spec-defined exponential used by Sinkhorn, in fp32: Cody-Waite
// reduction x = k ln2 + r with ln2 split into a 15-bit head (22713 / 32768,
// so k * head is exact for |k| < 512) and its remainder, then the degree-7
// Taylor polynomial sum r^j / j! by Horner with fused multiply-adds, scaled
// by 2^k.  Truncation error |r|^8 / 8! < 5.2e-9 for |r| <= ln2 / 2.
// ---------------------------------------------------------------------------
float exp_spec(float x) {
  if (std::isnan(x)) return x;
  if (x < -104.0f) return 0.0f;
  if (x > 88.72f) return INFINITY;
  const float log2e = 1.44269504088896340736f;
  const float ln2_hi = 0.693145751953125f;       // 22713 / 32768
  const float ln2_lo = 1.42860682030941723212e-6f;  // ln 2 - ln2_hi
  const float k = std::nearbyint(x * log2e);
  float r = std::fma(-k, ln2_hi, x);
  r = std::fma(-k, ln2_lo, r);
  float p = 1.0f / 5040.0f;
  p = std::fma(p, r, 1.0f / 720.0f);
  p = std::fma(p, r, 1.0f / 120.0f);
  p = std::fma(p, r, 1.0f / 24.0f);
  p = std::fma(p, r, 1.0f / 6.0f);
  p = std::fma(p, r, 0.5f);
  p = std::fma(p, r, 1.0f);
  p = std::fma(p, r, 1.0f);
  return std::ldexp(p, (int)k);
}

// Sinkhorn (the mHC mixing map): exponentiate, then alternately divide each
// row by its sum and each column by its sum, `iters` times (rows first).  The
// global maximum is subtracted before exponentiating; the first row division
// cancels any common factor, so this changes nothing in exact arithmetic.
template <typename T, typename ExpFn>
void sinkhorn_one(const T* l, T* P, int n, int iters, ExpFn ex) {
  T mx = l[0];
  for (int i = 1; i < n * n; ++i) mx = l[i] > mx ? l[i] : mx;
  for (int i = 0; i < n * n; ++i) P[i] = ex(l[i] - mx);
  for (int it = 0; it < iters; ++it) {
    for (int r = 0; r < n; ++r) {
      T s = 0;
      for (int c = 0; c < n; ++c) s = s + P[r * n + c];
      for (int c = 0; c < n; ++c) P[r * n + c] = P[r * n + c] / s;
    }
    for (int c = 0; c < n; ++c) {
      T s = 0;
      for (int r = 0; r < n; ++r) s = s + P[r * n + c];
      for (int r = 0; r < n; ++r) P[r * n + c] = P[r * n + c] / s;
    }
  }
}

double sigmoid(double x) { return 1.0 / (1.0 + std::exp(-x)); }

// ---------------------------------------------------------------------------
// Model
// ---------------------------------------------------------------------------
enum WeightSlot { W_ATTN_GAIN, W_Q, W_K, W_V, W_G, W_O, W_FFN_GAIN, W_GATE, W_UP, W_DOWN, W_PER_LAYER };

struct Model {
  oracle_config c{};
  int n_phys = 0, n_exec = 0, n_full = 0, n_lin = 0, n_coef = 0;
  std::vector<int32_t> table;            // n_exec x 5
  std::vector<std::vector<float>> w;     // by weight index
  std::vector<std::vector<float>> kc, vc;  // per full slot [max_batch][n_kv][max_ctx][hd]
  std::vector<std::vector<double>> st;   // per linear slot [max_batch][n_lin][ld][ld]
  std::vector<int32_t> seq_len;

  bool bf16() const { return c.dtype == 1; }
  bool is_full(int phys) const { return phys % c.group == c.full_slot; }
  int widx_layer(int phys, int slot) const { return 2 + W_PER_LAYER * phys + slot; }
  int widx_site(int site, int which) const { return 2 + W_PER_LAYER * n_phys + 2 * site + which; }
};

bool config_ok(const oracle_config* c) {
  if (!c) return false;
  if (c->n_prelude < 0 || c->n_block <= 0 || c->n_loops <= 0 || c->n_coda < 0) return false;
  if (c->group <= 0 || c->full_slot < 0 || c->full_slot >= c->group) return false;
  if (c->n_prelude % c->group || c->n_block % c->group) return false;
  if (c->hidden <= 0 || c->ffn <= 0 || c->n_streams <= 0 || c->sinkhorn_iters < 0) return false;
  if (c->n_q <= 0 || c->n_kv <= 0 || c->n_q % c->n_kv || c->head_dim <= 0 || c->head_dim % 2) return false;
  if (c->n_lin <= 0 || c->lin_dim <= 0) return false;
  if (c->io_mode == 0 && c->vocab <= 0) return false;
  if (c->max_batch <= 0 || c->max_ctx <= 0) return false;
  return true;
}

std::vector<int64_t> weight_shape(const oracle_config& c, int index) {
  const int n_phys = c.n_prelude + c.n_block + c.n_coda;
  const int64_t H = c.hidden, F = c.ffn;
  if (index == 0) return c.io_mode == 0 ? std::vector<int64_t>{c.vocab, H} : std::vector<int64_t>{0};
  if (index == 1) return {H};
  int i = index - 2;
  if (i < W_PER_LAYER * n_phys) {
    const int phys = i / W_PER_LAYER, slot = i % W_PER_LAYER;
    const bool full = phys % c.group == c.full_slot;
    const int64_t nq = full ? (int64_t)c.n_q * c.head_dim : (int64_t)c.n_lin * c.lin_dim;
    const int64_t nkv = full ? (int64_t)c.n_kv * c.head_dim : (int64_t)c.n_lin * c.lin_dim;
    switch (slot) {
      case W_ATTN_GAIN: case W_FFN_GAIN: return {H};
      case W_Q: return {nq, H};
      case W_K: case W_V: return {nkv, H};
      case W_G: return full ? std::vector<int64_t>{0} : std::vector<int64_t>{c.n_lin, H};
      case W_O: return {H, nq};
      case W_GATE: case W_UP: return {F, H};
      case W_DOWN: return {H, F};
    }
  }
  i -= W_PER_LAYER * n_phys;
  const int n = c.n_streams;
  if (i < 4 * c.n_block) return (i % 2 == 0) ? std::vector<int64_t>{n * H}
                                             : std::vector<int64_t>{2 * n + n * n, n * H};
  return {-1};
}

int64_t numel(const std::vector<int64_t>& s) {
  int64_t p = 1;
  for (auto d : s) p *= d;
  return p;
}

void fill_normal(std::vector<float>& v, uint64_t seed, uint64_t stream, bool bf16) {
  const uint64_t key = stream_key(seed, stream);
  const int64_t n = (int64_t)v.size();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    float x = (float)(0.02 * normal_at(key, (uint64_t)i));
    v[i] = bf16 ? round_bf16(x) : x;
  }
}

// y[t][o] = sum_k x[t][k] * W[o][k]     (W stored [out][in])
void linear(const std::vector<double>& x, const float* W, std::vector<double>& y, int64_t T, int64_t K,
            int64_t N) {
  y.assign(T * N, 0.0);
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < N; ++o) {
    const float* wr = W + o * K;
    for (int64_t t = 0; t < T; ++t) {
      const double* xr = x.data() + t * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += xr[k] * (double)wr[k];
      y[t * N + o] = acc;
    }
  }
}

void rmsnorm_rows(const double* x, const double* gain, double* y, int64_t rows, int dim, double eps) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    double ss = 0.0;
    for (int i = 0; i < dim; ++i) ss += x[r * dim + i] * x[r * dim + i];
    const double inv = 1.0 / std::sqrt(ss / dim + eps);
    for (int i = 0; i < dim; ++i) y[r * dim + i] = x[r * dim + i] * inv * gain[i];
  }
}

// Rotate-half RoPE: pairs (i, i + d/2) rotate by pos * base^(-2i/d).
void rope_rows(double* x, int64_t T, int heads, int d, const int32_t* pos, double base) {
  const int half = d / 2;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int h = 0; h < heads; ++h) {
      double* v = x + (t * heads + h) * d;
      for (int i = 0; i < half; ++i) {
        const double ang = (double)pos[t] * std::pow(base, -2.0 * i / d);
        const double c = std::cos(ang), s = std::sin(ang);
        const double a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
      }
    }
  }
}

// One mHC site for one token: read coefficients from the flattened streams,
// then read x = sum_i H_pre[i] s_i and normalise it.
//   r   = RMS over all n*H stream entries
//   l   = ((s / r) * gamma_m) . Phi          (2n + n^2 values)
//   H_pre = sigmoid(l[0:n]), H_post = 2 sigmoid(l[n:2n]),
//   H_res = Sinkhorn_iters(exp(l[2n:] as n x n, row-major))
void mhc_site_one(const double* s, const double* gamma_m, const float* phi_f, const double* phi_d,
                  const double* gain, int n, int H, int iters, double eps, double* coef, double* xhat) {
  const int nc = 2 * n + n * n;
  const int64_t D = (int64_t)n * H;
  double ss = 0.0;
  for (int64_t i = 0; i < D; ++i) ss += s[i] * s[i];
  const double inv = 1.0 / std::sqrt(ss / D + eps);
  std::vector<double> l(nc, 0.0);
  for (int c = 0; c < nc; ++c) {
    double acc = 0.0;
    for (int64_t i = 0; i < D; ++i) {
      const double p = phi_f ? (double)phi_f[c * D + i] : phi_d[c * D + i];
      acc += s[i] * inv * gamma_m[i] * p;
    }
    l[c] = acc;
  }
  for (int i = 0; i < n; ++i) coef[i] = sigmoid(l[i]);
  for (int i = 0; i < n; ++i) coef[n + i] = 2.0 * sigmoid(l[n + i]);
  sinkhorn_one<double>(l.data() + 2 * n, coef + 2 * n, n, iters, [](double v) { return std::exp(v); });
  std::vector<double> x(H, 0.0);
  for (int i = 0; i < n; ++i)
    for (int k = 0; k < H; ++k) x[k] += coef[i] * s[(int64_t)i * H + k];
  double xs = 0.0;
  for (int k = 0; k < H; ++k) xs += x[k] * x[k];
  const double xinv = 1.0 / std::sqrt(xs / H + eps);
  for (int k = 0; k < H; ++k) xhat[k] = x[k] * xinv * gain[k];
}

// Write the sublayer output back: s_i <- sum_j H_res[i][j] s_j + H_post[i] y.
void mhc_write_one(double* s, const double* coef, const double* y, int n, int H) {
  std::vector<double> out((size_t)n * H, 0.0);
  const double* post = coef + n;
  const double* res = coef + 2 * n;
  for (int i = 0; i < n; ++i)
    for (int k = 0; k < H; ++k) {
      double acc = 0.0;
      for (int j = 0; j < n; ++j) acc += res[i * n + j] * s[(int64_t)j * H + k];
      out[(size_t)i * H + k] = acc + post[i] * y[k];
    }
  std::memcpy(s, out.data(), sizeof(double) * n * H);
}

std::vector<double> to_double(const std::vector<float>& v) { return std::vector<double>(v.begin(), v.end()); }

// Weights of one attention sublayer ([out][in] fp32 values).  wg is the
// linear-attention gate projection (unused by full attention).
struct AttnWeights {
  const float *wq, *wk, *wv, *wg, *wo;
};

// The full-attention sublayer over B sequences of S new tokens each, the
// tokens of sequence b at positions start[b] ..: q, k, v projections, RoPE on
// q and k, K and V appended to the cache slot (K, V: [B][n_kv][max_ctx][hd]),
// causal softmax attention with kv head = q head / (n_q / n_kv) and scale
// 1/sqrt(hd), then the output projection into y [T][H].
void full_attention_core(const oracle_config& c, const AttnWeights& w, float* K, float* V,
                         const std::vector<double>& xh, int B, int S, const std::vector<int32_t>& start,
                         std::vector<double>& y) {
  const int64_t T = (int64_t)B * S, H = c.hidden, hd = c.head_dim;
  const int nq = c.n_q, nkv = c.n_kv, grp = nq / nkv;
  std::vector<double> q, k, v;
  linear(xh, w.wq, q, T, H, nq * hd);
  linear(xh, w.wk, k, T, H, nkv * hd);
  linear(xh, w.wv, v, T, H, nkv * hd);
  std::vector<int32_t> pos(T);
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < S; ++t) pos[(int64_t)b * S + t] = start[b] + t;
  rope_rows(q.data(), T, nq, hd, pos.data(), c.rope_base);
  rope_rows(k.data(), T, nkv, hd, pos.data(), c.rope_base);
  const bool bf = c.dtype == 1;
  for (auto& x : q) x = round_act(x, bf);
  for (auto& x : k) x = round_act(x, bf);
  for (auto& x : v) x = round_act(x, bf);
  // append K, V to this execution's cache slot
  const int64_t L = c.max_ctx;
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < S; ++t)
      for (int h = 0; h < nkv; ++h)
        for (int i = 0; i < hd; ++i) {
          const int64_t src = (((int64_t)b * S + t) * nkv + h) * hd + i;
          const int64_t dst = (((int64_t)b * nkv + h) * L + start[b] + t) * hd + i;
          K[dst] = (float)k[src];
          V[dst] = (float)v[src];
        }
  std::vector<double> o(T * nq * hd, 0.0);
  const double scale = 1.0 / std::sqrt((double)hd);
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < nq; ++h) {
      const int kh = h / grp;
      const float* Kb = K + ((int64_t)b * nkv + kh) * L * hd;
      const float* Vb = V + ((int64_t)b * nkv + kh) * L * hd;
      std::vector<double> sc;
      for (int t = 0; t < S; ++t) {
        const int p = start[b] + t;
        const double* qr = q.data() + (((int64_t)b * S + t) * nq + h) * hd;
        sc.assign(p + 1, 0.0);
        double mx = -INFINITY;
        for (int j = 0; j <= p; ++j) {
          double acc = 0.0;
          for (int i = 0; i < hd; ++i) acc += qr[i] * (double)Kb[(int64_t)j * hd + i];
          sc[j] = acc * scale;
          mx = sc[j] > mx ? sc[j] : mx;
        }
        double den = 0.0;
        for (int j = 0; j <= p; ++j) {
          sc[j] = std::exp(sc[j] - mx);
          den += sc[j];
        }
        double* orow = o.data() + (((int64_t)b * S + t) * nq + h) * hd;
        for (int j = 0; j <= p; ++j) {
          const double wgt = sc[j] / den;
          for (int i = 0; i < hd; ++i) orow[i] += wgt * (double)Vb[(int64_t)j * hd + i];
        }
      }
    }
  for (auto& x : o) x = round_act(x, bf);
  linear(o, w.wo, y, T, nq * hd, H);
}

// The gated-linear-attention sublayer: q, k L2-normalised per head (eps
// inside the square root), scalar gate g = sigmoid(x W_g) per head;
// S_t = g_t S_{t-1} + k_t v_t^T, o_t = q_t S_t, starting from and leaving the
// state in `state` [B][n_lin][d][d]; then the output projection into y.
void linear_attention_core(const oracle_config& c, const AttnWeights& w, double* state,
                           const std::vector<double>& xh, int B, int S, std::vector<double>& y) {
  const int64_t T = (int64_t)B * S, H = c.hidden, d = c.lin_dim;
  const int nh = c.n_lin;
  std::vector<double> q, k, v, z;
  linear(xh, w.wq, q, T, H, nh * d);
  linear(xh, w.wk, k, T, H, nh * d);
  linear(xh, w.wv, v, T, H, nh * d);
  linear(xh, w.wg, z, T, H, nh);
  const double eps = c.norm_eps;
  for (int64_t r = 0; r < T * nh; ++r) {
    double sq = 0.0, sk = 0.0;
    for (int i = 0; i < d; ++i) {
      sq += q[r * d + i] * q[r * d + i];
      sk += k[r * d + i] * k[r * d + i];
    }
    const double iq = 1.0 / std::sqrt(sq + eps), ik = 1.0 / std::sqrt(sk + eps);
    for (int i = 0; i < d; ++i) {
      q[r * d + i] *= iq;
      k[r * d + i] *= ik;
    }
  }
  const bool bf = c.dtype == 1;
  for (auto& x : q) x = round_act(x, bf);
  for (auto& x : k) x = round_act(x, bf);
  for (auto& x : v) x = round_act(x, bf);
  std::vector<double> o(T * nh * d, 0.0);
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < nh; ++h) {
      double* Sm = state + ((int64_t)b * nh + h) * d * d;
      for (int t = 0; t < S; ++t) {
        const int64_t row = (int64_t)b * S + t;
        const double g = sigmoid(z[row * nh + h]);
        const double* kt = k.data() + (row * nh + h) * d;
        const double* vt = v.data() + (row * nh + h) * d;
        const double* qt = q.data() + (row * nh + h) * d;
        for (int a = 0; a < d; ++a)
          for (int e = 0; e < d; ++e) Sm[a * d + e] = g * Sm[a * d + e] + kt[a] * vt[e];
        double* ot = o.data() + (row * nh + h) * d;
        for (int e = 0; e < d; ++e) {
          double acc = 0.0;
          for (int a = 0; a < d; ++a) acc += qt[a] * Sm[a * d + e];
          ot[e] = acc;
        }
      }
    }
  for (auto& x : o) x = round_act(x, bf);
  linear(o, w.wo, y, T, nh * d, H);
}

// SwiGLU: y = W_down (silu(x W_gate) * (x W_up)).
void ffn_core(const oracle_config& c, const float* w_gate, const float* w_up, const float* w_down,
              const std::vector<double>& xh, int64_t T, std::vector<double>& y) {
  std::vector<double> g, u;
  linear(xh, w_gate, g, T, c.hidden, c.ffn);
  linear(xh, w_up, u, T, c.hidden, c.ffn);
  const bool bf = c.dtype == 1;
  for (int64_t i = 0; i < T * c.ffn; ++i) g[i] = round_act(g[i] * sigmoid(g[i]) * u[i], bf);
  linear(g, w_down, y, T, c.ffn, c.hidden);
}

AttnWeights layer_weights(const Model& m, int phys) {
  return {m.w[m.widx_layer(phys, W_Q)].data(), m.w[m.widx_layer(phys, W_K)].data(),
          m.w[m.widx_layer(phys, W_V)].data(), m.w[m.widx_layer(phys, W_G)].data(),
          m.w[m.widx_layer(phys, W_O)].data()};
}

void full_attention(Model& m, int phys, int slot, const std::vector<double>& xh, int B, int S,
                    const std::vector<int32_t>& start, std::vector<double>& y) {
  full_attention_core(m.c, layer_weights(m, phys), m.kc[slot].data(), m.vc[slot].data(), xh, B, S, start, y);
}

void linear_attention(Model& m, int phys, int slot, const std::vector<double>& xh, int B, int S,
                      std::vector<double>& y) {
  linear_attention_core(m.c, layer_weights(m, phys), m.st[slot].data(), xh, B, S, y);
}

void ffn(Model& m, int phys, const std::vector<double>& xh, int64_t T, std::vector<double>& y) {
  ffn_core(m.c, m.w[m.widx_layer(phys, W_GATE)].data(), m.w[m.widx_layer(phys, W_UP)].data(),
           m.w[m.widx_layer(phys, W_DOWN)].data(), xh, T, y);
}

// The forward pass over B sequences of S new tokens starting at start[b].
int forward(Model& m, const int32_t* tokens, const float* hidden, int B, int S,
            const std::vector<int32_t>& start, float* out, uint32_t flags, bool last_only) {
  const oracle_config& c = m.c;
  const int64_t T = (int64_t)B * S, H = c.hidden;
  const int n = c.n_streams;
  const bool bf = m.bf16();
  std::vector<double> h(T * H);
  if (c.io_mode == 0) {
    const std::vector<float>& E = m.w[0];
    for (int64_t t = 0; t < T; ++t) {
      const int32_t tok = tokens[t];
      if (tok < 0 || tok >= c.vocab) return -1;
      for (int64_t i = 0; i < H; ++i) h[t * H + i] = E[(int64_t)tok * H + i];
    }
  } else {
    for (int64_t i = 0; i < T * H; ++i) h[i] = hidden[i];
  }
  std::vector<double> s;  // streams [n][T][H]
  std::vector<double> xh(T * H), y, coef((size_t)T * (2 * n + n * n));
  const int first_block = c.n_prelude, last_block = c.n_prelude + c.n_block * c.n_loops - 1;
  for (int e = 0; e < m.n_exec; ++e) {
    const int32_t* row = &m.table[5 * e];
    const int phys = row[0], kind = row[2], slot = row[3], region = row[4];
    if (e == first_block) {  // expand: every stream starts as a copy of h
      s.assign((size_t)n * T * H, 0.0);
      for (int i = 0; i < n; ++i) std::memcpy(&s[(size_t)i * T * H], h.data(), sizeof(double) * T * H);
    }
    for (int sub = 0; sub < 2; ++sub) {
      const std::vector<double> gain = to_double(m.w[m.widx_layer(phys, sub == 0 ? W_ATTN_GAIN : W_FFN_GAIN)]);
      if (region == ORACLE_BLOCK) {
        const int site = 2 * (phys - c.n_prelude) + sub;
        const std::vector<double> gm = to_double(m.w[m.widx_site(site, 0)]);
        const float* phi = m.w[m.widx_site(site, 1)].data();
        const int nc = 2 * n + n * n;
#pragma omp parallel for schedule(dynamic)
        for (int64_t t = 0; t < T; ++t) {
          std::vector<double> sv((size_t)n * H);
          for (int i = 0; i < n; ++i)
            std::memcpy(&sv[(size_t)i * H], &s[((size_t)i * T + t) * H], sizeof(double) * H);
          mhc_site_one(sv.data(), gm.data(), phi, nullptr, gain.data(), n, (int)H, c.sinkhorn_iters,
                       c.norm_eps, &coef[t * nc], &xh[t * H]);
        }
      } else {
        rmsnorm_rows(h.data(), gain.data(), xh.data(), T, (int)H, c.norm_eps);
      }
      for (auto& x : xh) x = round_act(x, bf);
      if (sub == 0) {
        if (kind == ORACLE_FULL) full_attention(m, phys, slot, xh, B, S, start, y);
        else linear_attention(m, phys, slot, xh, B, S, y);
      } else {
        ffn(m, phys, xh, T, y);
      }
      if (region == ORACLE_BLOCK) {
        const int nc = 2 * n + n * n;
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
          std::vector<double> sv((size_t)n * H);
          for (int i = 0; i < n; ++i)
            std::memcpy(&sv[(size_t)i * H], &s[((size_t)i * T + t) * H], sizeof(double) * H);
          mhc_write_one(sv.data(), &coef[t * nc], &y[t * H], n, (int)H);
          for (int i = 0; i < n; ++i)
            std::memcpy(&s[((size_t)i * T + t) * H], &sv[(size_t)i * H], sizeof(double) * H);
        }
      } else {
        for (int64_t i = 0; i < T * H; ++i) h[i] += y[i];
      }
    }
    if (e == last_block) {  // collapse: h = sum of the streams
      for (int64_t i = 0; i < T * H; ++i) {
        double acc = 0.0;
        for (int j = 0; j < n; ++j) acc += s[(size_t)j * T * H + i];
        h[i] = acc;
      }
    }
  }
  if (c.io_mode == 1) {
    for (int64_t i = 0; i < T * H; ++i) out[i] = (float)h[i];
    return 0;
  }
  // final norm + tied head
  std::vector<int64_t> rows;
  if ((flags & ORACLE_ALL_POSITIONS) && !last_only)
    for (int64_t t = 0; t < T; ++t) rows.push_back(t);
  else
    for (int b = 0; b < B; ++b) rows.push_back((int64_t)b * S + S - 1);
  const std::vector<double> fg = to_double(m.w[1]);
  std::vector<double> xr(rows.size() * H), xn(rows.size() * H);
  for (size_t r = 0; r < rows.size(); ++r)
    std::memcpy(&xr[r * H], &h[rows[r] * H], sizeof(double) * H);
  rmsnorm_rows(xr.data(), fg.data(), xn.data(), (int64_t)rows.size(), (int)H, c.norm_eps);
  for (auto& x : xn) x = round_act(x, bf);
  std::vector<double> lg;
  linear(xn, m.w[0].data(), lg, (int64_t)rows.size(), H, c.vocab);
  for (size_t i = 0; i < lg.size(); ++i) out[i] = (float)lg[i];
  return 0;
}

}  // namespace

extern "C" {

uint64_t oracle_rng_u64(uint64_t seed, uint64_t stream, uint64_t j) { return draw(stream_key(seed, stream), j); }

double oracle_rng_normal(uint64_t seed, uint64_t stream, uint64_t i) {
  return normal_at(stream_key(seed, stream), i);
}

float oracle_exp_spec(float x) { return exp_spec(x); }

void oracle_sinkhorn_f32(const float* logits, float* out, int64_t count, int32_t n, int32_t iters) {
  for (int64_t i = 0; i < count; ++i)
    sinkhorn_one<float>(logits + i * n * n, out + i * n * n, n, iters, exp_spec);
}

void oracle_sinkhorn_f64(const double* logits, double* out, int64_t count, int32_t n, int32_t iters) {
  for (int64_t i = 0; i < count; ++i)
    sinkhorn_one<double>(logits + i * n * n, out + i * n * n, n, iters, [](double v) { return std::exp(v); });
}

int32_t oracle_num_exec(const oracle_config* c) {
  if (!config_ok(c)) return -1;
  return c->n_prelude + c->n_block * c->n_loops + c->n_coda;
}

// Execution table.  Prelude execution e runs layer e; block execution
// e = n_prelude + p * n_block + j runs layer n_prelude + j in pass p; coda
// executions run the remaining layers once.  A layer is full attention when
// its position in its group equals full_slot.  Each execution owns its own
// cache slot: the k-th full-attention execution owns KV slot k and the k-th
// linear execution owns state slot k, so the two passes keep separate caches.
int32_t oracle_schedule(const oracle_config* c, int32_t* table) {
  const int n_exec = oracle_num_exec(c);
  if (n_exec < 0) return -1;
  int nf = 0, nl = 0;
  for (int e = 0; e < n_exec; ++e) {
    int phys, pass, region;
    if (e < c->n_prelude) {
      phys = e; pass = 0; region = ORACLE_PRELUDE;
    } else if (e < c->n_prelude + c->n_block * c->n_loops) {
      const int j = e - c->n_prelude;
      pass = j / c->n_block; phys = c->n_prelude + j % c->n_block; region = ORACLE_BLOCK;
    } else {
      phys = c->n_prelude + c->n_block + (e - c->n_prelude - c->n_block * c->n_loops);
      pass = 0; region = ORACLE_CODA;
    }
    const int kind = (phys % c->group == c->full_slot) ? ORACLE_FULL : ORACLE_LINEAR;
    table[5 * e + 0] = phys;
    table[5 * e + 1] = pass;
    table[5 * e + 2] = kind;
    table[5 * e + 3] = kind == ORACLE_FULL ? nf++ : nl++;
    table[5 * e + 4] = region;
  }
  return n_exec;
}

void oracle_rmsnorm(const double* x, const double* gain, double* y, int64_t rows, int32_t dim, double eps) {
  rmsnorm_rows(x, gain, y, rows, dim, eps);
}

void oracle_gla_recurrent(const double* q, const double* k, const double* v, const double* g, double* o,
                          double* state, int32_t T, int32_t dk, int32_t dv) {
  for (int t = 0; t < T; ++t) {
    for (int a = 0; a < dk; ++a)
      for (int e = 0; e < dv; ++e)
        state[a * dv + e] = g[t] * state[a * dv + e] + k[t * dk + a] * v[t * dv + e];
    for (int e = 0; e < dv; ++e) {
      double acc = 0.0;
      for (int a = 0; a < dk; ++a) acc += q[t * dk + a] * state[a * dv + e];
      o[t * dv + e] = acc;
    }
  }
}

void oracle_attention_naive(const double* q, const double* k, const double* v, double* o, int32_t Tq,
                            int32_t Tk, int32_t q0, int32_t d) {
  const double scale = 1.0 / std::sqrt((double)d);
  for (int i = 0; i < Tq; ++i) {
    const int last = std::min(q0 + i, Tk - 1);
    std::vector<double> sc(last + 1);
    double mx = -INFINITY;
    for (int j = 0; j <= last; ++j) {
      double acc = 0.0;
      for (int a = 0; a < d; ++a) acc += q[i * d + a] * k[j * d + a];
      sc[j] = acc * scale;
      mx = std::max(mx, sc[j]);
    }
    double den = 0.0;
    for (int j = 0; j <= last; ++j) den += (sc[j] = std::exp(sc[j] - mx));
    for (int a = 0; a < d; ++a) {
      double acc = 0.0;
      for (int j = 0; j <= last; ++j) acc += sc[j] / den * v[j * d + a];
      o[i * d + a] = acc;
    }
  }
}

void oracle_rope(double* x, int32_t T, int32_t n_heads, int32_t d, const int32_t* pos, double base) {
  rope_rows(x, T, n_heads, d, pos, base);
}

void oracle_mhc_site(const double* s, const double* gamma_m, const double* phi, const double* gain, int32_t n,
                     int32_t H, int32_t iters, double eps, double* coef, double* xhat) {
  mhc_site_one(s, gamma_m, nullptr, phi, gain, n, H, iters, eps, coef, xhat);
}

void oracle_mhc_write(double* s, const double* coef, const double* y, int32_t n, int32_t H) {
  mhc_write_one(s, coef, y, n, H);
}

// The three sublayers the model runs, on caller arrays (the model calls the
// same functions with its own weights and cache slots).  xh [B*S][hidden] and
// y [B*S][hidden] are fp64; weights are fp32 [out][in]; dtype 1 rounds the
// activations entering matrix products to bf16 as the model does.
int32_t oracle_attention_sublayer(const oracle_config* c, const float* wq, const float* wk, const float* wv,
                                  const float* wo, float* kcache, float* vcache, const double* xh, int32_t B,
                                  int32_t S, const int32_t* start, double* y) {
  if (!config_ok(c) || B <= 0 || S <= 0 || B > c->max_batch) return -1;
  for (int b = 0; b < B; ++b)
    if (start[b] < 0 || start[b] + S > c->max_ctx) return -1;
  const int64_t T = (int64_t)B * S, H = c->hidden;
  std::vector<double> x(xh, xh + T * H), out;
  const AttnWeights w{wq, wk, wv, nullptr, wo};
  full_attention_core(*c, w, kcache, vcache, x, B, S, std::vector<int32_t>(start, start + B), out);
  std::memcpy(y, out.data(), sizeof(double) * T * H);
  return 0;
}

int32_t oracle_gla_sublayer(const oracle_config* c, const float* wq, const float* wk, const float* wv,
                            const float* wg, const float* wo, double* state, const double* xh, int32_t B, int32_t S,
                            double* y) {
  if (!config_ok(c) || B <= 0 || S <= 0) return -1;
  const int64_t T = (int64_t)B * S, H = c->hidden;
  std::vector<double> x(xh, xh + T * H), out;
  const AttnWeights w{wq, wk, wv, wg, wo};
  linear_attention_core(*c, w, state, x, B, S, out);
  std::memcpy(y, out.data(), sizeof(double) * T * H);
  return 0;
}

int32_t oracle_ffn_sublayer(const oracle_config* c, const float* w_gate, const float* w_up, const float* w_down,
                            const double* xh, int64_t T, double* y) {
  if (!config_ok(c) || T <= 0) return -1;
  const int64_t H = c->hidden;
  std::vector<double> x(xh, xh + T * H), out;
  ffn_core(*c, w_gate, w_up, w_down, x, T, out);
  std::memcpy(y, out.data(), sizeof(double) * T * H);
  return 0;
}

int32_t oracle_num_weights(const oracle_config* c) {
  if (!config_ok(c)) return -1;
  return 2 + W_PER_LAYER * (c->n_prelude + c->n_block + c->n_coda) + 4 * c->n_block;
}

void* oracle_model_create(const oracle_config* c, uint64_t seed, const float* const* weights) {
  if (!config_ok(c)) return nullptr;
  auto m = std::make_unique<Model>();
  m->c = *c;
  m->n_phys = c->n_prelude + c->n_block + c->n_coda;
  m->n_exec = oracle_num_exec(c);
  m->n_coef = 2 * c->n_streams + c->n_streams * c->n_streams;
  m->table.resize(5 * m->n_exec);
  oracle_schedule(c, m->table.data());
  for (int e = 0; e < m->n_exec; ++e) (m->table[5 * e + 2] == ORACLE_FULL ? m->n_full : m->n_lin)++;
  const int nw = oracle_num_weights(c);
  m->w.resize(nw);
  const bool bf = c->dtype == 1;
  for (int i = 0; i < nw; ++i) {
    m->w[i].assign(numel(weight_shape(*c, i)), 0.0f);
    if (weights) {
      if (!m->w[i].empty()) {
        if (!weights[i]) return nullptr;
        std::memcpy(m->w[i].data(), weights[i], sizeof(float) * m->w[i].size());
      }
      continue;
    }
    // seeded: gains are 1, matrices 0.02 * N(0, 1)
    if (i == 0) {
      fill_normal(m->w[i], seed, kStreamEmbed, bf);
    } else if (i == 1) {
      std::fill(m->w[i].begin(), m->w[i].end(), 1.0f);
    } else if (i - 2 < W_PER_LAYER * m->n_phys) {
      const int phys = (i - 2) / W_PER_LAYER, slot = (i - 2) % W_PER_LAYER;
      if (slot == W_ATTN_GAIN || slot == W_FFN_GAIN) std::fill(m->w[i].begin(), m->w[i].end(), 1.0f);
      else fill_normal(m->w[i], seed, layer_stream(phys, slot), bf);
    } else {
      const int j = i - 2 - W_PER_LAYER * m->n_phys;
      if (j % 2 == 0) std::fill(m->w[i].begin(), m->w[i].end(), 1.0f);
      else fill_normal(m->w[i], seed, site_stream(j / 2), false);  // mHC parameters stay fp32
    }
  }
  const int64_t L = c->max_ctx, Bm = c->max_batch;
  m->kc.resize(m->n_full);
  m->vc.resize(m->n_full);
  for (int i = 0; i < m->n_full; ++i) {
    m->kc[i].assign(Bm * c->n_kv * L * c->head_dim, 0.0f);
    m->vc[i].assign(Bm * c->n_kv * L * c->head_dim, 0.0f);
  }
  m->st.resize(m->n_lin);
  for (int i = 0; i < m->n_lin; ++i) m->st[i].assign(Bm * c->n_lin * (int64_t)c->lin_dim * c->lin_dim, 0.0);
  m->seq_len.assign(Bm, 0);
  return m.release();
}

int64_t oracle_weight_numel(void* mp, int32_t index) {
  Model* m = (Model*)mp;
  if (!m || index < 0 || index >= (int)m->w.size()) return -1;
  return (int64_t)m->w[index].size();
}

int32_t oracle_get_weight(void* mp, int32_t index, float* out) {
  Model* m = (Model*)mp;
  if (!m || index < 0 || index >= (int)m->w.size()) return -1;
  std::memcpy(out, m->w[index].data(), sizeof(float) * m->w[index].size());
  return 0;
}

int32_t oracle_prefill(void* mp, const int32_t* tokens, const float* hidden, int32_t B, int32_t S, float* out,
                       uint32_t flags) {
  Model* m = (Model*)mp;
  if (!m || B <= 0 || S <= 0 || B > m->c.max_batch || S > m->c.max_ctx) return -1;
  for (int i = 0; i < m->n_lin; ++i)
    std::fill(m->st[i].begin(), m->st[i].begin() + (int64_t)B * m->c.n_lin * m->c.lin_dim * m->c.lin_dim, 0.0);
  std::vector<int32_t> start(B, 0);
  const int rc = forward(*m, tokens, hidden, B, S, start, out, flags, false);
  if (rc == 0)
    for (int b = 0; b < B; ++b) m->seq_len[b] = S;
  return rc;
}

int32_t oracle_decode_step(void* mp, const int32_t* tokens, int32_t B, float* logits) {
  Model* m = (Model*)mp;
  if (!m || B <= 0 || B > m->c.max_batch || m->c.io_mode != 0) return -1;
  std::vector<int32_t> start(m->seq_len.begin(), m->seq_len.begin() + B);
  for (int b = 0; b < B; ++b)
    if (start[b] + 1 > m->c.max_ctx) return -1;
  const int rc = forward(*m, tokens, nullptr, B, 1, start, logits, 0, true);
  if (rc == 0)
    for (int b = 0; b < B; ++b) m->seq_len[b] += 1;
  return rc;
}

int32_t oracle_seq_len(void* mp, int32_t b) {
  Model* m = (Model*)mp;
  if (!m || b < 0 || b >= m->c.max_batch) return -1;
  return m->seq_len[b];
}

int32_t oracle_cache_read(void* mp, int32_t kind, int32_t slot, int32_t B, int32_t len, float* out) {
  Model* m = (Model*)mp;
  if (!m || B <= 0 || B > m->c.max_batch) return -1;
  const oracle_config& c = m->c;
  if (kind == ORACLE_FULL) {
    if (slot < 0 || slot >= m->n_full || len < 0 || len > c.max_ctx) return -1;
    const int64_t hd = c.head_dim, L = c.max_ctx;
    int64_t o = 0;
    for (int which = 0; which < 2; ++which) {
      const std::vector<float>& src = which == 0 ? m->kc[slot] : m->vc[slot];
      for (int b = 0; b < B; ++b)
        for (int h = 0; h < c.n_kv; ++h)
          for (int p = 0; p < len; ++p)
            for (int i = 0; i < hd; ++i) out[o++] = src[(((int64_t)b * c.n_kv + h) * L + p) * hd + i];
    }
    return 0;
  }
  if (slot < 0 || slot >= m->n_lin) return -1;
  const int64_t n = (int64_t)B * c.n_lin * c.lin_dim * c.lin_dim;
  for (int64_t i = 0; i < n; ++i) out[i] = (float)m->st[slot][i];
  return 0;
}

// Test-only loading of caches: the inverse of oracle_cache_read for sequences
// 0..B-1 (kind FULL: K then V, [B][n_kv][len][d], positions 0..len-1; kind
// LINEAR: the state [B][n_lin][dk][dv]).  No arithmetic of the method.
int32_t oracle_cache_write(void* mp, int32_t kind, int32_t slot, int32_t B, int32_t len, const float* in) {
  Model* m = (Model*)mp;
  if (!m || B <= 0 || B > m->c.max_batch) return -1;
  const oracle_config& c = m->c;
  if (kind == ORACLE_FULL) {
    if (slot < 0 || slot >= m->n_full || len < 0 || len > c.max_ctx) return -1;
    const int64_t hd = c.head_dim, L = c.max_ctx;
    int64_t o = 0;
    for (int which = 0; which < 2; ++which) {
      std::vector<float>& dst = which == 0 ? m->kc[slot] : m->vc[slot];
      for (int b = 0; b < B; ++b)
        for (int h = 0; h < c.n_kv; ++h)
          for (int p = 0; p < len; ++p)
            for (int i = 0; i < hd; ++i) dst[(((int64_t)b * c.n_kv + h) * L + p) * hd + i] = in[o++];
    }
    return 0;
  }
  if (slot < 0 || slot >= m->n_lin) return -1;
  const int64_t n = (int64_t)B * c.n_lin * c.lin_dim * c.lin_dim;
  for (int64_t i = 0; i < n; ++i) m->st[slot][i] = (double)in[i];
  return 0;
}

// Test-only: set the length of sequence b (the position its next token takes).
int32_t oracle_set_seq_len(void* mp, int32_t b, int32_t len) {
  Model* m = (Model*)mp;
  if (!m || b < 0 || b >= m->c.max_batch || len < 0 || len > m->c.max_ctx) return -1;
  m->seq_len[b] = len;
  return 0;
}

// Test-only: replace weight tensor `index` with the caller's values.
int32_t oracle_set_weight(void* mp, int32_t index, const float* in) {
  Model* m = (Model*)mp;
  if (!m || index < 0 || index >= (int)m->w.size()) return -1;
  std::memcpy(m->w[index].data(), in, sizeof(float) * m->w[index].size());
  return 0;
}

void oracle_model_destroy(void* mp) { delete (Model*)mp; }

}  // extern "C"
