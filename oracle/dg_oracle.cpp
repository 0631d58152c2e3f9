// Plain C++ CPU oracle of the denoising step (TEST INFRASTRUCTURE).
//
// This file is test infrastructure, not product code: only tests/,
// __graft_entry__ and the bench's CPU-baseline legs may load the library built
// from it, and it shares no code with the CUDA library.  It restates, in plain
// loops over float64 (or float32, to measure what a single-precision evaluation
// of the same definitions gives), the definitions the numpy oracle
// (dg_oracle.py) writes out, in the same order, with the same named readings
// of the pages (R-norm, R-rope, R-router, R-sample, R-keep, R-stats, R-noise,
// R-sc).  There is no blocking, fusion or reordering beyond the definitions:
// every dot product runs over its index in order, every softmax subtracts the
// row maximum first, every sum runs in index order.
//
// Sources, by tag:
//   [P1] the DiffusionGemma technical-report summary: 一 (canvas of random
//        tokens), 二 (MoE 128 experts / top-8, causal prompt + bidirectional
//        canvas, self-conditioning), 四 (the sampler), 五 (per-step cost).
//   [P2] the DiffusionGemma overview: 架构基础 (causal encoder into the KV
//        cache, bidirectional denoiser), 离散文本扩散的运作机制 (canvas init,
//        re-noising).
//   [Philox] Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3",
//        SC'11: Philox4x32 with 10 rounds.
//
// Parity pins: tests/test_oracle_cpp.py checks every exported function against
// the published Philox vectors, closed forms, brute force and the numpy oracle.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>

namespace {

// ------------------------------------------------------------------ Philox
// [Philox] Philox4x32-10: ten rounds of two 32x32 -> 64-bit products, the
// high halves xored with the other two words and the key, the key bumped by
// two Weyl constants between rounds.
void philox(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  const uint64_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    const uint64_t p0 = M0 * c0, p1 = M1 * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    const uint32_t n1 = (uint32_t)p1;
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    const uint32_t n3 = (uint32_t)p0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

// The four words of counter (position, step, block, request) under the seed.
void sampler_words(uint64_t seed, uint32_t pos, uint32_t step, uint32_t block, uint32_t req, uint32_t out[4]) {
  const uint32_t ctr[4] = {pos, step, block, req};
  const uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
  philox(ctr, key, out);
}

// R-sample: u = (w0 >> 8) * 2^-24.  R-noise: floor(w1 * V / 2^32).
double unit_uniform(uint32_t w0) { return (double)(w0 >> 8) * (1.0 / 16777216.0); }
int64_t uniform_token(uint32_t w1, uint32_t vocab) { return (int64_t)(((uint64_t)w1 * vocab) >> 32); }

// ------------------------------------------------------------------ model pieces
struct Cfg {
  int d, hq, hkv, hd, n_exp, top_k, d_ff;
  double rope_base, eps;
};

// R-norm: x * w / sqrt(mean(x^2) + eps), one row.
template <typename R>
void rms_norm_row(const R* x, const double* w, int d, double eps, R* y) {
  R ss = 0;
  for (int j = 0; j < d; ++j) ss += x[j] * x[j];
  const R inv = (R)1 / std::sqrt(ss / (R)d + (R)eps);
  for (int j = 0; j < d; ++j) y[j] = x[j] * inv * (R)w[j];
}

// y[n][m] = x[n][k] . W[m][k] (W row-major [out, in]), each dot product in order.
template <typename R>
void matmul_t(const R* x, const double* W, int n, int k, int m, R* y) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < n; ++i)
    for (int o = 0; o < m; ++o) {
      R acc = 0;
      const double* w = W + (size_t)o * k;
      const R* xi = x + (size_t)i * k;
      for (int j = 0; j < k; ++j) acc += xi[j] * (R)w[j];
      y[(size_t)i * m + o] = acc;
    }
}

// R-rope: rotate-half at integer position pos, theta_j = base^(-2j/hd).
template <typename R>
void rope_row(R* x, int hd, int64_t pos, double base) {
  const int half = hd / 2;
  for (int j = 0; j < half; ++j) {
    const double theta = std::pow(base, -2.0 * j / hd);
    const double ang = (double)pos * theta;
    const R c = (R)std::cos(ang), s = (R)std::sin(ang);
    const R x1 = x[j], x2 = x[j + half];
    x[j] = x1 * c - x2 * s;
    x[j + half] = x2 * c + x1 * s;
  }
}

template <typename R>
R silu(R x) { return x / ((R)1 + std::exp(-x)); }

// R-router selection on gate logits g[E]: top_k by logit, ties to the lower
// id (-inf last, among themselves by id); weights = softmax over the selected.
template <typename R>
void router_select_row(const R* g, int n_exp, int top_k, int64_t* ids, R* wts) {
  std::vector<int> order(n_exp);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return g[a] > g[b]; });
  for (int s = 0; s < top_k; ++s) ids[s] = order[s];
  R mx = g[order[0]];
  R sum = 0;
  std::vector<R> e(top_k);
  for (int s = 0; s < top_k; ++s) {
    e[s] = std::exp(g[ids[s]] - mx);
    sum += e[s];
  }
  for (int s = 0; s < top_k; ++s) wts[s] = e[s] / sum;
}

struct Layer {
  const double *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *router_w, *router_b, *w_gate, *w_up, *w_down;
};

// One transformer layer on n rows of h at positions pos ([P1 二], [P2 架构基础]):
// RMSNorm, Q|K|V, RoPE, attention over the cache [0, P) followed by the new rows
// (causal: new row i sees keys <= P + i; otherwise all), O + residual, RMSNorm,
// top-k mixture of SwiGLU experts + residual.  h is updated in place; the new
// rows' K and V go to k_new / v_new [Hkv][n][hd].
template <typename R>
void layer(const Cfg& c, const Layer& L, R* h, int n, const int64_t* pos, const double* kc, const double* vc,
           int P, int causal, R* k_new, R* v_new) {
  const int d = c.d, hq = c.hq, hkv = c.hkv, hd = c.hd;
  std::vector<R> x((size_t)n * d), q((size_t)n * hq * hd), k((size_t)n * hkv * hd), v((size_t)n * hkv * hd);
  for (int i = 0; i < n; ++i) rms_norm_row(h + (size_t)i * d, L.attn_norm, d, c.eps, x.data() + (size_t)i * d);
  matmul_t(x.data(), L.wq, n, d, hq * hd, q.data());
  matmul_t(x.data(), L.wk, n, d, hkv * hd, k.data());
  matmul_t(x.data(), L.wv, n, d, hkv * hd, v.data());
  for (int i = 0; i < n; ++i) {
    for (int hh = 0; hh < hq; ++hh) rope_row(q.data() + ((size_t)i * hq + hh) * hd, hd, pos[i], c.rope_base);
    for (int g = 0; g < hkv; ++g) rope_row(k.data() + ((size_t)i * hkv + g) * hd, hd, pos[i], c.rope_base);
  }
  for (int g = 0; g < hkv; ++g)
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < hd; ++j) {
        k_new[((size_t)g * n + i) * hd + j] = k[((size_t)i * hkv + g) * hd + j];
        v_new[((size_t)g * n + i) * hd + j] = v[((size_t)i * hkv + g) * hd + j];
      }
  // attention: query head hh reads KV head floor(hh * Hkv / Hq); scores / sqrt(hd)
  const int nk = P + n;
  std::vector<R> o((size_t)n * hq * hd);
  const R scale = (R)(1.0 / std::sqrt((double)hd));
#pragma omp parallel for collapse(2) schedule(static)
  for (int hh = 0; hh < hq; ++hh)
    for (int i = 0; i < n; ++i) {
      const int g = hh * hkv / hq;
      const R* qi = q.data() + ((size_t)i * hq + hh) * hd;
      std::vector<R> s(nk);
      R mx = -std::numeric_limits<R>::infinity();
      for (int t = 0; t < nk; ++t) {
        const bool vis = !causal || t <= P + i;
        if (!vis) {
          s[t] = -std::numeric_limits<R>::infinity();
          continue;
        }
        R acc = 0;
        if (t < P) {
          const double* kt = kc + ((size_t)g * P + t) * hd;
          for (int j = 0; j < hd; ++j) acc += qi[j] * (R)kt[j];
        } else {
          const R* kt = k_new + ((size_t)g * n + (t - P)) * hd;
          for (int j = 0; j < hd; ++j) acc += qi[j] * kt[j];
        }
        s[t] = acc * scale;
        mx = std::max(mx, s[t]);
      }
      R sum = 0;
      for (int t = 0; t < nk; ++t) {
        s[t] = std::isinf(s[t]) && s[t] < 0 ? (R)0 : std::exp(s[t] - mx);
        sum += s[t];
      }
      R* oi = o.data() + ((size_t)i * hq + hh) * hd;
      for (int j = 0; j < hd; ++j) oi[j] = 0;
      for (int t = 0; t < nk; ++t) {
        const R p = s[t] / sum;
        if (t < P) {
          const double* vt = vc + ((size_t)g * P + t) * hd;
          for (int j = 0; j < hd; ++j) oi[j] += p * (R)vt[j];
        } else {
          const R* vt = v_new + ((size_t)g * n + (t - P)) * hd;
          for (int j = 0; j < hd; ++j) oi[j] += p * vt[j];
        }
      }
    }
  std::vector<R> ao((size_t)n * d);
  matmul_t(o.data(), L.wo, n, hq * hd, d, ao.data());
  for (size_t z = 0; z < (size_t)n * d; ++z) h[z] += ao[z];
  // mixture of experts ([P1 二]): router on the normed rows, then each token's
  // top-k experts, added in selection order with the router weights
  for (int i = 0; i < n; ++i) rms_norm_row(h + (size_t)i * d, L.ffn_norm, d, c.eps, x.data() + (size_t)i * d);
  std::vector<R> gl((size_t)n * c.n_exp);
  matmul_t(x.data(), L.router_w, n, d, c.n_exp, gl.data());
  const int F = c.d_ff;
#pragma omp parallel for schedule(static)
  for (int i = 0; i < n; ++i) {
    R* gi = gl.data() + (size_t)i * c.n_exp;
    if (L.router_b)
      for (int e = 0; e < c.n_exp; ++e) gi[e] += (R)L.router_b[e];
    std::vector<int64_t> ids(c.top_k);
    std::vector<R> w(c.top_k), a(F), acc(d, (R)0);
    router_select_row(gi, c.n_exp, c.top_k, ids.data(), w.data());
    const R* xi = x.data() + (size_t)i * d;
    for (int s = 0; s < c.top_k; ++s) {
      const int e = (int)ids[s];
      const double* Wg = L.w_gate + (size_t)e * F * d;
      const double* Wu = L.w_up + (size_t)e * F * d;
      const double* Wd = L.w_down + (size_t)e * d * F;
      for (int f = 0; f < F; ++f) {
        R gg = 0, uu = 0;
        for (int j = 0; j < d; ++j) {
          gg += xi[j] * (R)Wg[(size_t)f * d + j];
          uu += xi[j] * (R)Wu[(size_t)f * d + j];
        }
        a[f] = silu(gg) * uu;
      }
      for (int j = 0; j < d; ++j) {
        R y = 0;
        for (int f = 0; f < F; ++f) y += a[f] * (R)Wd[(size_t)j * F + f];
        acc[j] += w[s] * y;
      }
    }
    R* hi = h + (size_t)i * d;
    for (int j = 0; j < d; ++j) hi[j] += acc[j];
  }
}

}  // namespace

extern "C" {

// Philox4x32-10 of one counter under one key.
void dgo_philox(const uint32_t* ctr, const uint32_t* key, uint32_t* out) { philox(ctr, key, out); }

// Canvas initialisation ([P1 一], [P2]): word 1 of counter (i, 0, block, req) -> a token.
void dgo_init_canvas(uint64_t seed, int n, uint32_t vocab, uint32_t block, uint32_t req, int64_t* out) {
  for (int i = 0; i < n; ++i) {
    uint32_t w[4];
    sampler_words(seed, (uint32_t)i, 0, block, req, w);
    out[i] = uniform_token(w[1], vocab);
  }
}

// One layer (see layer() above).  fp32 != 0 evaluates it in float32 (inputs
// and weights are rounded to float on use); otherwise float64.  h [n][d]
// float64 in / out; pos [n]; cache kc / vc [Hkv][P][hd] float64; k_new /
// v_new [Hkv][n][hd] float64 out.  Weights float64, [out, in].
void dgo_layer(int d, int hq, int hkv, int hd, int n_exp, int top_k, int d_ff, double rope_base, double eps,
               const double* attn_norm, const double* wq, const double* wk, const double* wv, const double* wo,
               const double* ffn_norm, const double* router_w, const double* router_b, const double* w_gate,
               const double* w_up, const double* w_down, double* h, int n, const int64_t* pos, const double* kc,
               const double* vc, int P, int causal, double* k_new, double* v_new, int fp32) {
  const Cfg c{d, hq, hkv, hd, n_exp, top_k, d_ff, rope_base, eps};
  const Layer L{attn_norm, wq, wk, wv, wo, ffn_norm, router_w, router_b, w_gate, w_up, w_down};
  if (!fp32) {
    layer<double>(c, L, h, n, pos, kc, vc, P, causal, k_new, v_new);
    return;
  }
  std::vector<float> hf((size_t)n * d), kf((size_t)hkv * n * hd), vf((size_t)hkv * n * hd);
  for (size_t z = 0; z < hf.size(); ++z) hf[z] = (float)h[z];
  layer<float>(c, L, hf.data(), n, pos, kc, vc, P, causal, kf.data(), vf.data());
  for (size_t z = 0; z < hf.size(); ++z) h[z] = hf[z];
  for (size_t z = 0; z < kf.size(); ++z) { k_new[z] = kf[z]; v_new[z] = vf[z]; }
}

// R-router on gate logits g [T][E] (bias included): ids [T][k], weights [T][k].
void dgo_router_select(const double* g, int T, int n_exp, int top_k, int64_t* ids, double* wts) {
  for (int t = 0; t < T; ++t)
    router_select_row(g + (size_t)t * n_exp, n_exp, top_k, ids + (size_t)t * top_k, wts + (size_t)t * top_k);
}

// Token embedding plus self-conditioning (R-sc): h = E[tok] + E[prev] W_sc^T
// (prev may be NULL).  h [n][d].
void dgo_embed(const double* embed, const double* w_sc, int d, const int64_t* tok, const int64_t* prev, int n,
               double* h) {
  for (int i = 0; i < n; ++i) {
    const double* e = embed + (size_t)tok[i] * d;
    for (int j = 0; j < d; ++j) h[(size_t)i * d + j] = e[j];
    if (prev) {
      const double* p = embed + (size_t)prev[i] * d;
      for (int o = 0; o < d; ++o) {
        double acc = 0;
        for (int j = 0; j < d; ++j) acc += p[j] * w_sc[(size_t)o * d + j];
        h[(size_t)i * d + o] += acc;
      }
    }
  }
}

// Final RMSNorm and the tied LM head ([P1 五]): logits [n][V] = norm(h) E^T.
void dgo_head(const double* h, const double* final_norm, const double* embed, int n, int d, int vocab, double eps,
              double* logits) {
  std::vector<double> x((size_t)n * d);
  for (int i = 0; i < n; ++i) rms_norm_row(h + (size_t)i * d, final_norm, d, eps, x.data() + (size_t)i * d);
  matmul_t(x.data(), embed, n, d, vocab, logits);
}

// The sampler for one canvas ([P1 四], R-stats / R-sample / R-keep / R-noise):
// z = s * l / T per position; pmax = 1 / sum exp(z - max z); H in nats; the
// token drawn by inverse CDF with u from word 0 of counter (i, step, block,
// req) (T == 0: the first maximum); keep the keep_k largest pmax (ties ->
// lower index); the others take the re-noise token from word 1; mean H; the
// stop flag (stop_threshold < 0 disables it).  logits [N][V] float64.
void dgo_sample_canvas(const double* logits, int N, int V, uint64_t seed, uint32_t step, uint32_t block,
                       uint32_t req, double temperature, double logit_scale, int keep_k, double stop_threshold,
                       int64_t* x_hat, double* pmax, double* ent, int32_t* keep, int64_t* x_new, double* mean_h,
                       int32_t* stop, int64_t* argmax) {
  std::vector<double> z(V);
  double hsum = 0;
  for (int i = 0; i < N; ++i) {
    const double* l = logits + (size_t)i * V;
    double mx = -std::numeric_limits<double>::infinity();
    int am = 0;
    for (int v = 0; v < V; ++v) {
      z[v] = l[v] * logit_scale;
      if (temperature != 0.0) z[v] /= temperature;
      if (z[v] > mx) { mx = z[v]; am = v; }
    }
    argmax[i] = am;
    uint32_t w[4];
    sampler_words(seed, (uint32_t)i, step, block, req, w);
    if (temperature == 0.0) {
      int cnt = 0;
      for (int v = 0; v < V; ++v) cnt += z[v] == mx;
      pmax[i] = 1.0 / cnt;
      ent[i] = std::log((double)cnt);
      x_hat[i] = am;
    } else {
      double S = 0, Sz = 0;
      for (int v = 0; v < V; ++v) {
        const double e = std::exp(z[v] - mx);
        S += e;
        Sz += e * (z[v] - mx);
      }
      pmax[i] = 1.0 / S;
      ent[i] = std::log(S) - Sz / S;
      const double target = unit_uniform(w[0]) * S;
      double c = 0;
      int64_t pick = -1, last_pos = 0;
      for (int v = 0; v < V; ++v) {
        const double e = std::exp(z[v] - mx);
        if (e > 0) last_pos = v;
        c += e;
        if (c > target) { pick = v; break; }
      }
      x_hat[i] = pick >= 0 ? pick : last_pos;
    }
    hsum += ent[i];
  }
  std::vector<int> order(N);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return pmax[a] > pmax[b]; });
  for (int i = 0; i < N; ++i) keep[i] = 0;
  for (int r = 0; r < keep_k && r < N; ++r) keep[order[r]] = 1;
  for (int i = 0; i < N; ++i) {
    uint32_t w[4];
    sampler_words(seed, (uint32_t)i, step, block, req, w);
    x_new[i] = keep[i] ? x_hat[i] : uniform_token(w[1], (uint32_t)V);
  }
  *mean_h = hsum / N;
  *stop = stop_threshold >= 0 && *mean_h < stop_threshold;
}

}  // extern "C"
