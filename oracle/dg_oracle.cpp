// dg_oracle.cpp - a plain, slow CPU implementation in C++ of one denoising
// round of the DiffusionGemma method (and of the causal context encoding it
// reads), in double precision with plain loops.  Test infrastructure only:
// the tests call it through ctypes (oracle/cpp.py) to cross-check the float64
// numpy oracle of this directory, which it shares no code with; nothing of the
// GPU library uses it, and it uses nothing of the GPU library.
//
// What the pages fix (the laozijiushiniubi.cn article "谷歌DeepMind如何将一台
// '逐字打稿机'改造成'整段喷墨机'", sections 一, 二, 四, 五): a 256-token canvas
// starts from uniformly random tokens; every position is predicted at once by
// a mixture-of-experts transformer (128 experts, 8 per token) that attends
// causally over the prompt and bidirectionally over the canvas; a
// self-conditioning input feeds back the previous round's prediction; each
// round the positions are ordered by entropy and the confident ones are kept,
// the others re-randomised to any vocabulary token; the temperature falls
// linearly from 0.8 to 0.4 over the rounds; the block stops early once the
// mean entropy is low.
//
// Readings where the pages are silent are the same as the numpy oracle's (its
// module docstrings state them): pre-norm RMSNorm (eps 1e-6, gain 1), RoPE
// (theta 1e4, rotate halves), grouped-query attention, top-k routing by router
// logit with ties to the lower expert id and the k weights renormalised,
// SwiGLU experts, untied embedding and LM head; the untempered softmax for the
// entropy and the largest probability; the Gumbel-max draw at the annealed
// temperature in float32; Philox4x32-10 draws (Salmon et al., SC'11) with the
// counter layout (c0 element, c1 position, c2 block * 256 + step, c3
// purpose << 24 | canvas); and the precision contract: bf16 at norm outputs,
// q / k (after RoPE), v, the attention output, the SwiGLU product and the
// self-conditioning input, fp32 for the residual stream, router logits and
// weights, expert outputs and LM-head logits, double in between.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

namespace {

// ---- number formats ----------------------------------------------------------------

double from_bf16(uint16_t bits) {
  const uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// nearest value with 8 significant bits (bfloat16), ties to even, taken from
// the double directly: the value is scaled so that its 8 significant bits are
// the integer part, rounded to the nearest integer (even on ties) and scaled
// back; magnitudes below the smallest normal float flush to a signed zero
double bf16(double x) {
  if (!(std::fabs(x) >= 0x1p-126)) return x * 0.0;
  const double scale = std::ldexp(1.0, std::ilogb(x) - 7);
  return std::nearbyint(x / scale) * scale;
}

double f32(double x) { return (double)(float)x; }

// ---- Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) --------------------------------

struct Draw {
  uint32_t w[4];
};

Draw philox(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0, uint32_t k1) {
  for (int round = 0; round < 10; ++round) {
    const uint64_t a = (uint64_t)0xD2511F53u * c0;
    const uint64_t b = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(b >> 32) ^ c1 ^ k0;
    const uint32_t n2 = (uint32_t)(a >> 32) ^ c3 ^ k1;
    c1 = (uint32_t)b;
    c3 = (uint32_t)a;
    c0 = n0;
    c2 = n2;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return Draw{{c0, c1, c2, c3}};
}

enum Purpose { kInit = 1, kGumbel = 2, kRenoise = 3 };

Draw method_draw(uint64_t seed, int purpose, int canvas, int block, int step, int position, uint32_t c0 = 0) {
  return philox(c0, (uint32_t)position, (uint32_t)(block * 256 + step), ((uint32_t)purpose << 24) | (uint32_t)canvas,
                (uint32_t)seed, (uint32_t)(seed >> 32));
}

// uniform token in [0, V): floor(r V / 2^32)
int64_t uniform_token(uint32_t r, int V) { return (int64_t)(((uint64_t)r * (uint64_t)V) >> 32); }

}  // namespace

extern "C" {

// model shape
struct dgo_config {
  int32_t n_layers, d_model, n_q_heads, n_kv_heads, head_dim, n_experts, top_k, d_ff, vocab, self_cond;
  double rope_theta, rms_eps;
};

// one layer's weights, bf16 bit patterns, row-major: wq [Hq hd, d], wk and wv
// [Hkv hd, d], wo [d, Hq hd], wr [E, d], wg and wu [E, d_ff, d], wd [E, d, d_ff]
struct dgo_layer {
  const uint16_t *wq, *wk, *wv, *wo, *wr, *wg, *wu, *wd;
};

// embedding and LM head [V, d], self-conditioning projection [d, d] (unused
// without self-conditioning), layers [n_layers]
struct dgo_weights {
  const uint16_t *emb, *lm, *sc;
  const dgo_layer* layers;
};

// per layer keys (after RoPE) and values [batch, c_max, Hkv, hd], float32
// holding bf16 values; `length` keys are valid
struct dgo_kv {
  float** k;
  float** v;
  int32_t batch, c_max, length;
};

}  // extern "C"

namespace {

struct Mat {
  int rows = 0, cols = 0;
  std::vector<double> a;
  const double* row(int r) const { return a.data() + (size_t)r * cols; }
};

Mat decode(const uint16_t* bits, int rows, int cols) {
  Mat m;
  m.rows = rows;
  m.cols = cols;
  m.a.resize((size_t)rows * cols);
  for (size_t i = 0; i < m.a.size(); ++i) m.a[i] = from_bf16(bits[i]);
  return m;
}

double dot(const double* x, const double* y, int n) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += x[i] * y[i];
  return s;
}

// x / sqrt(mean(x^2) + eps), gain 1, rounded to bf16
void norm_bf16(const double* x, int d, double eps, double* out) {
  double ss = 0.0;
  for (int i = 0; i < d; ++i) ss += x[i] * x[i];
  const double r = std::sqrt(ss / d + eps);
  for (int i = 0; i < d; ++i) out[i] = bf16(x[i] / r);
}

// rotary embedding of one head vector at `pos`: dims i and i + hd/2 rotated by
// pos * theta^(-2i/hd)
void rope(double* v, int hd, int pos, double theta) {
  const int half = hd / 2;
  for (int i = 0; i < half; ++i) {
    const double ang = pos * std::pow(theta, -2.0 * i / hd);
    const double c = std::cos(ang), s = std::sin(ang);
    const double a = v[i], b = v[i + half];
    v[i] = a * c - b * s;
    v[i + half] = b * c + a * s;
  }
}

// The attention half of a layer on x [B, n, d] (tokens at L0 .. L0 + n - 1):
// RMSNorm, projections, RoPE, attention over the cached keys [0, L0) plus the
// pass's own n keys (causal: a query sees keys at positions up to its own;
// otherwise every key: the article, section 二, the prompt is read causally
// and the canvas bidirectionally), output projection, residual; with
// `append` the pass's keys and values are written to the cache at [L0, L0 + n).
void attention_half(const dgo_config& c, const dgo_layer& lw, int layer, std::vector<double>& x, int B, int n,
                    dgo_kv* kv, int L0, bool causal, bool append) {
  const int d = c.d_model, hd = c.head_dim, Hq = c.n_q_heads, Hkv = c.n_kv_heads, G = Hq / Hkv;
  const Mat wq = decode(lw.wq, Hq * hd, d), wk = decode(lw.wk, Hkv * hd, d), wv = decode(lw.wv, Hkv * hd, d);
  const Mat wo = decode(lw.wo, d, Hq * hd);
  const int nk = L0 + n;
  std::vector<double> h(d), q((size_t)n * Hq * hd), k((size_t)nk * Hkv * hd), v((size_t)nk * Hkv * hd);
  std::vector<double> o(Hq * hd), s(nk), e(nk);
  for (int b = 0; b < B; ++b) {
    const size_t cache0 = ((size_t)b * kv->c_max) * Hkv * hd;
    for (int j = 0; j < L0 * Hkv * hd; ++j) {
      k[j] = kv->k[layer][cache0 + j];
      v[j] = kv->v[layer][cache0 + j];
    }
    for (int t = 0; t < n; ++t) {
      const double* xt = x.data() + ((size_t)b * n + t) * d;
      norm_bf16(xt, d, c.rms_eps, h.data());
      double* qt = q.data() + (size_t)t * Hq * hd;
      double* kt = k.data() + (size_t)(L0 + t) * Hkv * hd;
      double* vt = v.data() + (size_t)(L0 + t) * Hkv * hd;
      for (int r = 0; r < Hq * hd; ++r) qt[r] = dot(h.data(), wq.row(r), d);
      for (int r = 0; r < Hkv * hd; ++r) {
        kt[r] = dot(h.data(), wk.row(r), d);
        vt[r] = bf16(dot(h.data(), wv.row(r), d));
      }
      for (int hh = 0; hh < Hq; ++hh) rope(qt + hh * hd, hd, L0 + t, c.rope_theta);
      for (int hh = 0; hh < Hkv; ++hh) rope(kt + hh * hd, hd, L0 + t, c.rope_theta);
      for (int r = 0; r < Hq * hd; ++r) qt[r] = bf16(qt[r]);
      for (int r = 0; r < Hkv * hd; ++r) kt[r] = bf16(kt[r]);
      if (append) {
        const size_t at = ((size_t)b * kv->c_max + L0 + t) * Hkv * hd;
        for (int r = 0; r < Hkv * hd; ++r) {
          kv->k[layer][at + r] = (float)kt[r];
          kv->v[layer][at + r] = (float)vt[r];
        }
      }
    }
    const double sqrt_hd = std::sqrt((double)hd);
    for (int t = 0; t < n; ++t) {
      const int visible = causal ? L0 + t + 1 : nk;
      for (int hh = 0; hh < Hq; ++hh) {
        const int g = hh / G;
        const double* qv = q.data() + ((size_t)t * Hq + hh) * hd;
        double mx = -INFINITY;
        for (int j = 0; j < visible; ++j) {
          s[j] = dot(qv, k.data() + ((size_t)j * Hkv + g) * hd, hd) / sqrt_hd;
          mx = std::max(mx, s[j]);
        }
        double sum = 0.0;
        for (int j = 0; j < visible; ++j) sum += (e[j] = std::exp(s[j] - mx));
        double* ov = o.data() + hh * hd;
        std::fill(ov, ov + hd, 0.0);
        for (int j = 0; j < visible; ++j) {
          const double p = e[j] / sum;
          const double* vv = v.data() + ((size_t)j * Hkv + g) * hd;
          for (int i = 0; i < hd; ++i) ov[i] += p * vv[i];
        }
      }
      for (int r = 0; r < Hq * hd; ++r) o[r] = bf16(o[r]);
      double* xt = x.data() + ((size_t)b * n + t) * d;
      for (int r = 0; r < d; ++r) xt[r] = f32(xt[r] + f32(dot(o.data(), wo.row(r), Hq * hd)));
    }
  }
}

// The mixture-of-experts half (the article, section 二: 128 experts, 8 called
// per token): RMSNorm, router logits (fp32), the top-k experts by logit (ties
// to the lower id), their softmax weights renormalised
// over the k (fp32), SwiGLU experts bf16(silu(x W_g) * (x W_u)) W_d (fp32),
// the k outputs summed in slot order with their weights, residual.  The chosen
// experts go to idx [T, k] when it is given.
void moe_half(const dgo_config& c, const dgo_layer& lw, std::vector<double>& x, int T, int32_t* idx) {
  const int d = c.d_model, E = c.n_experts, K = c.top_k, F = c.d_ff;
  const Mat wr = decode(lw.wr, E, d);
  std::vector<Mat> wg(E), wu(E), wd(E);
  for (int e = 0; e < E; ++e) {
    wg[e] = decode(lw.wg + (size_t)e * F * d, F, d);
    wu[e] = decode(lw.wu + (size_t)e * F * d, F, d);
    wd[e] = decode(lw.wd + (size_t)e * d * F, d, F);
  }
  std::vector<double> h(d), logit(E), hh(F), acc(d), y(d);
  std::vector<int> order(E);
  for (int t = 0; t < T; ++t) {
    double* xt = x.data() + (size_t)t * d;
    norm_bf16(xt, d, c.rms_eps, h.data());
    for (int e = 0; e < E; ++e) logit[e] = f32(dot(h.data(), wr.row(e), d));
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return logit[a] > logit[b]; });
    double mx = -INFINITY;
    for (int j = 0; j < K; ++j) mx = std::max(mx, logit[order[j]]);
    double z = 0.0;
    for (int j = 0; j < K; ++j) z += std::exp(logit[order[j]] - mx);
    std::fill(acc.begin(), acc.end(), 0.0);
    for (int j = 0; j < K; ++j) {
      const int e = order[j];
      if (idx) idx[(size_t)t * K + j] = e;
      const double w = f32(std::exp(logit[e] - mx) / z);
      for (int f = 0; f < F; ++f) {
        const double a = dot(h.data(), wg[e].row(f), d), u = dot(h.data(), wu[e].row(f), d);
        hh[f] = bf16(a / (1.0 + std::exp(-a)) * u);
      }
      for (int r = 0; r < d; ++r) y[r] = f32(dot(hh.data(), wd[e].row(r), F));
      for (int r = 0; r < d; ++r) acc[r] += w * y[r];
    }
    for (int r = 0; r < d; ++r) xt[r] = f32(xt[r] + f32(acc[r]));
  }
}

// every layer over x [B, n, d]; route_idx (optional) gets [L, B n, k]
void forward_layers(const dgo_config& c, const dgo_weights& w, std::vector<double>& x, int B, int n, dgo_kv* kv,
                    bool causal, bool append, int32_t* route_idx) {
  const int L0 = kv->length;
  for (double& v : x) v = f32(v);
  for (int l = 0; l < c.n_layers; ++l) {
    attention_half(c, w.layers[l], l, x, B, n, kv, L0, causal, append);
    moe_half(c, w.layers[l], x, B * n, route_idx ? route_idx + (size_t)l * B * n * c.top_k : nullptr);
  }
  if (append) kv->length = L0 + n;
}

// embedding rows (bf16 values) of tokens [T]
void embed(const dgo_config& c, const dgo_weights& w, const int64_t* tokens, int T, std::vector<double>& x) {
  const int d = c.d_model;
  x.assign((size_t)T * d, 0.0);
  for (int t = 0; t < T; ++t)
    for (int i = 0; i < d; ++i) x[(size_t)t * d + i] = from_bf16(w.emb[(size_t)tokens[t] * d + i]);
}

}  // namespace

extern "C" {

// sampler settings
struct dgo_sampler {
  int32_t lock_policy;          // 0: lock where the largest probability > threshold; 1: the entropy budget
  int32_t max_steps;            // the block's round budget
  int32_t stop_require_stable;  // the stop also needs the argmax sequence unchanged from the last round
  int32_t persistent_lock;      // a locked position keeps its token for the rest of the block
  int32_t selfcond_topk;        // 0: the full expected embedding; K: over each position's K largest logits
  int32_t reserved;
  double lock_threshold, t_start, t_end, stop_entropy;
  uint64_t seed;
};

// canvas state of `batch` canvases x N positions (updated in place)
struct dgo_state {
  int64_t* tokens;       // [B, N]
  double* sc;            // [B, N, d] self-conditioning input (bf16 values), zeros before the first round
  int64_t* prev_argmax;  // [B, N]
  uint8_t* done;         // [B]
  uint8_t* locked;       // [B, N] positions committed so far (persistent lock)
};

// one round's results; any pointer may be null
struct dgo_out {
  float* logits;          // [B, N, V]
  int64_t* argmax;        // [B, N]
  int64_t* sample;        // [B, N]
  double* entropy;        // [B, N]
  double* pmax;           // [B, N]
  double* mean_entropy;   // [B]
  uint8_t* stop;          // [B]
  uint8_t* final_round;   // [B] stopped, or the last round of the budget
  uint8_t* lock;          // [B, N]
  int32_t* route_idx;     // [L, B N, k] the experts each token was sent to
};

}  // extern "C"

namespace {

// the temperature falls linearly from t_start at round 0 to t_end at the last
// round of the budget (the article, section 四)
double temperature(int step, int max_steps, double t0, double t1) {
  if (max_steps <= 1) return t0;
  return t0 + (t1 - t0) * step / (max_steps - 1);
}

// the LM head's fp32 logits [T, V] of x [T, d] after the final RMSNorm
void lm_head(const dgo_config& c, const dgo_weights& w, const std::vector<double>& x, int T, std::vector<float>& out) {
  const int d = c.d_model, V = c.vocab;
  const Mat lm = decode(w.lm, V, d);
  std::vector<double> h(d);
  out.assign((size_t)T * V, 0.f);
  for (int t = 0; t < T; ++t) {
    norm_bf16(x.data() + (size_t)t * d, d, c.rms_eps, h.data());
    for (int v = 0; v < V; ++v) out[(size_t)t * V + v] = (float)dot(h.data(), lm.row(v), d);
  }
}

}  // namespace

extern "C" {

// uniform starting tokens of B canvases (draw purpose 1, round 0)
int32_t dgo_init_canvas(uint64_t seed, int32_t block, int32_t B, int32_t N, int32_t V, int64_t* tokens) {
  if (!tokens || B < 1 || N < 1 || V < 1) return 1;
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < N; ++i) tokens[(size_t)b * N + i] = uniform_token(method_draw(seed, kInit, b, block, 0, i).w[0], V);
  return 0;
}

// causal encoding of tokens [batch, n] appended at kv->length (keys stored)
int32_t dgo_encode_context(const dgo_config* c, const dgo_weights* w, dgo_kv* kv, const int64_t* tokens, int32_t n) {
  if (!c || !w || !kv || n < 0 || kv->length + n > kv->c_max || (n > 0 && !tokens)) return 1;
  if (n == 0) return 0;
  for (size_t i = 0; i < (size_t)kv->batch * n; ++i)
    if (tokens[i] < 0 || tokens[i] >= c->vocab) return 1;
  std::vector<double> x;
  embed(*c, *w, tokens, kv->batch * n, x);
  forward_layers(*c, *w, x, kv->batch, n, kv, true, true, nullptr);
  return 0;
}

// one denoising round (a1-a9) of every canvas (the article, sections 一, 二
// and 四: every position predicted at once, the confident ones kept, the rest
// re-randomised to any token, an adaptive stop): embedding plus the
// self-conditioning input, the layers over the canvas (no mask; the canvas's
// own keys are not kept), logits and per-position entropy, largest
// probability, argmax and Gumbel-max sample, the next self-conditioning input,
// then the mean entropy, the stop flag, the lock mask and the next canvas
int32_t dgo_denoise_step(const dgo_config* cp, const dgo_weights* wp, dgo_kv* kv, int32_t N, dgo_state* st,
                         const dgo_sampler* sp, int32_t block, int32_t step, dgo_out* out) {
  if (!cp || !wp || !kv || !st || !sp || !out || N < 1 || !st->tokens || !st->prev_argmax || !st->done ||
      kv->length + N > kv->c_max || (cp->self_cond && (!st->sc || !wp->sc)) || (sp->persistent_lock && !st->locked))
    return 1;
  const dgo_config& c = *cp;
  const dgo_weights& w = *wp;
  const dgo_sampler& sc = *sp;
  const int B = kv->batch, d = c.d_model, V = c.vocab, T = B * N;
  for (int t = 0; t < T; ++t)
    if (st->tokens[t] < 0 || st->tokens[t] >= V) return 1;

  // a1: canvas embedding plus the self-conditioning input bf16(e_prev) W_sc^T
  std::vector<double> x;
  embed(c, w, st->tokens, T, x);
  if (c.self_cond) {
    const Mat wsc = decode(w.sc, d, d);
    for (int t = 0; t < T; ++t)
      for (int r = 0; r < d; ++r)
        x[(size_t)t * d + r] = f32(x[(size_t)t * d + r] + f32(dot(st->sc + (size_t)t * d, wsc.row(r), d)));
  }
  // a2-a6: the layers, bidirectional over the canvas
  forward_layers(c, w, x, B, N, kv, false, false, out->route_idx);
  // a7: logits, statistics and samples
  std::vector<float> logits;
  lm_head(c, w, x, T, logits);
  const float inv_t = (float)(1.0 / temperature(step, sc.max_steps, sc.t_start, sc.t_end));
  std::vector<double> H(T), pmax(T), e_new;
  std::vector<int64_t> amax(T), samp(T);
  const bool topk = c.self_cond && sc.selfcond_topk > 0;
  Mat emb;
  if (c.self_cond) {
    emb = decode(w.emb, V, d);
    e_new.assign((size_t)T * d, 0.0);
  }
  std::vector<double> acc(d);
  for (int t = 0; t < T; ++t) {
    const int b = t / N, i = t % N;
    const float* l = logits.data() + (size_t)t * V;
    double m = -INFINITY;
    int am = 0;
    for (int v = 0; v < V; ++v) {
      m = std::max(m, (double)l[v]);
      if (l[v] > l[am]) am = v;
    }
    double Z = 0.0;
    for (int v = 0; v < V; ++v) Z += std::exp(l[v] - m);
    double h = 0.0, pm = 0.0;
    for (int v = 0; v < V; ++v) {
      const double p = std::exp(l[v] - m) / Z;
      if (p > 0) h -= p * std::log(p);
      pm = std::max(pm, p);
    }
    H[t] = h;
    pmax[t] = pm;
    amax[t] = am;
    // the Gumbel-max draw: key_v = float32(l_v / T) + float32(-ln(-ln u_v)),
    // u_v from word v % 4 of the draw at c0 = v / 4
    float best = -INFINITY;
    int64_t arg = 0;
    for (int v0 = 0; v0 < V; v0 += 4) {
      const Draw dr = method_draw(sc.seed, kGumbel, b, block, step, i, (uint32_t)(v0 / 4));
      for (int q = 0; q < 4 && v0 + q < V; ++q) {
        const float u = ((float)(dr.w[q] >> 9) + 0.5f) * 0x1p-23f;
        const float g = -std::log(-std::log(u));
        float key = l[v0 + q] * inv_t;
        key = key + g;
        if (key > best) {
          best = key;
          arg = v0 + q;
        }
      }
    }
    samp[t] = arg;
    // a8: the next round's self-conditioning input
    if (c.self_cond && !topk) {
      // p_v = exp(bf16(l_v) - m) / Z (the logits are stored in bf16 for this use)
      std::fill(acc.begin(), acc.end(), 0.0);
      for (int v = 0; v < V; ++v) {
        const double p = bf16(std::exp(bf16(l[v]) - m) / Z);
        if (p == 0.0) continue;
        const double* er = emb.row(v);
        for (int r = 0; r < d; ++r) acc[r] += p * er[r];
      }
      for (int r = 0; r < d; ++r) e_new[(size_t)t * d + r] = bf16(acc[r]);
    } else if (topk) {
      // over the K largest bf16 logits (ties to the lower id), in id order
      const int K = std::min(sc.selfcond_topk, V);
      std::vector<int> ord(V);
      std::iota(ord.begin(), ord.end(), 0);
      std::stable_sort(ord.begin(), ord.end(), [&](int a, int b2) { return bf16(l[a]) > bf16(l[b2]); });
      std::vector<int> sel(ord.begin(), ord.begin() + K);
      std::sort(sel.begin(), sel.end());
      double M = -INFINITY, zs = 0.0;
      for (int v : sel) M = std::max(M, bf16(l[v]));
      for (int v : sel) zs += std::exp(bf16(l[v]) - M);
      std::fill(acc.begin(), acc.end(), 0.0);
      for (int v : sel) {
        const double p = bf16(std::exp(bf16(l[v]) - M) / zs);
        const double* er = emb.row(v);
        for (int r = 0; r < d; ++r) acc[r] += p * er[r];
      }
      for (int r = 0; r < d; ++r) e_new[(size_t)t * d + r] = bf16(acc[r]);
    }
  }
  // a9: mean entropy, stop, lock and the next canvas, per canvas
  for (int b = 0; b < B; ++b) {
    double hs = 0.0;
    for (int i = 0; i < N; ++i) hs += H[(size_t)b * N + i];
    const double meanH = hs / N;
    std::vector<uint8_t> lock(N, 0), committed(N, 0);
    if (sc.lock_policy == 0) {
      for (int i = 0; i < N; ++i) lock[i] = pmax[(size_t)b * N + i] > sc.lock_threshold;
    } else {
      // positions by entropy, lowest first (ties by position): as many are
      // locked, in that order, as running sums stay within the budget (the
      // article, section 四)
      std::vector<int> ord(N);
      std::iota(ord.begin(), ord.end(), 0);
      std::stable_sort(ord.begin(), ord.end(),
                       [&](int a, int b2) { return H[(size_t)b * N + a] < H[(size_t)b * N + b2]; });
      double cs = 0.0;
      int count = 0;
      for (int j = 0; j < N; ++j) {
        cs += H[(size_t)b * N + ord[j]];
        count += cs <= sc.lock_threshold;
      }
      for (int j = 0; j < count; ++j) lock[ord[j]] = 1;
    }
    if (sc.persistent_lock)
      for (int i = 0; i < N; ++i) committed[i] = st->locked[(size_t)b * N + i];
    for (int i = 0; i < N; ++i) lock[i] |= committed[i];
    uint8_t stop = 0, fin = 0;
    if (!st->done[b]) {
      stop = meanH < sc.stop_entropy;
      if (sc.stop_require_stable) {
        bool same = step > 0;
        for (int i = 0; i < N && same; ++i) same = st->prev_argmax[(size_t)b * N + i] == amax[(size_t)b * N + i];
        stop = stop && same;
      }
      fin = stop || step == sc.max_steps - 1;
      for (int i = 0; i < N; ++i) {
        int64_t& tok = st->tokens[(size_t)b * N + i];
        if (committed[i]) continue;
        if (fin)
          tok = amax[(size_t)b * N + i];
        else
          tok = lock[i] ? samp[(size_t)b * N + i]
                        : uniform_token(method_draw(sc.seed, kRenoise, b, block, step, i).w[0], V);
      }
      if (fin) st->done[b] = 1;
      for (int i = 0; i < N; ++i) st->prev_argmax[(size_t)b * N + i] = amax[(size_t)b * N + i];
      if (sc.persistent_lock)
        for (int i = 0; i < N; ++i) st->locked[(size_t)b * N + i] |= lock[i];
      if (c.self_cond)
        std::copy(e_new.begin() + (size_t)b * N * d, e_new.begin() + (size_t)(b + 1) * N * d, st->sc + (size_t)b * N * d);
    }
    if (out->mean_entropy) out->mean_entropy[b] = meanH;
    if (out->stop) out->stop[b] = stop;
    if (out->final_round) out->final_round[b] = fin;
    if (out->lock) std::copy(lock.begin(), lock.end(), out->lock + (size_t)b * N);
  }
  if (out->logits) std::copy(logits.begin(), logits.end(), out->logits);
  if (out->argmax) std::copy(amax.begin(), amax.end(), out->argmax);
  if (out->sample) std::copy(samp.begin(), samp.end(), out->sample);
  if (out->entropy) std::copy(H.begin(), H.end(), out->entropy);
  if (out->pmax) std::copy(pmax.begin(), pmax.end(), out->pmax);
  return 0;
}

}  // extern "C"

extern "C" {

// the four words of one Philox4x32-10 block (for checking the generator)
void dgo_philox(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0, uint32_t k1, uint32_t* out) {
  const Draw d = philox(c0, c1, c2, c3, k0, k1);
  for (int i = 0; i < 4; ++i) out[i] = d.w[i];
}

// the nearest bf16 value of x (for checking the rounding)
double dgo_bf16(double x) { return bf16(x); }

}  // extern "C"
