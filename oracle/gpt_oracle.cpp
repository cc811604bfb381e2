// Oracle for one GPT-2-style training step -- TEST INFRASTRUCTURE ONLY.
//
// Plain single-threaded CPU loops that define what the step computes. Only the tests, the
// smoke check and the benchmark's CPU-baseline leg use it; the CUDA library never does.
// No blocking, fusion or reordering: every sum runs in index order.
//
// What each part follows (pages are cited by title and section):
//  * Model: the nanoGPT decoder (nanoGPT README, intro: "reproduces GPT-2 (124M)", can load
//    OpenAI's GPT-2 weights) with the config fields of the Panthalia "Create a Plugin" page
//    (GPTConfig: block_size, vocab_size, n_layer, n_head, n_embd, bias=False). Reading: the
//    GPT-2 pre-LayerNorm block x += Attn(LN1(x)) W_ap^T ; x += GELU(LN2(x) W_fc^T) W_mp^T,
//    learned absolute positions, tied lm_head (logits = LN_f(x) wte^T), no biases, dropout 0.
//  * LayerNorm without bias (bias=False), eps 1e-5, biased variance (reading).
//  * Causal attention with an optional left window per layer (nanochat architecture page,
//    "Modellarchitektur und FLOPs-Berechnung": (left,right) window tuple). Reading: window
//    w >= 0 admits keys j with i-w <= j <= i.
//  * GELU, tanh form (Hendrycks & Gimpel approximation).
//  * Mean softmax cross-entropy over the B*T positions (NiNo README, "Usage":
//    F.cross_entropy on the logits). Reading: padded vocab rows are outside the softmax.
//  * Global grad-norm clipping (llm.c summary, "Proceso de entrenamiento": exploding
//    gradients are tamed by clipping). Reading: coef = min(1, clip / (norm + 1e-6)).
//  * AdamW in the order the nanochat page gives (section "Optimierungsstrategien Muon und
//    AdamW", "AdamW Fused Step"): decoupled decay p *= 1 - lr*wd, m = lerp(m, g, 1-beta1),
//    bias1 = 1 - beta1^t, p -= (lr/bias1) * m / denom. The second moment and denom are not
//    printed; reading: v = beta2 v + (1-beta2) g^2, denom = sqrt(v / (1 - beta2^t)) + eps.
#include "gpt_oracle.h"

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <vector>

namespace {

struct Layout {
  size_t wte, wpe, lnf, total;
  std::vector<size_t> ln1, wqkv, wap, ln2, wfc, wmp;
};

Layout make_layout(const oracle_cfg *c) {
  Layout L;
  const size_t C = (size_t)c->n_embd, m = (size_t)c->mlp_mult;
  size_t off = 0;
  L.wte = off; off += (size_t)c->vocab_padded * C;
  L.wpe = off; off += (size_t)c->max_T * C;
  for (int l = 0; l < c->n_layer; ++l) {
    L.ln1.push_back(off); off += C;
    L.wqkv.push_back(off); off += 3 * C * C;
    L.wap.push_back(off); off += C * C;
    L.ln2.push_back(off); off += C;
    L.wfc.push_back(off); off += m * C * C;
    L.wmp.push_back(off); off += m * C * C;
  }
  L.lnf = off; off += C;
  L.total = off;
  return L;
}

int window_of(const oracle_cfg *c, int l) { return c->window_left ? c->window_left[l] : -1; }

// ---------------------------------------------------------------------------------------
// Pieces
// ---------------------------------------------------------------------------------------

// y[r][o] = sum_i x[r][i] * w[o][i]   (w row-major [out, in])
template <typename R>
void matmul_xwT(const R *x, const R *w, int rows, int in, int out, R *y) {
  for (int r = 0; r < rows; ++r)
    for (int o = 0; o < out; ++o) {
      R s = 0;
      for (int i = 0; i < in; ++i) s += x[(size_t)r * in + i] * w[(size_t)o * in + i];
      y[(size_t)r * out + o] = s;
    }
}

// Backward of y = x w^T: dx[r][i] = sum_o dy[r][o] w[o][i]; dw[o][i] += sum_r dy[r][o] x[r][i]
template <typename R>
void matmul_xwT_bwd(const R *x, const R *w, const R *dy, int rows, int in, int out, R *dx,
                    R *dw) {
  for (int r = 0; r < rows; ++r)
    for (int i = 0; i < in; ++i) {
      R s = 0;
      for (int o = 0; o < out; ++o) s += dy[(size_t)r * out + o] * w[(size_t)o * in + i];
      dx[(size_t)r * in + i] = s;
    }
  for (int o = 0; o < out; ++o)
    for (int i = 0; i < in; ++i) {
      R s = 0;
      for (int r = 0; r < rows; ++r) s += dy[(size_t)r * out + o] * x[(size_t)r * in + i];
      dw[(size_t)o * in + i] += s;
    }
}

// LayerNorm without bias: mean, biased variance, y = (x - mean) / sqrt(var + eps) * g
template <typename R>
void layernorm_fwd(const R *x, const R *g, int rows, int C, R eps, R *y, R *mean, R *rstd) {
  for (int r = 0; r < rows; ++r) {
    const R *xr = x + (size_t)r * C;
    R mu = 0;
    for (int c = 0; c < C; ++c) mu += xr[c];
    mu /= (R)C;
    R var = 0;
    for (int c = 0; c < C; ++c) var += (xr[c] - mu) * (xr[c] - mu);
    var /= (R)C;
    R rs = (R)1 / std::sqrt(var + eps);
    for (int c = 0; c < C; ++c) y[(size_t)r * C + c] = (xr[c] - mu) * rs * g[c];
    mean[r] = mu;
    rstd[r] = rs;
  }
}

// dxhat = dy*g; dx = rstd * (dxhat - mean(dxhat) - xhat * mean(dxhat*xhat)); dg += sum dy*xhat
template <typename R>
void layernorm_bwd(const R *x, const R *g, const R *mean, const R *rstd, const R *dy, int rows,
                   int C, R *dx, R *dg) {
  for (int r = 0; r < rows; ++r) {
    const R *xr = x + (size_t)r * C, *dyr = dy + (size_t)r * C;
    R a = 0, b = 0;
    for (int c = 0; c < C; ++c) {
      R xhat = (xr[c] - mean[r]) * rstd[r];
      R dxh = dyr[c] * g[c];
      a += dxh;
      b += dxh * xhat;
    }
    a /= (R)C;
    b /= (R)C;
    for (int c = 0; c < C; ++c) {
      R xhat = (xr[c] - mean[r]) * rstd[r];
      R dxh = dyr[c] * g[c];
      dx[(size_t)r * C + c] = rstd[r] * (dxh - a - xhat * b);
      dg[c] += dyr[c] * xhat;
    }
  }
}

template <typename R>
R gelu(R x) {
  const R k = (R)0.7978845608028654;  // sqrt(2/pi)
  R u = k * (x + (R)0.044715 * x * x * x);
  return (R)0.5 * x * ((R)1 + std::tanh(u));
}

template <typename R>
R gelu_grad(R x) {
  const R k = (R)0.7978845608028654;
  R u = k * (x + (R)0.044715 * x * x * x);
  R t = std::tanh(u);
  R du = k * ((R)1 + (R)3 * (R)0.044715 * x * x);
  return (R)0.5 * ((R)1 + t) + (R)0.5 * x * ((R)1 - t * t) * du;
}

bool allowed(int i, int j, int window) {
  if (j > i) return false;
  if (window >= 0 && j < i - window) return false;
  return true;
}

// Attention for all (b, h). qkv [B,T,3C]; o [B,T,C]; P [B,H,T,T] probabilities (0 where masked).
template <typename R>
void attention_fwd(const R *qkv, int B, int T, int C, int H, int window, R *o, R *P) {
  const int hd = C / H;
  const R scale = (R)1 / std::sqrt((R)hd);
  std::vector<R> s(T);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < T; ++i) {
        const R *q = qkv + ((size_t)b * T + i) * 3 * C + h * hd;
        R mx = -INFINITY;
        for (int j = 0; j < T; ++j) {
          if (!allowed(i, j, window)) continue;
          const R *k = qkv + ((size_t)b * T + j) * 3 * C + C + h * hd;
          R d = 0;
          for (int e = 0; e < hd; ++e) d += q[e] * k[e];
          s[j] = d * scale;
          if (s[j] > mx) mx = s[j];
        }
        R den = 0;
        for (int j = 0; j < T; ++j)
          if (allowed(i, j, window)) den += std::exp(s[j] - mx);
        R *Prow = P + (((size_t)b * H + h) * T + i) * T;
        for (int j = 0; j < T; ++j) Prow[j] = allowed(i, j, window) ? std::exp(s[j] - mx) / den : (R)0;
        R *orow = o + ((size_t)b * T + i) * C + h * hd;
        for (int e = 0; e < hd; ++e) {
          R acc = 0;
          for (int j = 0; j < T; ++j) {
            if (!allowed(i, j, window)) continue;
            acc += Prow[j] * qkv[((size_t)b * T + j) * 3 * C + 2 * C + h * hd + e];
          }
          orow[e] = acc;
        }
      }
}

// Softmax-attention backward with the stored probabilities P.
template <typename R>
void attention_bwd(const R *qkv, const R *P, const R *dout, int B, int T, int C, int H,
                   int window, R *dqkv) {
  const int hd = C / H;
  const R scale = (R)1 / std::sqrt((R)hd);
  std::vector<R> dP(T), dS(T);
  for (size_t i = 0; i < (size_t)B * T * 3 * C; ++i) dqkv[i] = 0;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < T; ++i) {
        const R *Prow = P + (((size_t)b * H + h) * T + i) * T;
        const R *dO = dout + ((size_t)b * T + i) * C + h * hd;
        // dP_ij = dO_i . v_j ; dV_j += P_ij dO_i
        for (int j = 0; j < T; ++j) {
          if (!allowed(i, j, window)) continue;
          const R *v = qkv + ((size_t)b * T + j) * 3 * C + 2 * C + h * hd;
          R *dv = dqkv + ((size_t)b * T + j) * 3 * C + 2 * C + h * hd;
          R d = 0;
          for (int e = 0; e < hd; ++e) d += dO[e] * v[e];
          dP[j] = d;
          for (int e = 0; e < hd; ++e) dv[e] += Prow[j] * dO[e];
        }
        // dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik)
        R rs = 0;
        for (int j = 0; j < T; ++j)
          if (allowed(i, j, window)) rs += Prow[j] * dP[j];
        for (int j = 0; j < T; ++j) dS[j] = allowed(i, j, window) ? Prow[j] * (dP[j] - rs) : (R)0;
        // dq_i = scale * sum_j dS_ij k_j ; dk_j += scale * dS_ij q_i
        const R *q = qkv + ((size_t)b * T + i) * 3 * C + h * hd;
        R *dq = dqkv + ((size_t)b * T + i) * 3 * C + h * hd;
        for (int j = 0; j < T; ++j) {
          if (!allowed(i, j, window)) continue;
          const R *k = qkv + ((size_t)b * T + j) * 3 * C + C + h * hd;
          R *dk = dqkv + ((size_t)b * T + j) * 3 * C + C + h * hd;
          for (int e = 0; e < hd; ++e) {
            dq[e] += scale * dS[j] * k[e];
            dk[e] += scale * dS[j] * q[e];
          }
        }
      }
}

// Mean cross-entropy over rows; softmax over the first V of Vp columns.
template <typename R>
R cross_entropy(const R *logits, const int *targets, int rows, int V, int Vp, R *per_row,
                R *dlogits) {
  double total = 0;
  for (int r = 0; r < rows; ++r) {
    const R *l = logits + (size_t)r * Vp;
    R mx = -INFINITY;
    for (int v = 0; v < V; ++v)
      if (l[v] > mx) mx = l[v];
    R se = 0;
    for (int v = 0; v < V; ++v) se += std::exp(l[v] - mx);
    R lse = mx + std::log(se);
    R loss = lse - l[targets[r]];
    if (per_row) per_row[r] = loss;
    total += (double)loss;
    if (dlogits) {
      R *d = dlogits + (size_t)r * Vp;
      for (int v = 0; v < Vp; ++v) {
        if (v >= V) { d[v] = 0; continue; }
        R p = std::exp(l[v] - lse);
        d[v] = (p - (v == targets[r] ? (R)1 : (R)0)) / (R)rows;
      }
    }
  }
  return (R)(total / rows);
}

// ---------------------------------------------------------------------------------------
// Whole model
// ---------------------------------------------------------------------------------------

template <typename R>
struct Acts {
  // per layer
  std::vector<std::vector<R>> x_in, a, mu1, rs1, qkv, P, o, x_mid, c, mu2, rs2, pre, h;
  std::vector<R> x_out, yf, muf, rsf, logits;
};

template <typename R>
R forward(const oracle_cfg *cf, const R *p, const int *tok, const int *tgt, int B, int T,
          R *per_token_loss, Acts<R> &A, R *dlogits) {
  const Layout L = make_layout(cf);
  const int C = cf->n_embd, H = cf->n_head, mC = cf->mlp_mult * C;
  const int M = B * T, V = cf->vocab, Vp = cf->vocab_padded;
  const R eps = (R)cf->ln_eps;
  const size_t MC = (size_t)M * C;
  std::vector<R> x(MC);
  // token + position embedding: x[b,t] = wte[tok[b,t]] + wpe[t]
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t) {
      const int id = tok[b * T + t];
      for (int e = 0; e < C; ++e)
        x[((size_t)b * T + t) * C + e] = p[L.wte + (size_t)id * C + e] + p[L.wpe + (size_t)t * C + e];
    }
  const int NL = cf->n_layer;
  A.x_in.assign(NL, {}); A.a.assign(NL, {}); A.mu1.assign(NL, {}); A.rs1.assign(NL, {});
  A.qkv.assign(NL, {}); A.P.assign(NL, {}); A.o.assign(NL, {}); A.x_mid.assign(NL, {});
  A.c.assign(NL, {}); A.mu2.assign(NL, {}); A.rs2.assign(NL, {}); A.pre.assign(NL, {});
  A.h.assign(NL, {});
  for (int l = 0; l < NL; ++l) {
    A.x_in[l] = x;
    A.a[l].resize(MC); A.mu1[l].resize(M); A.rs1[l].resize(M);
    layernorm_fwd(x.data(), p + L.ln1[l], M, C, eps, A.a[l].data(), A.mu1[l].data(), A.rs1[l].data());
    A.qkv[l].resize((size_t)M * 3 * C);
    matmul_xwT(A.a[l].data(), p + L.wqkv[l], M, C, 3 * C, A.qkv[l].data());
    A.o[l].resize(MC);
    A.P[l].resize((size_t)B * H * T * T);
    attention_fwd(A.qkv[l].data(), B, T, C, H, window_of(cf, l), A.o[l].data(), A.P[l].data());
    std::vector<R> y(MC);
    matmul_xwT(A.o[l].data(), p + L.wap[l], M, C, C, y.data());
    for (size_t i = 0; i < MC; ++i) x[i] += y[i];
    A.x_mid[l] = x;
    A.c[l].resize(MC); A.mu2[l].resize(M); A.rs2[l].resize(M);
    layernorm_fwd(x.data(), p + L.ln2[l], M, C, eps, A.c[l].data(), A.mu2[l].data(), A.rs2[l].data());
    A.pre[l].resize((size_t)M * mC);
    matmul_xwT(A.c[l].data(), p + L.wfc[l], M, C, mC, A.pre[l].data());
    A.h[l].resize((size_t)M * mC);
    for (size_t i = 0; i < (size_t)M * mC; ++i) A.h[l][i] = gelu(A.pre[l][i]);
    matmul_xwT(A.h[l].data(), p + L.wmp[l], M, mC, C, y.data());
    for (size_t i = 0; i < MC; ++i) x[i] += y[i];
  }
  A.x_out = x;
  A.yf.resize(MC); A.muf.resize(M); A.rsf.resize(M);
  layernorm_fwd(x.data(), p + L.lnf, M, C, eps, A.yf.data(), A.muf.data(), A.rsf.data());
  // tied lm_head: logits[m][v] = yf[m] . wte[v] for v < V (columns >= V are not computed)
  A.logits.assign((size_t)M * Vp, (R)0);
  for (int m = 0; m < M; ++m)
    for (int v = 0; v < V; ++v) {
      R s = 0;
      for (int e = 0; e < C; ++e) s += A.yf[(size_t)m * C + e] * p[L.wte + (size_t)v * C + e];
      A.logits[(size_t)m * Vp + v] = s;
    }
  return cross_entropy(A.logits.data(), tgt, M, V, Vp, per_token_loss, dlogits);
}

template <typename R>
void backward(const oracle_cfg *cf, const R *p, const int *tok, int B, int T, Acts<R> &A,
              const R *dlogits, R *g) {
  const Layout L = make_layout(cf);
  const int C = cf->n_embd, H = cf->n_head, mC = cf->mlp_mult * C;
  const int M = B * T, V = cf->vocab;
  const int Vp = cf->vocab_padded;
  const size_t MC = (size_t)M * C;
  for (size_t i = 0; i < L.total; ++i) g[i] = 0;
  // lm_head (tied): dyf[m] = sum_v dl[m][v] wte[v]; dwte[v] += sum_m dl[m][v] yf[m]
  std::vector<R> dyf(MC, (R)0);
  for (int m = 0; m < M; ++m)
    for (int e = 0; e < C; ++e) {
      R s = 0;
      for (int v = 0; v < V; ++v) s += dlogits[(size_t)m * Vp + v] * p[L.wte + (size_t)v * C + e];
      dyf[(size_t)m * C + e] = s;
    }
  for (int v = 0; v < V; ++v)
    for (int e = 0; e < C; ++e) {
      R s = 0;
      for (int m = 0; m < M; ++m) s += dlogits[(size_t)m * Vp + v] * A.yf[(size_t)m * C + e];
      g[L.wte + (size_t)v * C + e] += s;
    }
  std::vector<R> dx(MC);
  layernorm_bwd(A.x_out.data(), p + L.lnf, A.muf.data(), A.rsf.data(), dyf.data(), M, C,
                dx.data(), g + L.lnf);
  std::vector<R> tmp(MC), dh, dpre, dqkv, dout(MC), da(MC);
  for (int l = cf->n_layer - 1; l >= 0; --l) {
    // x_out = x_mid + h W_mp^T
    dh.assign((size_t)M * mC, (R)0);
    matmul_xwT_bwd(A.h[l].data(), p + L.wmp[l], dx.data(), M, mC, C, dh.data(), g + L.wmp[l]);
    dpre.resize((size_t)M * mC);
    for (size_t i = 0; i < (size_t)M * mC; ++i) dpre[i] = dh[i] * gelu_grad(A.pre[l][i]);
    std::vector<R> dc(MC);
    matmul_xwT_bwd(A.c[l].data(), p + L.wfc[l], dpre.data(), M, C, mC, dc.data(), g + L.wfc[l]);
    layernorm_bwd(A.x_mid[l].data(), p + L.ln2[l], A.mu2[l].data(), A.rs2[l].data(), dc.data(),
                  M, C, tmp.data(), g + L.ln2[l]);
    for (size_t i = 0; i < MC; ++i) dx[i] += tmp[i];  // dx is now dL/dx_mid
    // x_mid = x_in + o W_ap^T
    matmul_xwT_bwd(A.o[l].data(), p + L.wap[l], dx.data(), M, C, C, dout.data(), g + L.wap[l]);
    dqkv.resize((size_t)M * 3 * C);
    attention_bwd(A.qkv[l].data(), A.P[l].data(), dout.data(), B, T, C, H, window_of(cf, l),
                  dqkv.data());
    matmul_xwT_bwd(A.a[l].data(), p + L.wqkv[l], dqkv.data(), M, C, 3 * C, da.data(),
                   g + L.wqkv[l]);
    layernorm_bwd(A.x_in[l].data(), p + L.ln1[l], A.mu1[l].data(), A.rs1[l].data(), da.data(),
                  M, C, tmp.data(), g + L.ln1[l]);
    for (size_t i = 0; i < MC; ++i) dx[i] += tmp[i];  // dL/dx_in
  }
  // embedding: dwte[tok] += dx ; dwpe[t] += dx
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t) {
      const int id = tok[b * T + t];
      for (int e = 0; e < C; ++e) {
        g[L.wte + (size_t)id * C + e] += dx[((size_t)b * T + t) * C + e];
        g[L.wpe + (size_t)t * C + e] += dx[((size_t)b * T + t) * C + e];
      }
    }
}

template <typename R>
double grad_norm(size_t n, const R *g) {
  double s = 0;
  for (size_t i = 0; i < n; ++i) s += (double)g[i] * (double)g[i];
  return std::sqrt(s);
}

template <typename R>
void adamw(size_t n, R *p, const R *g, R *m, R *v, R lr, R wd, R b1, R b2, R eps, long step,
           R coef) {
  const R bias1 = (R)1 - (R)std::pow((double)b1, (double)step);
  const R bias2 = (R)1 - (R)std::pow((double)b2, (double)step);
  for (size_t i = 0; i < n; ++i) {
    R gi = coef * g[i];
    p[i] = p[i] * ((R)1 - lr * wd);                 // decoupled weight decay
    m[i] = m[i] + ((R)1 - b1) * (gi - m[i]);        // lerp toward g by (1 - beta1)
    v[i] = b2 * v[i] + ((R)1 - b2) * gi * gi;       // second moment (reading)
    R denom = std::sqrt(v[i] / bias2) + eps;        // (reading)
    p[i] = p[i] - (lr / bias1) * m[i] / denom;
  }
}

template <typename R>
R train_step(const oracle_cfg *cf, R *p, R *g, R *m, R *v, const int *tok, const int *tgt, int B,
             int T, R lr, R wd, R clip, R b1, R b2, R eps, long step, double *gnorm) {
  const Layout L = make_layout(cf);
  Acts<R> A;
  std::vector<R> dl((size_t)B * T * cf->vocab_padded);
  R loss = forward(cf, p, tok, tgt, B, T, (R *)nullptr, A, dl.data());
  backward(cf, p, tok, B, T, A, dl.data(), g);
  double n = grad_norm(L.total, g);
  if (gnorm) *gnorm = n;
  double coef = (double)clip / (n + 1e-6);
  if (coef > 1.0) coef = 1.0;
  adamw(L.total, p, g, m, v, lr, wd, b1, b2, eps, step, (R)coef);
  return loss;
}

// Gradient accumulation (llm.c summary, "Ejecución": the total batch of -d tokens is reached
// with several micro-batches per optimizer step): the loss is the mean over all
// n_micro*B*T positions, so with equal micro-batches it is the mean of the micro-batch losses
// and its gradient the mean of the micro-batch gradients; then one clip and one AdamW update.
// Micro-batch i holds tokens [i*B*T, (i+1)*B*T).
template <typename R>
R train_step_accum(const oracle_cfg *cf, R *p, R *g, R *m, R *v, const int *tok, const int *tgt,
                   int n_micro, int B, int T, R lr, R wd, R clip, R b1, R b2, R eps, long step,
                   double *gnorm) {
  const Layout L = make_layout(cf);
  std::vector<R> gi(L.total);
  std::vector<R> dl((size_t)B * T * cf->vocab_padded);
  for (size_t k = 0; k < L.total; ++k) g[k] = (R)0;
  R loss = (R)0;
  for (int i = 0; i < n_micro; ++i) {
    Acts<R> A;
    const int *ti = tok + (size_t)i * B * T, *gi_t = tgt + (size_t)i * B * T;
    loss += forward(cf, p, ti, gi_t, B, T, (R *)nullptr, A, dl.data());
    backward(cf, p, ti, B, T, A, dl.data(), gi.data());
    for (size_t k = 0; k < L.total; ++k) g[k] += gi[k];
  }
  loss /= (R)n_micro;
  for (size_t k = 0; k < L.total; ++k) g[k] /= (R)n_micro;
  double n = grad_norm(L.total, g);
  if (gnorm) *gnorm = n;
  double coef = (double)clip / (n + 1e-6);
  if (coef > 1.0) coef = 1.0;
  adamw(L.total, p, g, m, v, lr, wd, b1, b2, eps, step, (R)coef);
  return loss;
}

}  // namespace

extern "C" {

size_t oracle_num_params(const oracle_cfg *c) { return make_layout(c).total; }

int oracle_layout(const oracle_cfg *c, int64_t *offsets, int64_t *numels, int cap) {
  const Layout L = make_layout(c);
  const int64_t C = c->n_embd, mC = (int64_t)c->mlp_mult * c->n_embd;
  std::vector<std::pair<int64_t, int64_t>> t;
  t.push_back({(int64_t)L.wte, (int64_t)c->vocab_padded * C});
  t.push_back({(int64_t)L.wpe, (int64_t)c->max_T * C});
  for (int l = 0; l < c->n_layer; ++l) {
    t.push_back({(int64_t)L.ln1[l], C});
    t.push_back({(int64_t)L.wqkv[l], 3 * C * C});
    t.push_back({(int64_t)L.wap[l], C * C});
    t.push_back({(int64_t)L.ln2[l], C});
    t.push_back({(int64_t)L.wfc[l], mC * C});
    t.push_back({(int64_t)L.wmp[l], mC * C});
  }
  t.push_back({(int64_t)L.lnf, C});
  for (int i = 0; i < (int)t.size() && i < cap; ++i) {
    offsets[i] = t[i].first;
    numels[i] = t[i].second;
  }
  return (int)t.size();
}

double oracle_forward_f64(const oracle_cfg *c, const double *p, const int *tok, const int *tgt,
                          int B, int T, double *ptl) {
  Acts<double> A;
  return forward<double>(c, p, tok, tgt, B, T, ptl, A, nullptr);
}
float oracle_forward_f32(const oracle_cfg *c, const float *p, const int *tok, const int *tgt,
                         int B, int T, float *ptl) {
  Acts<float> A;
  return forward<float>(c, p, tok, tgt, B, T, ptl, A, nullptr);
}

double oracle_forward_backward_f64(const oracle_cfg *c, const double *p, const int *tok,
                                   const int *tgt, int B, int T, double *g, double *ptl) {
  Acts<double> A;
  std::vector<double> dl((size_t)B * T * c->vocab_padded);
  double loss = forward<double>(c, p, tok, tgt, B, T, ptl, A, dl.data());
  backward<double>(c, p, tok, B, T, A, dl.data(), g);
  return loss;
}
float oracle_forward_backward_f32(const oracle_cfg *c, const float *p, const int *tok,
                                  const int *tgt, int B, int T, float *g, float *ptl) {
  Acts<float> A;
  std::vector<float> dl((size_t)B * T * c->vocab_padded);
  float loss = forward<float>(c, p, tok, tgt, B, T, ptl, A, dl.data());
  backward<float>(c, p, tok, B, T, A, dl.data(), g);
  return loss;
}

double oracle_grad_norm_f64(size_t n, const double *g) { return grad_norm(n, g); }
double oracle_grad_norm_f32(size_t n, const float *g) { return grad_norm(n, g); }

void oracle_adamw_f64(size_t n, double *p, const double *g, double *m, double *v, double lr,
                      double wd, double b1, double b2, double eps, long step, double coef) {
  adamw<double>(n, p, g, m, v, lr, wd, b1, b2, eps, step, coef);
}
void oracle_adamw_f32(size_t n, float *p, const float *g, float *m, float *v, float lr, float wd,
                      float b1, float b2, float eps, long step, float coef) {
  adamw<float>(n, p, g, m, v, lr, wd, b1, b2, eps, step, coef);
}

double oracle_train_step_f64(const oracle_cfg *c, double *p, double *g, double *m, double *v,
                             const int *tok, const int *tgt, int B, int T, double lr, double wd,
                             double clip, double b1, double b2, double eps, long step,
                             double *gnorm) {
  return train_step<double>(c, p, g, m, v, tok, tgt, B, T, lr, wd, clip, b1, b2, eps, step, gnorm);
}
float oracle_train_step_f32(const oracle_cfg *c, float *p, float *g, float *m, float *v,
                            const int *tok, const int *tgt, int B, int T, float lr, float wd,
                            float clip, float b1, float b2, float eps, long step, double *gnorm) {
  return train_step<float>(c, p, g, m, v, tok, tgt, B, T, lr, wd, clip, b1, b2, eps, step, gnorm);
}

double oracle_train_step_accum_f64(const oracle_cfg *c, double *p, double *g, double *m,
                                   double *v, const int *tok, const int *tgt, int n_micro, int B,
                                   int T, double lr, double wd, double clip, double b1, double b2,
                                   double eps, long step, double *gnorm) {
  return train_step_accum<double>(c, p, g, m, v, tok, tgt, n_micro, B, T, lr, wd, clip, b1, b2,
                                  eps, step, gnorm);
}
float oracle_train_step_accum_f32(const oracle_cfg *c, float *p, float *g, float *m, float *v,
                                  const int *tok, const int *tgt, int n_micro, int B, int T,
                                  float lr, float wd, float clip, float b1, float b2, float eps,
                                  long step, double *gnorm) {
  return train_step_accum<float>(c, p, g, m, v, tok, tgt, n_micro, B, T, lr, wd, clip, b1, b2,
                                 eps, step, gnorm);
}

void oracle_layernorm_fwd_f64(const double *x, const double *g, int rows, int C, double eps,
                              double *y, double *mean, double *rstd) {
  layernorm_fwd<double>(x, g, rows, C, eps, y, mean, rstd);
}
void oracle_layernorm_bwd_f64(const double *x, const double *g, const double *mean,
                              const double *rstd, const double *dy, int rows, int C, double *dx,
                              double *dg) {
  layernorm_bwd<double>(x, g, mean, rstd, dy, rows, C, dx, dg);
}
void oracle_attention_fwd_f64(const double *qkv, int B, int T, int C, int H, int window,
                              double *o) {
  std::vector<double> P((size_t)B * H * T * T);
  attention_fwd<double>(qkv, B, T, C, H, window, o, P.data());
}
void oracle_attention_bwd_f64(const double *qkv, const double *dout, int B, int T, int C, int H,
                              int window, double *dqkv) {
  std::vector<double> P((size_t)B * H * T * T), o((size_t)B * T * C);
  attention_fwd<double>(qkv, B, T, C, H, window, o.data(), P.data());
  attention_bwd<double>(qkv, P.data(), dout, B, T, C, H, window, dqkv);
}
double oracle_gelu_f64(double x) { return gelu<double>(x); }
double oracle_gelu_grad_f64(double x) { return gelu_grad<double>(x); }
double oracle_cross_entropy_f64(const double *logits, const int *targets, int rows, int V, int Vp,
                                double *dlogits) {
  return cross_entropy<double>(logits, targets, rows, V, Vp, nullptr, dlogits);
}

}  // extern "C"
