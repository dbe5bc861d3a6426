// GPT-2 training-step ORACLE — test infrastructure, not product code.
//
// A plain, slow, directly-readable CPU implementation of one GPT-2 training
// step: embedding, pre-LN blocks, final LayerNorm, tied LM head, mean
// next-token cross-entropy, the backward pass, global grad-norm clipping and
// AdamW.  Only the test suite, the smoke check and the benchmark's CPU
// baseline may load it.  It shares no code, header, table or helper with the
// CUDA library; the two meet only through seeded inputs.
//
// Every function is a template over the scalar type S and is exported twice,
// as *_f32 (S = float) and *_f64 (S = double).  Loops are the definitions
// written out (OpenMP only spreads independent rows/columns over cores; a
// `simd reduction` only lets a dot product use vector lanes).
//
// Sources (the pages describe the method; cited by page and section):
//   [LECTURE]  "Andrej Karpathy: reproducing GPT-2 from scratch" (lecture
//              summary, youtublog.net) — architecture, approximate GELU,
//              weight tying, padded vocabulary, decay groups, clipping.
//   [CH28]     "Chapter 28: data, evaluation and recovery" (book.ozine.me),
//              §28.3 (B*T+1 slicing), §28.4 (validation loss, perplexity).
//   [CS336]    "CS336 from scratch — pretraining" (fengye404.top), §1
//              training objective (cross-entropy, perplexity), §2 optimizer
//              (AdamW, learning-rate schedule, gradient clipping).
//   [ZERO]     "GPT training" (Zero framework docs, ismantic.github.io),
//              sections: autoregressive objective, Embedding, Attention,
//              Transformer Block, output layer, training loop.
//
// Readings where the pages are silent (each one is also listed in the design
// notes): LayerNorm eps is a parameter (1e-5 in every workload) with the
// biased variance; GELU is the tanh form; the causal mask excludes future
// positions; the softmax runs over every padded-vocabulary column; weight
// decay applies to 2-D tensors only; the clip scale is min(1, c/(n+1e-6)) and
// is applied to the gradient as it is read, the stored gradient is not
// rewritten.
//
// Parity is pinned (see tests/test_oracle_pins.py) by the pages' worked
// values, closed forms, invariants, PyTorch float64 library routines and
// central finite differences; no function here is "parity unpinned".

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>
#include <algorithm>
#include <omp.h>

extern "C" {
typedef struct {
  int n_layer;       // L
  int n_embd;        // C
  int n_head;        // H
  int vocab_size;    // V: ids a token or a target may take
  int padded_vocab;  // Vp >= V: rows of the token-embedding matrix
  int max_T;         // rows of the position-embedding matrix
  double ln_eps;     // LayerNorm epsilon
} oracle_cfg;
}

namespace {

enum { OK = 0, ERR_ARG = 1, ERR_TOKEN = 2, ERR_NONFINITE = 3 };

struct Tensor {
  std::string name;
  int64_t rows, cols;  // cols == 1 and ndim == 1 for vectors
  int ndim;
  int64_t offset;      // element offset in the flat parameter array
};

// Parameter order, names and shapes [LECTURE: module naming; ZERO: Embedding,
// output layer].  Linear weights are [out, in] and y = x W^T + b.  The QKV
// matrix stacks the q, k and v rows; head h owns channels [hD, (h+1)D).
std::vector<Tensor> tensor_list(const oracle_cfg& c) {
  std::vector<Tensor> t;
  int64_t off = 0;
  auto add = [&](const std::string& n, int64_t r, int64_t cl, int nd) {
    t.push_back({n, r, cl, nd, off});
    off += r * cl;
  };
  const int64_t C = c.n_embd, F = 4 * C;
  add("wte", c.padded_vocab, C, 2);
  add("wpe", c.max_T, C, 2);
  for (int l = 0; l < c.n_layer; ++l) {
    std::string p = "h." + std::to_string(l) + ".";
    add(p + "ln1.w", C, 1, 1);
    add(p + "ln1.b", C, 1, 1);
    add(p + "attn.qkv.w", 3 * C, C, 2);
    add(p + "attn.qkv.b", 3 * C, 1, 1);
    add(p + "attn.proj.w", C, C, 2);
    add(p + "attn.proj.b", C, 1, 1);
    add(p + "ln2.w", C, 1, 1);
    add(p + "ln2.b", C, 1, 1);
    add(p + "mlp.fc.w", F, C, 2);
    add(p + "mlp.fc.b", F, 1, 1);
    add(p + "mlp.proj.w", C, F, 2);
    add(p + "mlp.proj.b", C, 1, 1);
  }
  add("lnf.w", C, 1, 1);
  add("lnf.b", C, 1, 1);
  return t;
}

int64_t param_count(const oracle_cfg& c) {
  auto t = tensor_list(c);
  return t.back().offset + t.back().rows * t.back().cols;
}

bool cfg_ok(const oracle_cfg* c) {
  return c && c->n_layer >= 1 && c->n_embd >= 1 && c->n_head >= 1 &&
         c->n_embd % c->n_head == 0 && c->vocab_size >= 1 &&
         c->padded_vocab >= c->vocab_size && c->max_T >= 1 && c->ln_eps > 0;
}

// ---------------------------------------------------------------------------
// Building blocks (forward and closed-form backward)
// ---------------------------------------------------------------------------

// y = x W^T + b for x [M,K], W [N,K], b [N] (b may be null).
template <typename S>
void linear_fwd(const S* x, const S* W, const S* b, int64_t M, int64_t K, int64_t N, S* y) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    const S* xr = x + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const S* wr = W + n * K;
      S acc = 0;
#pragma omp simd reduction(+ : acc)
      for (int64_t k = 0; k < K; ++k) acc += xr[k] * wr[k];
      y[m * N + n] = acc + (b ? b[n] : S(0));
    }
  }
}

// Backward of y = x W^T + b:  dx = dy W (overwrites dx when non-null),
// dW += dy^T x, db += sum over rows of dy.
template <typename S>
void linear_bwd(const S* dy, const S* x, const S* W, int64_t M, int64_t K, int64_t N,
                S* dx, S* dW, S* db) {
  if (dx) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
      S* dxr = dx + m * K;
      for (int64_t k = 0; k < K; ++k) dxr[k] = 0;
      for (int64_t n = 0; n < N; ++n) {
        const S g = dy[m * N + n];
        const S* wr = W + n * K;
#pragma omp simd
        for (int64_t k = 0; k < K; ++k) dxr[k] += g * wr[k];
      }
    }
  }
  if (dW) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
      S* dwr = dW + n * K;
      for (int64_t m = 0; m < M; ++m) {
        const S g = dy[m * N + n];
        const S* xr = x + m * K;
#pragma omp simd
        for (int64_t k = 0; k < K; ++k) dwr[k] += g * xr[k];
      }
    }
  }
  if (db) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
      S acc = 0;
      for (int64_t m = 0; m < M; ++m) acc += dy[m * N + n];
      db[n] += acc;
    }
  }
}

// LayerNorm over the last dimension, biased variance:
// y = gamma * (x - mu) / sqrt(var + eps) + beta  [ZERO: Transformer Block, LN].
template <typename S>
void layernorm_fwd(const S* x, const S* gam, const S* bet, int64_t M, int64_t C, double eps,
                   S* y, S* mean, S* rstd) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    const S* xr = x + m * C;
    S mu = 0;
    for (int64_t c = 0; c < C; ++c) mu += xr[c];
    mu /= S(C);
    S var = 0;
    for (int64_t c = 0; c < C; ++c) {
      S d = xr[c] - mu;
      var += d * d;
    }
    var /= S(C);
    S r = S(1) / std::sqrt(var + S(eps));
    for (int64_t c = 0; c < C; ++c) y[m * C + c] = (xr[c] - mu) * r * gam[c] + bet[c];
    if (mean) mean[m] = mu;
    if (rstd) rstd[m] = r;
  }
}

// Closed-form LayerNorm backward.  With xh = (x - mu) * rstd and
// dxh = dy * gamma:  dx = rstd * (dxh - mean(dxh) - xh * mean(dxh * xh)),
// dgamma += sum_m dy * xh,  dbeta += sum_m dy.  dx is ADDED into `dx`.
template <typename S>
void layernorm_bwd(const S* dy, const S* x, const S* mean, const S* rstd, const S* gam,
                   int64_t M, int64_t C, S* dx, S* dgam, S* dbet) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    const S* xr = x + m * C;
    const S* dyr = dy + m * C;
    S a = 0, b = 0;  // mean(dxh), mean(dxh * xh)
    for (int64_t c = 0; c < C; ++c) {
      S xh = (xr[c] - mean[m]) * rstd[m];
      S dxh = dyr[c] * gam[c];
      a += dxh;
      b += dxh * xh;
    }
    a /= S(C);
    b /= S(C);
    for (int64_t c = 0; c < C; ++c) {
      S xh = (xr[c] - mean[m]) * rstd[m];
      S dxh = dyr[c] * gam[c];
      dx[m * C + c] += rstd[m] * (dxh - a - xh * b);
    }
  }
#pragma omp parallel for schedule(static)
  for (int64_t c = 0; c < C; ++c) {
    S sg = 0, sb = 0;
    for (int64_t m = 0; m < M; ++m) {
      S xh = (x[m * C + c] - mean[m]) * rstd[m];
      sg += dy[m * C + c] * xh;
      sb += dy[m * C + c];
    }
    dgam[c] += sg;
    dbet[c] += sb;
  }
}

// GPT-2's approximate GELU, the tanh form of Hendrycks & Gimpel (2016):
// g(u) = u/2 * (1 + tanh(k (u + a u^3))), k = sqrt(2/pi), a = 0.044715
// [LECTURE: feed-forward network uses GPT-2's approximate GELU; ZERO: FFN].
template <typename S>
inline S gelu_k() { return std::sqrt(S(2) / S(M_PI)); }

template <typename S>
void gelu_fwd(const S* u, int64_t n, S* g) {
  const S k = gelu_k<S>(), a = S(0.044715);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    S x = u[i];
    g[i] = S(0.5) * x * (S(1) + std::tanh(k * (x + a * x * x * x)));
  }
}

// du = dg * g'(u),  g'(u) = (1 + tau)/2 + u/2 * (1 - tau^2) * k (1 + 3 a u^2),
// tau = tanh(k (u + a u^3))  (derivative of the expression above).
template <typename S>
void gelu_bwd(const S* dg, const S* u, int64_t n, S* du) {
  const S k = gelu_k<S>(), a = S(0.044715);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    S x = u[i];
    S tau = std::tanh(k * (x + a * x * x * x));
    S d = S(0.5) * (S(1) + tau) + S(0.5) * x * (S(1) - tau * tau) * k * (S(1) + S(3) * a * x * x);
    du[i] = dg[i] * d;
  }
}

// Causal multi-head attention on a packed qkv [B, T, 3C] (q | k | v; head h
// = channels [hD, (h+1)D)): o_i = sum_{j<=i} softmax_j(q_i.k_j / sqrt(D)) v_j.
// Future positions are excluded before the softmax [ZERO: Attention;
// LECTURE: causal attention excludes future scores].  out is [B, T, C].
template <typename S>
void attention_fwd(const S* qkv, int64_t B, int64_t T, int64_t C, int64_t H, S* out) {
  const int64_t D = C / H;
  const S scale = S(1) / std::sqrt(S(D));
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < H; ++h) {
      std::vector<S> s(T);
      for (int64_t i = 0; i < T; ++i) {
        const S* q = qkv + (b * T + i) * 3 * C + h * D;
        S mx = -INFINITY;
        for (int64_t j = 0; j <= i; ++j) {
          const S* k = qkv + (b * T + j) * 3 * C + C + h * D;
          S acc = 0;
          for (int64_t d = 0; d < D; ++d) acc += q[d] * k[d];
          s[j] = acc * scale;
          mx = std::max(mx, s[j]);
        }
        S z = 0;
        for (int64_t j = 0; j <= i; ++j) {
          s[j] = std::exp(s[j] - mx);
          z += s[j];
        }
        S* o = out + (b * T + i) * C + h * D;
        for (int64_t d = 0; d < D; ++d) o[d] = 0;
        for (int64_t j = 0; j <= i; ++j) {
          const S p = s[j] / z;
          const S* v = qkv + (b * T + j) * 3 * C + 2 * C + h * D;
          for (int64_t d = 0; d < D; ++d) o[d] += p * v[d];
        }
      }
    }
}

// Closed-form attention backward (probabilities recomputed row by row):
// dv_j += p_ij do_i;  dp_ij = do_i.v_j;  ds_ij = p_ij (dp_ij - sum_k p_ik dp_ik);
// dq_i = sum_j ds_ij k_j / sqrt(D);  dk_j += ds_ij q_i / sqrt(D).
// dqkv [B, T, 3C] is overwritten.
template <typename S>
void attention_bwd(const S* dout, const S* qkv, int64_t B, int64_t T, int64_t C, int64_t H,
                   S* dqkv) {
  const int64_t D = C / H;
  const S scale = S(1) / std::sqrt(S(D));
  std::fill(dqkv, dqkv + B * T * 3 * C, S(0));
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < H; ++h) {
      std::vector<S> p(T), dp(T);
      for (int64_t i = 0; i < T; ++i) {
        const S* q = qkv + (b * T + i) * 3 * C + h * D;
        const S* go = dout + (b * T + i) * C + h * D;
        S mx = -INFINITY;
        for (int64_t j = 0; j <= i; ++j) {
          const S* k = qkv + (b * T + j) * 3 * C + C + h * D;
          S acc = 0;
          for (int64_t d = 0; d < D; ++d) acc += q[d] * k[d];
          p[j] = acc * scale;
          mx = std::max(mx, p[j]);
        }
        S z = 0;
        for (int64_t j = 0; j <= i; ++j) {
          p[j] = std::exp(p[j] - mx);
          z += p[j];
        }
        for (int64_t j = 0; j <= i; ++j) p[j] /= z;
        S pdp = 0;
        for (int64_t j = 0; j <= i; ++j) {
          const S* v = qkv + (b * T + j) * 3 * C + 2 * C + h * D;
          S acc = 0;
          for (int64_t d = 0; d < D; ++d) acc += go[d] * v[d];
          dp[j] = acc;
          pdp += p[j] * acc;
        }
        S* dq = dqkv + (b * T + i) * 3 * C + h * D;
        for (int64_t j = 0; j <= i; ++j) {
          const S ds = p[j] * (dp[j] - pdp);
          const S* k = qkv + (b * T + j) * 3 * C + C + h * D;
          S* dk = dqkv + (b * T + j) * 3 * C + C + h * D;
          S* dv = dqkv + (b * T + j) * 3 * C + 2 * C + h * D;
          for (int64_t d = 0; d < D; ++d) {
            dq[d] += ds * k[d] * scale;
            dk[d] += ds * q[d] * scale;
            dv[d] += p[j] * go[d];
          }
        }
      }
    }
}

// Cross-entropy of one row of logits z[0..V) against target y, with the row
// maximum subtracted before exponentiating [CS336 §1 "Cross-Entropy"]:
// loss = log sum_v exp(z_v - max) + max - z_y.  Returns the loss; writes the
// log-normaliser to *lse.
template <typename S>
S ce_row(const S* z, int64_t V, int64_t y, S* lse) {
  S mx = -INFINITY;
  for (int64_t v = 0; v < V; ++v) mx = std::max(mx, z[v]);
  S s = 0;
  for (int64_t v = 0; v < V; ++v) s += std::exp(z[v] - mx);
  S l = std::log(s) + mx;
  if (lse) *lse = l;
  return l - z[y];
}

// Tied LM head + mean cross-entropy over M rows [ZERO: output layer, fused
// projection + cross-entropy; LECTURE: weight tying, padded vocabulary]:
// z = h W^T over all Vp rows of W (padding rows enter the softmax), row loss
// l_m = lse_m - z_{m,y_m}, contribution `scale * l_m` to the loss.
// Backward with dz = scale * (softmax(z) - onehot(y)):  dh = dz W (overwrites
// dh), dW += dz^T h.  Processed in row chunks so only a chunk of logits is
// held.  Returns the sum of row losses in double; row losses go to row_loss.
template <typename S>
double lmhead_ce(const S* h, const S* W, const int32_t* y, int64_t M, int64_t C, int64_t Vp,
                 S scale, S* row_loss, S* dh, S* dW) {
  const int64_t CH = 64;
  std::vector<S> z(CH * Vp);
  double total = 0;
  for (int64_t m0 = 0; m0 < M; m0 += CH) {
    const int64_t mc = std::min(CH, M - m0);
    linear_fwd<S>(h + m0 * C, W, nullptr, mc, C, Vp, z.data());
    std::vector<S> lse(mc), loss(mc);
    for (int64_t r = 0; r < mc; ++r) {
      loss[r] = ce_row<S>(z.data() + r * Vp, Vp, y[m0 + r], &lse[r]);
      total += double(loss[r]);
      if (row_loss) row_loss[m0 + r] = loss[r];
    }
    if (!dh && !dW) continue;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < mc; ++r) {
      S* zr = z.data() + r * Vp;
      for (int64_t v = 0; v < Vp; ++v) zr[v] = scale * std::exp(zr[v] - lse[r]);
      zr[y[m0 + r]] -= scale;
    }
    linear_bwd<S>(z.data(), h + m0 * C, W, mc, C, Vp, dh ? dh + m0 * C : nullptr, dW, nullptr);
  }
  return total;
}

// ---------------------------------------------------------------------------
// Full model
// ---------------------------------------------------------------------------

template <typename S>
struct Layer {
  const S *ln1w, *ln1b, *qkvw, *qkvb, *projw, *projb, *ln2w, *ln2b, *fcw, *fcb, *fpw, *fpb;
};

template <typename S>
struct LayerGrad {
  S *ln1w, *ln1b, *qkvw, *qkvb, *projw, *projb, *ln2w, *ln2b, *fcw, *fcb, *fpw, *fpb;
};

template <typename P, typename S>
void bind_layers(const oracle_cfg& c, P* base, std::vector<S>& out) {
  auto t = tensor_list(c);
  out.resize(c.n_layer);
  for (int l = 0; l < c.n_layer; ++l) {
    const Tensor* q = &t[2 + 12 * l];
    out[l] = S{base + q[0].offset, base + q[1].offset, base + q[2].offset, base + q[3].offset,
               base + q[4].offset, base + q[5].offset, base + q[6].offset, base + q[7].offset,
               base + q[8].offset, base + q[9].offset, base + q[10].offset, base + q[11].offset};
  }
}

// One forward (and optionally backward) pass.
//   loss      = (1/(BT)) sum_{b,t} -log P(y_bt | x_b,<=t)   [ZERO: autoregressive
//               objective; CH28 §28.3]
//   grads    += grad_scale * dloss/dparams (when grads != null) [LECTURE:
//               gradient accumulation divides each micro-loss]
//   row_loss  = per-position loss (optional), logits (optional) [B*T, Vp].
template <typename S>
int fwd_bwd(const oracle_cfg* cp, const S* params, const int32_t* x, const int32_t* y, int64_t B,
            int64_t T, double grad_scale, double* loss_out, S* row_loss, S* grads, S* logits) {
  if (!cfg_ok(cp) || B < 1 || T < 1 || T > cp->max_T) return ERR_ARG;
  const oracle_cfg& c = *cp;
  const int64_t M = B * T, C = c.n_embd, F = 4 * C, H = c.n_head, Vp = c.padded_vocab;
  const int L = c.n_layer;
  for (int64_t m = 0; m < M; ++m)
    if (x[m] < 0 || x[m] >= c.vocab_size || y[m] < 0 || y[m] >= c.vocab_size) return ERR_TOKEN;

  auto tl = tensor_list(c);
  const S* wte = params + tl[0].offset;
  const S* wpe = params + tl[1].offset;
  const S* lnfw = params + tl[tl.size() - 2].offset;
  const S* lnfb = params + tl[tl.size() - 1].offset;
  std::vector<Layer<S>> P;
  bind_layers<const S, Layer<S>>(c, params, P);

  // Saved activations.
  std::vector<std::vector<S>> xin(L), a1(L), mu1(L), rs1(L), qkv(L), att(L), xmid(L), a2(L),
      mu2(L), rs2(L), u(L), g(L);
  std::vector<S> xfin(M * C), hf(M * C), muf(M), rsf(M);

  // Embedding: h0[b,t] = wte[x_bt] + wpe[t]; positions restart at 0 in every
  // row [ZERO: Embedding; CH28 §28.3 "each row is its own causal window"].
  std::vector<S> h(M * C);
  for (int64_t b = 0; b < B; ++b)
    for (int64_t t = 0; t < T; ++t)
      for (int64_t k = 0; k < C; ++k)
        h[(b * T + t) * C + k] = wte[int64_t(x[b * T + t]) * C + k] + wpe[t * C + k];

  // Blocks: H' = H + Attn(LN1(H)), H'' = H' + FFN(LN2(H')), FFN(x) =
  // GELU(x W1 + b1) W2 + b2 with inner width 4C [ZERO: Transformer Block].
  for (int l = 0; l < L; ++l) {
    const Layer<S>& p = P[l];
    xin[l] = h;
    a1[l].resize(M * C); mu1[l].resize(M); rs1[l].resize(M);
    layernorm_fwd<S>(h.data(), p.ln1w, p.ln1b, M, C, c.ln_eps, a1[l].data(), mu1[l].data(), rs1[l].data());
    qkv[l].resize(M * 3 * C);
    linear_fwd<S>(a1[l].data(), p.qkvw, p.qkvb, M, C, 3 * C, qkv[l].data());
    att[l].resize(M * C);
    attention_fwd<S>(qkv[l].data(), B, T, C, H, att[l].data());
    std::vector<S> tmp(M * C);
    linear_fwd<S>(att[l].data(), p.projw, p.projb, M, C, C, tmp.data());
    for (int64_t i = 0; i < M * C; ++i) h[i] += tmp[i];
    xmid[l] = h;
    a2[l].resize(M * C); mu2[l].resize(M); rs2[l].resize(M);
    layernorm_fwd<S>(h.data(), p.ln2w, p.ln2b, M, C, c.ln_eps, a2[l].data(), mu2[l].data(), rs2[l].data());
    u[l].resize(M * F);
    linear_fwd<S>(a2[l].data(), p.fcw, p.fcb, M, C, F, u[l].data());
    g[l].resize(M * F);
    gelu_fwd<S>(u[l].data(), M * F, g[l].data());
    linear_fwd<S>(g[l].data(), p.fpw, p.fpb, M, F, C, tmp.data());
    for (int64_t i = 0; i < M * C; ++i) h[i] += tmp[i];
  }
  xfin = h;
  layernorm_fwd<S>(xfin.data(), lnfw, lnfb, M, C, c.ln_eps, hf.data(), muf.data(), rsf.data());

  if (logits) linear_fwd<S>(hf.data(), wte, nullptr, M, C, Vp, logits);

  // Tied head + mean cross-entropy (forward, and backward when asked).
  const S scale = S(grad_scale / double(M));
  std::vector<S> dhf;
  S* gwte = nullptr;
  if (grads) {
    dhf.resize(M * C);
    gwte = grads + tl[0].offset;
  }
  double total = lmhead_ce<S>(hf.data(), wte, y, M, C, Vp, scale, row_loss,
                              grads ? dhf.data() : nullptr, gwte);
  if (loss_out) *loss_out = total / double(M);
  if (!grads) return OK;

  // Backward.
  std::vector<LayerGrad<S>> G;
  bind_layers<S, LayerGrad<S>>(c, grads, G);
  S* gwpe = grads + tl[1].offset;
  S* glnfw = grads + tl[tl.size() - 2].offset;
  S* glnfb = grads + tl[tl.size() - 1].offset;

  std::vector<S> dh(M * C, S(0));  // gradient of the residual stream
  layernorm_bwd<S>(dhf.data(), xfin.data(), muf.data(), rsf.data(), lnfw, M, C, dh.data(), glnfw, glnfb);
  std::vector<S> dg(M * F), du(M * F), da(M * C), datt(M * C), dqkv(M * 3 * C);
  for (int l = L - 1; l >= 0; --l) {
    const Layer<S>& p = P[l];
    const LayerGrad<S>& q = G[l];
    // h'' = h' + proj(gelu(fc(ln2(h'))))
    linear_bwd<S>(dh.data(), g[l].data(), p.fpw, M, F, C, dg.data(), q.fpw, q.fpb);
    gelu_bwd<S>(dg.data(), u[l].data(), M * F, du.data());
    linear_bwd<S>(du.data(), a2[l].data(), p.fcw, M, C, F, da.data(), q.fcw, q.fcb);
    layernorm_bwd<S>(da.data(), xmid[l].data(), mu2[l].data(), rs2[l].data(), p.ln2w, M, C,
                     dh.data(), q.ln2w, q.ln2b);
    // h' = h + proj(attn(qkv(ln1(h))))
    linear_bwd<S>(dh.data(), att[l].data(), p.projw, M, C, C, datt.data(), q.projw, q.projb);
    attention_bwd<S>(datt.data(), qkv[l].data(), B, T, C, H, dqkv.data());
    linear_bwd<S>(dqkv.data(), a1[l].data(), p.qkvw, M, C, 3 * C, da.data(), q.qkvw, q.qkvb);
    layernorm_bwd<S>(da.data(), xin[l].data(), mu1[l].data(), rs1[l].data(), p.ln1w, M, C,
                     dh.data(), q.ln1w, q.ln1b);
  }
  // Embedding backward: dwte[x_bt] += dh0[b,t] (both uses of the tied matrix
  // add into one gradient [LECTURE: weight tying]); dwpe[t] += sum_b dh0[b,t].
  for (int64_t m = 0; m < M; ++m) {
    const int64_t t = m % T;
    for (int64_t k = 0; k < C; ++k) {
      gwte[int64_t(x[m]) * C + k] += dh[m * C + k];
      gwpe[t * C + k] += dh[m * C + k];
    }
  }
  return OK;
}

// Global-norm clipping then AdamW [CS336 §2 "AdamW", "gradient clipping";
// ZERO: training loop; LECTURE: decay matrices only].
//   n  = sqrt(sum over every gradient element of g^2)
//   s  = min(1, max_norm / (n + 1e-6));  g' = s * g
//   m  = b1 m + (1 - b1) g';  v = b2 v + (1 - b2) g'^2
//   p *= 1 - lr * wd                      (2-D tensors only)
//   p -= lr * sqrt(1 - b2^t) / (1 - b1^t) * m / (sqrt(v) + eps)
// t is the 1-based step number of this update.  A non-finite n leaves every
// array untouched and returns ERR_NONFINITE.
template <typename S>
int clip_adamw(const oracle_cfg* cp, S* params, const S* grads, S* m, S* v, int t, double lr,
               double b1, double b2, double eps, double wd, double max_norm, double* norm_out) {
  if (!cfg_ok(cp) || t < 1) return ERR_ARG;
  auto tl = tensor_list(*cp);
  const int64_t N = param_count(*cp);
  // the sum of squares in a fixed order, whatever the thread count: blocks
  // of 4096 elements summed one by one, then the block sums in block order
  // (an OpenMP reduction would combine the threads' sums in arrival order)
  constexpr int64_t kBlk = 4096;
  const int64_t nblk = (N + kBlk - 1) / kBlk;
  std::vector<double> part(size_t(std::max<int64_t>(nblk, 1)), 0.0);
#pragma omp parallel for schedule(static)
  for (int64_t bI = 0; bI < nblk; ++bI) {
    double acc = 0;
    const int64_t end = std::min(N, (bI + 1) * kBlk);
    for (int64_t i = bI * kBlk; i < end; ++i) acc += double(grads[i]) * double(grads[i]);
    part[size_t(bI)] = acc;
  }
  double n2 = 0;
  for (int64_t bI = 0; bI < nblk; ++bI) n2 += part[size_t(bI)];
  const double n = std::sqrt(n2);
  if (norm_out) *norm_out = n;
  if (!std::isfinite(n)) return ERR_NONFINITE;
  const S s = S(std::min(1.0, max_norm / (n + 1e-6)));
  const S alpha = S(lr * std::sqrt(1.0 - std::pow(b2, t)) / (1.0 - std::pow(b1, t)));
  const S B1 = S(b1), B2 = S(b2), EPS = S(eps);
  for (const Tensor& te : tl) {
    const S decay = te.ndim == 2 ? S(1.0 - lr * wd) : S(1);
    const int64_t n_el = te.rows * te.cols;
#pragma omp parallel for schedule(static)
    for (int64_t i = te.offset; i < te.offset + n_el; ++i) {
      const S g = s * grads[i];
      m[i] = B1 * m[i] + (S(1) - B1) * g;
      v[i] = B2 * v[i] + (S(1) - B2) * g * g;
      params[i] *= decay;
      params[i] -= alpha * m[i] / (std::sqrt(v[i]) + EPS);
    }
  }
  return OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// C exports
// ---------------------------------------------------------------------------
extern "C" {

int oracle_num_threads(void) { return omp_get_max_threads(); }

int oracle_num_tensors(const oracle_cfg* c) {
  return cfg_ok(c) ? int(tensor_list(*c).size()) : -1;
}

// Name, shape and weight-decay flag (1 for 2-D tensors) of tensor i.
int oracle_tensor_info(const oracle_cfg* c, int i, char* name, int name_len, int64_t* rows,
                       int64_t* cols, int* ndim, int64_t* offset) {
  if (!cfg_ok(c)) return ERR_ARG;
  auto t = tensor_list(*c);
  if (i < 0 || i >= int(t.size())) return ERR_ARG;
  std::snprintf(name, size_t(name_len), "%s", t[i].name.c_str());
  *rows = t[i].rows;
  *cols = t[i].cols;
  *ndim = t[i].ndim;
  *offset = t[i].offset;
  return OK;
}

int64_t oracle_param_count(const oracle_cfg* c) { return cfg_ok(c) ? param_count(*c) : -1; }

// x = s[off : off+BT] viewed [B,T], y = s[off+1 : off+BT+1] [CH28 §28.3].
int oracle_batch_from_stream(const uint16_t* s, int64_t len, int64_t off, int B, int T,
                             int32_t* x, int32_t* y) {
  if (B < 1 || T < 1 || off < 0 || off + int64_t(B) * T + 1 > len) return ERR_ARG;
  for (int64_t i = 0; i < int64_t(B) * T; ++i) {
    x[i] = int32_t(s[off + i]);
    y[i] = int32_t(s[off + i + 1]);
  }
  return OK;
}

#define ORACLE_EXPORTS(S, SUF)                                                                  \
  int oracle_fwd_bwd_##SUF(const oracle_cfg* c, const S* params, const int32_t* x,              \
                           const int32_t* y, int B, int T, double grad_scale, double* loss,      \
                           S* row_loss, S* grads, S* logits) {                                   \
    return fwd_bwd<S>(c, params, x, y, B, T, grad_scale, loss, row_loss, grads, logits);         \
  }                                                                                              \
  int oracle_clip_adamw_##SUF(const oracle_cfg* c, S* p, const S* g, S* m, S* v, int t,          \
                              double lr, double b1, double b2, double eps, double wd,            \
                              double max_norm, double* norm) {                                   \
    return clip_adamw<S>(c, p, g, m, v, t, lr, b1, b2, eps, wd, max_norm, norm);                 \
  }                                                                                              \
  int oracle_layernorm_##SUF(const S* x, const S* g, const S* b, int64_t M, int64_t C,           \
                             double eps, S* y, S* mean, S* rstd) {                               \
    layernorm_fwd<S>(x, g, b, M, C, eps, y, mean, rstd);                                         \
    return OK;                                                                                   \
  }                                                                                              \
  int oracle_layernorm_bwd_##SUF(const S* dy, const S* x, const S* mean, const S* rstd,          \
                                 const S* g, int64_t M, int64_t C, S* dx, S* dg, S* db) {        \
    layernorm_bwd<S>(dy, x, mean, rstd, g, M, C, dx, dg, db);                                    \
    return OK;                                                                                   \
  }                                                                                              \
  int oracle_gelu_##SUF(const S* u, int64_t n, S* g) {                                           \
    gelu_fwd<S>(u, n, g);                                                                        \
    return OK;                                                                                   \
  }                                                                                              \
  int oracle_gelu_bwd_##SUF(const S* dg, const S* u, int64_t n, S* du) {                         \
    gelu_bwd<S>(dg, u, n, du);                                                                   \
    return OK;                                                                                   \
  }                                                                                              \
  int oracle_attention_##SUF(const S* qkv, int B, int T, int C, int H, S* out) {                 \
    if (C % H) return ERR_ARG;                                                                   \
    attention_fwd<S>(qkv, B, T, C, H, out);                                                      \
    return OK;                                                                                   \
  }                                                                                              \
  int oracle_attention_bwd_##SUF(const S* dout, const S* qkv, int B, int T, int C, int H,        \
                                 S* dqkv) {                                                      \
    if (C % H) return ERR_ARG;                                                                   \
    attention_bwd<S>(dout, qkv, B, T, C, H, dqkv);                                               \
    return OK;                                                                                   \
  }                                                                                              \
  int oracle_ce_##SUF(const S* z, const int32_t* y, int64_t M, int64_t V, S* row_loss,           \
                      double* mean) {                                                            \
    double tot = 0;                                                                              \
    for (int64_t m = 0; m < M; ++m) {                                                            \
      if (y[m] < 0 || y[m] >= V) return ERR_TOKEN;                                               \
      S l = ce_row<S>(z + m * V, V, y[m], nullptr);                                              \
      if (row_loss) row_loss[m] = l;                                                             \
      tot += double(l);                                                                          \
    }                                                                                            \
    if (mean) *mean = tot / double(M);                                                           \
    return OK;                                                                                   \
  }                                                                                              \
  int oracle_lmhead_ce_##SUF(const S* h, const S* W, const int32_t* y, int64_t M, int64_t C,     \
                             int64_t Vp, int64_t V, double grad_scale, double* loss,             \
                             S* row_loss, S* dh, S* dW) {                                        \
    for (int64_t m = 0; m < M; ++m)                                                              \
      if (y[m] < 0 || y[m] >= V) return ERR_TOKEN;                                               \
    double tot = lmhead_ce<S>(h, W, y, M, C, Vp, S(grad_scale / double(M)), row_loss, dh, dW);   \
    if (loss) *loss = tot / double(M);                                                           \
    return OK;                                                                                   \
  }

ORACLE_EXPORTS(float, f32)
ORACLE_EXPORTS(double, f64)

}  // extern "C"
