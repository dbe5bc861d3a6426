// C ABI of the GPT-2 training step: the handle (parameter/gradient/Adam
// arenas, activation memory, workspaces) and the orchestration of one step on
// the caller's stream.  Every step of the computation runs in this library's
// kernels; this file only sequences them.
//
// Sources: [LECTURE] "Andrej Karpathy: reproducing GPT-2 from scratch"
// (architecture, tied head, padded vocabulary, mixed precision, gradient
// accumulation); [CH28] "Chapter 28: data, evaluation and recovery" §28.3,
// §28.4; [CS336] "CS336 from scratch — pretraining" §2 (AdamW, clipping),
// §3 (non-finite guard in the training loop); [ZERO] "GPT training" (model
// sections, training loop).
//
// Memory layout (HBM)
//   - parameter arena P (fp32), gradient arena G, Adam m and v: one
//     contiguous buffer each, every tensor 64-element (256 B) aligned; all 2-D
//     tensors first (the weight-decay range [0, n_decay)), then all vectors.
//   - bf16 mirror Pb of the whole arena (bf16 mode): GEMM operands.
//   - residual stream fp32: res[0] (embedding) ... res[2L] (input of LN_f);
//     per layer saved LN outputs, qkv, attention output + row log-normalisers,
//     fc pre-activation u and GELU output g (act type: bf16 or fp32).

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <string>
#include <type_traits>
#include <vector>

#include "attn_internal.h"
#include "dp_internal.h"
#include "kernels.h"

namespace gpt2_internal {
static thread_local std::string g_err;
void set_error(const std::string& msg) { g_err = msg; }
const std::string& get_error() { return g_err; }
int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}
static thread_local int64_t g_launches = 0;
void count_launches(int n) { g_launches += n; }
int64_t launches() { return g_launches; }
}  // namespace gpt2_internal

using gpt2_internal::set_error;

namespace {

struct TensorInfo {
  std::string name;
  int ndim;
  int64_t rows, cols;
  int decay;
  int64_t off;  // element offset in the arenas
};

struct LayerOff {
  int64_t ln1w, ln1b, qkvw, qkvb, projw, projb, ln2w, ln2b, fcw, fcb, fpw, fpb;
};

constexpr int64_t kAlign = 64;  // elements (256 B of fp32)

int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

}  // namespace

struct gpt2_handle {
  gpt2_config cfg{};
  cudaStream_t st = nullptr;
  int L = 0, C = 0, H = 0, V = 0, Vp = 0, Tmax = 0, F = 0, use_bf16 = 0;
  int64_t Mcap = 0;
  std::vector<TensorInfo> tensors;
  int64_t n_arena = 0, n_decay = 0;
  int64_t off_wte = 0, off_wpe = 0, off_lnfw = 0, off_lnfb = 0;
  std::vector<LayerOff> lo;
  float *P = nullptr, *G = nullptr, *Mo = nullptr, *Vo = nullptr;
  bf16* Pb = nullptr;
  // activations
  int32_t *xbuf = nullptr, *ybuf = nullptr;
  float* gen_logits = nullptr;  // [max_B, Vp] fp32, allocated by the first generation call
  // key/value cache of incremental decoding: per layer [max_B, H, kv_T, D] (activation type),
  // allocated by the first cached generation
  void* kcache = nullptr;
  void* vcache = nullptr;
  int kv_T = 0;
  int* gen_step = nullptr;  // device step counter of a replayed decoding step
  std::vector<float*> res;
  std::vector<void*> ln1, qkv, att, ln2, u, g;
  std::vector<float*> mu1, rs1, mu2, rs2, alse;
  void* hf = nullptr;
  float *muf = nullptr, *rsf = nullptr;
  float *row_loss = nullptr, *hlse = nullptr, *d_loss = nullptr, *d_norm = nullptr;
  // backward
  float* dres = nullptr;
  void *dres_a = nullptr, *dln = nullptr, *datt = nullptr, *dqkv = nullptr, *du = nullptr,
       *dhf = nullptr;
  void* lm_ws = nullptr;
  size_t lm_ws_bytes = 0;
  float* ws = nullptr;
  size_t ws_bytes = 0;
  // side stream: weight-gradient GEMMs overlap the input-gradient GEMMs they
  // are independent of (own workspace; joined back before anything else runs)
  cudaStream_t st2 = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr, ev_join2 = nullptr;
  float* ws2 = nullptr;
  bf16* ads = nullptr;  // attention score gradients (bf16 tcgen05 path), one layer at a time
  // per-block column sums of dqkv left by those kernels, one buffer per layer
  float* qkvb_parts = nullptr;
  size_t qkvb_stride = 0;  // floats per layer
  // partial sums of the vector gradients (LayerNorm gamma / beta, biases), one
  // buffer per producer, summed in one launch at the end of the backward
  float* ln_parts = nullptr;  // 2L + 1 LayerNorm backwards
  size_t ln_stride = 0;       // floats per LayerNorm
  float* cs_parts = nullptr;  // per layer: fc bias, then qkv bias (when not from attention)
  size_t cs_stride = 0, cs_qkv_off = 0;
  std::vector<RowSum> defer;
  void* ws_emb = nullptr;
  double* ws_norm = nullptr;
  DevStatus* status = nullptr;
  // training from a device token stream, one optimizer step recorded as a CUDA graph
  int64_t* d_cursor = nullptr;  // offset of the next window in the stream
  float* d_lr = nullptr;        // learning rate read by the optimizer kernel of the graph
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t graph_exec = nullptr;
  // state
  bool fwd_saved = false;
  int fB = 0, fT = 0;
  bool grads_zero = true;
  bool mirror_dirty = true;
  std::string err;
  std::vector<void*> allocs;
  // profiler
  struct Cat {
    int64_t launches = 0;
    double flops = 0, bytes = 0, ms = 0;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending;
  };
  bool prof_on = false;
  // data-parallel exchange: called as each gradient bucket becomes final in a
  // backward issued call by call (never while a step is being captured)
  gpt2_bucket_fn bucket_fn = nullptr;
  void* bucket_user = nullptr;
  bool capturing = false;
  // in-library exchange (gpt2_dp_init): NCCL communicator, communication
  // stream, the ranges of each bucket, whether the next backward exchanges
  void* dp_comm = nullptr;
  int dp_world = 1;
  bool dp_sync = true;
  bool dp_pending = false;  // this backward has enqueued exchanges to join
  cudaStream_t st_comm = nullptr;
  cudaEvent_t ev_dp = nullptr, ev_dp_join = nullptr;
  std::vector<std::vector<std::pair<int64_t, int64_t>>> dp_ranges;
  Cat cats[GPT2_PROF_NCAT];
  std::vector<cudaEvent_t> ev_pool;
  int64_t launches_total = 0;
  int64_t graph_kernels = 0;  // kernel launches recorded into the step graph

  size_t act_size() const { return use_bf16 ? 2 : 4; }
};

namespace {

int fail(gpt2_handle* h, int code, const std::string& msg) {
  if (h) h->err = msg;
  set_error(msg);
  return code;
}

#define H_CUDA(h, expr)                                                              \
  do {                                                                               \
    cudaError_t e_ = (expr);                                                         \
    if (e_ != cudaSuccess) return fail(h, GPT2_ERR_CUDA, std::string(#expr) + ": " + \
                                                             cudaGetErrorString(e_)); \
  } while (0)

#define H_TRY(h, expr)                                                \
  do {                                                                \
    int rc_ = (expr);                                                 \
    if (rc_ != GPT2_OK) {                                             \
      if (h) h->err = gpt2_internal::get_error();                     \
      return rc_;                                                     \
    }                                                                 \
  } while (0)

cudaEvent_t take_event(gpt2_handle* h) {
  if (!h->ev_pool.empty()) {
    cudaEvent_t e = h->ev_pool.back();
    h->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Brackets one kernel group: counts its launches and, when profiling is on,
// records CUDA events around it on the handle's stream.
struct ProfScope {
  gpt2_handle* h;
  int cat;
  int64_t l0;
  cudaEvent_t e0 = nullptr;
  ProfScope(gpt2_handle* hh, int c, double flops, double bytes)
      : h(hh), cat(c), l0(gpt2_internal::launches()) {
    h->cats[cat].flops += flops;
    h->cats[cat].bytes += bytes;
    if (h->prof_on) {
      e0 = take_event(h);
      cudaEventRecord(e0, h->st);
    }
  }
  ~ProfScope() {
    const int64_t n = gpt2_internal::launches() - l0;
    h->cats[cat].launches += n;
    h->launches_total += n;
    if (e0) {
      cudaEvent_t e1 = take_event(h);
      cudaEventRecord(e1, h->st);
      h->cats[cat].pending.push_back({e0, e1});
    }
  }
};

int prof_collect(gpt2_handle* h) {
  bool any = false;
  for (auto& c : h->cats) any |= !c.pending.empty();
  if (!any) return GPT2_OK;
  H_CUDA(h, cudaStreamSynchronize(h->st));
  for (auto& c : h->cats) {
    for (auto& pr : c.pending) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, pr.first, pr.second);
      c.ms += ms;
      h->ev_pool.push_back(pr.first);
      h->ev_pool.push_back(pr.second);
    }
    c.pending.clear();
  }
  return GPT2_OK;
}

void* dev_alloc(gpt2_handle* h, size_t bytes) {
  bytes = std::max<size_t>(256, (bytes + 255) / 256 * 256);
  void* p = nullptr;
  if (h->cfg.alloc) {
    p = h->cfg.alloc(bytes, h->cfg.alloc_ctx);
  } else if (cudaMalloc(&p, bytes) != cudaSuccess) {
    cudaGetLastError();
    p = nullptr;
  }
  if (p) h->allocs.push_back(p);
  return p;
}

void free_all(gpt2_handle* h) {
  for (void* p : h->allocs) {
    if (h->cfg.alloc)
      h->cfg.free(p, h->cfg.alloc_ctx);
    else
      cudaFree(p);
  }
  h->allocs.clear();
}

// Empty string when cfg is a valid configuration, else why not.
std::string config_problem(const gpt2_config& c) {
  if (c.n_layer < 1 || c.n_embd < 8 || c.n_head < 1 || c.n_embd % c.n_head || c.n_embd % 8 ||
      c.vocab_size < 1 || c.padded_vocab < c.vocab_size || c.padded_vocab % 8 || c.max_T < 1 ||
      c.max_B < 1 || c.max_Tseq < 1 || c.max_Tseq > c.max_T || !(c.ln_eps > 0.f) ||
      c.n_embd > 1024 || c.resid_init_scale != 0 || (c.alloc && !c.free))
    return "invalid gpt2_config";
  const int D = c.n_embd / c.n_head;
  if (D != 16 && D != 32 && D != 64) return "head size must be 16, 32 or 64";
  if (int64_t(c.max_B) * c.max_Tseq > (int64_t(1) << 26)) return "max_B * max_Tseq too large";
  return "";
}

void set_shape(gpt2_handle* h, const gpt2_config& c) {
  h->cfg = c;
  h->L = c.n_layer;
  h->C = c.n_embd;
  h->H = c.n_head;
  h->V = c.vocab_size;
  h->Vp = c.padded_vocab;
  h->Tmax = c.max_T;
  h->F = 4 * c.n_embd;
  h->use_bf16 = c.bf16 ? 1 : 0;
  h->Mcap = int64_t(c.max_B) * c.max_Tseq;
}

void build_layout(gpt2_handle* h) {
  const int64_t C = h->C, F = h->F;
  std::vector<TensorInfo>& t = h->tensors;
  auto add = [&](const std::string& n, int64_t r, int64_t c, int nd) {
    t.push_back({n, nd, r, c, nd == 2 ? 1 : 0, 0});
  };
  add("wte", h->Vp, C, 2);
  add("wpe", h->Tmax, C, 2);
  for (int l = 0; l < h->L; ++l) {
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
  // arena: 2-D tensors first, then vectors, each aligned
  int64_t off = 0;
  for (auto& x : t)
    if (x.ndim == 2) {
      x.off = off;
      off += align_up(x.rows * x.cols, kAlign);
    }
  h->n_decay = off;
  for (auto& x : t)
    if (x.ndim == 1) {
      x.off = off;
      off += align_up(x.rows, kAlign);
    }
  h->n_arena = off;
  h->off_wte = t[0].off;
  h->off_wpe = t[1].off;
  h->off_lnfw = t[t.size() - 2].off;
  h->off_lnfb = t[t.size() - 1].off;
  h->lo.resize(h->L);
  for (int l = 0; l < h->L; ++l) {
    const TensorInfo* q = &t[2 + 12 * l];
    h->lo[l] = {q[0].off, q[1].off, q[2].off, q[3].off, q[4].off,  q[5].off,
                q[6].off, q[7].off, q[8].off, q[9].off, q[10].off, q[11].off};
  }
}

// weight pointer in the GEMM operand type
const void* wptr(const gpt2_handle* h, int64_t off) {
  return h->use_bf16 ? static_cast<const void*>(h->Pb + off) : static_cast<const void*>(h->P + off);
}

void* aoff(void* base, int64_t elems, size_t esz) {
  return static_cast<char*>(base) + elems * int64_t(esz);
}

int gemm(gpt2_handle* h, const void* A, int ak, int64_t lda, const void* B, int bk, int64_t ldb,
         int M, int N, int K, const EpiParams& ep, cudaStream_t st = nullptr,
         float* ws = nullptr) {
  GemmArgs g{A, ak, lda, B, bk, ldb, h->use_bf16, M, N, K, ep, ws ? ws : h->ws, h->ws_bytes};
  g.ep.out_bf16 = (ep.kind == EPI_ACC || ep.kind == EPI_RESID) ? 0 : ep.out_bf16;
  H_TRY(h, gemm_launch(g, st ? st : h->st));
  return GPT2_OK;
}

// Fork / join of the side stream (recorded as parallel branches when the step
// is captured).  While the profiler is on, side work runs on the main stream
// so that every kernel group is timed on its own.
struct Side {
  gpt2_handle* h;
  bool on;
  cudaStream_t st() const { return on ? h->st2 : h->st; }
  float* ws() const { return on ? h->ws2 : h->ws; }
  int fork() {
    if (on) {
      H_CUDA(h, cudaEventRecord(h->ev_fork, h->st));
      H_CUDA(h, cudaStreamWaitEvent(h->st2, h->ev_fork, 0));
    }
    return GPT2_OK;
  }
  int join() {
    if (on) {
      H_CUDA(h, cudaEventRecord(h->ev_join, h->st2));
      H_CUDA(h, cudaStreamWaitEvent(h->st, h->ev_join, 0));
    }
    return GPT2_OK;
  }
};

EpiParams epi(int kind, void* out, int64_t ldo, int out_bf16) {
  EpiParams e;
  e.kind = kind;
  e.out = out;
  e.ldo = ldo;
  e.out_bf16 = out_bf16;
  return e;
}

int check_status(gpt2_handle* h) {
  DevStatus s;
  H_CUDA(h, cudaMemcpyAsync(&s, h->status, sizeof(s), cudaMemcpyDeviceToHost, h->st));
  H_CUDA(h, cudaStreamSynchronize(h->st));
  int* ew = device_error_word();
  int dev_err = 0;
  H_CUDA(h, cudaMemcpy(&dev_err, ew, sizeof(int), cudaMemcpyDeviceToHost));
  if (s.timeout || dev_err) {
    int z = 0;
    cudaMemcpy(ew, &z, sizeof(int), cudaMemcpyHostToDevice);
    DevStatus c = s;
    c.timeout = 0;
    cudaMemcpy(h->status, &c, sizeof(c), cudaMemcpyHostToDevice);
    return fail(h, GPT2_ERR_TIMEOUT, "a bounded device wait gave up (kernel timeout)");
  }
  if (s.window_bad) {
    DevStatus c = s;
    c.window_bad = 0;
    H_CUDA(h, cudaMemcpy(h->status, &c, sizeof(c), cudaMemcpyHostToDevice));
    h->fwd_saved = false;
    return fail(h, GPT2_ERR_ARG, "a batch window at the stream cursor ran past the stream "
                                 "(that step's update was skipped)");
  }
  if (s.token_bad) {
    DevStatus c = s;
    c.token_bad = 0;
    H_CUDA(h, cudaMemcpy(h->status, &c, sizeof(c), cudaMemcpyHostToDevice));
    h->fwd_saved = false;
    return fail(h, GPT2_ERR_TOKEN, "a token or target id is outside [0, vocab_size)");
  }
  if (s.nonfinite) {
    DevStatus c = s;
    c.nonfinite = 0;
    H_CUDA(h, cudaMemcpy(h->status, &c, sizeof(c), cudaMemcpyHostToDevice));
    return fail(h, GPT2_ERR_NONFINITE, "non-finite gradient norm: the update was skipped");
  }
  return GPT2_OK;
}

int refresh_mirror(gpt2_handle* h) {
  if (h->use_bf16 && h->mirror_dirty) H_TRY(h, launch_to_bf16(h->P, h->Pb, h->n_arena, h->st));
  h->mirror_dirty = false;
  return GPT2_OK;
}

int stage_tokens(gpt2_handle* h, const int32_t* x, const int32_t* y, int64_t M, int on_device) {
  const cudaMemcpyKind k = on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  H_CUDA(h, cudaMemcpyAsync(h->xbuf, x, M * sizeof(int32_t), k, h->st));
  H_CUDA(h, cudaMemcpyAsync(h->ybuf, y, M * sizeof(int32_t), k, h->st));
  return GPT2_OK;
}

// ------------------------------------------------------------------ forward
// Pre-LN block [ZERO: Transformer Block]: H' = H + Attn(LN1(H)),
// H'' = H' + FFN(LN2(H')), FFN(x) = GELU(x W1 + b1) W2 + b2; then LN_f and the
// tied head with mean cross-entropy [ZERO: output layer; LECTURE: tying].
#define PROF(cat, flops, bytes) ProfScope ps_##__LINE__(h, cat, double(flops), double(bytes))

double gemm_flops(int64_t M, int64_t N, int64_t K) { return 2.0 * double(M) * double(N) * double(K); }

// With d_logits the step ends after the final LayerNorm with the tied head
// applied to the last position of each sequence only (fp32 [B, ld_logits]).
// With kv the tokens sit at positions kv->pos0 .. pos0 + T - 1, each layer's
// keys and values are stored into the cache there, and (kv->decode, T = 1)
// attention reads the cache positions 0 .. pos0 instead of the batch.
struct KvStep {
  int pos0;
  bool decode;
  const int* d_step = nullptr;  // device offset added to pos0 (a replayed decoding step)
};
template <typename A>
int forward_t(gpt2_handle* h, int B, int T, float* d_row_loss, bool save,
              float* d_logits = nullptr, int64_t ld_logits = 0, const KvStep* kv = nullptr) {
  const int64_t M = int64_t(B) * T;
  const int C = h->C, F = h->F, Vp = h->Vp, Hh = h->H;
  const int ab = h->use_bf16;
  const double a = double(sizeof(A));
  const float* P = h->P;
  {
    PROF(GPT2_PROF_OTHER, 0, h->use_bf16 && h->mirror_dirty ? 6.0 * h->n_arena : 0);
    H_TRY(h, refresh_mirror(h));
  }
  {
    PROF(GPT2_PROF_EMBED, 0, 12.0 * M * C);
    H_TRY(h, launch_embed_fwd(h->xbuf, h->ybuf, P + h->off_wte, P + h->off_wpe, B, T, C, h->V,
                              h->res[0], h->status, h->st, kv ? kv->pos0 : 0,
                              kv ? kv->d_step : nullptr));
  }
  const double ln_bytes = M * C * (4.0 + a) + 8.0 * M;
  const double attn_flops = 2.0 * B * Hh * double(T) * T * (C / Hh);
  for (int l = 0; l < h->L; ++l) {
    const LayerOff& o = h->lo[l];
    A* ln1 = static_cast<A*>(h->ln1[l]);
    A* qkv = static_cast<A*>(h->qkv[l]);
    A* att = static_cast<A*>(h->att[l]);
    A* ln2 = static_cast<A*>(h->ln2[l]);
    {
      PROF(GPT2_PROF_LN_FWD, 0, ln_bytes);
      H_TRY(h, launch_layernorm_fwd<A>(h->res[2 * l], P + o.ln1w, P + o.ln1b, ln1, h->mu1[l],
                                       h->rs1[l], M, C, h->cfg.ln_eps, h->st));
    }
    {
      PROF(GPT2_PROF_GEMM, gemm_flops(M, 3 * C, C), a * (M * C + 3.0 * C * C + 3.0 * M * C));
      EpiParams e = epi(EPI_STORE, qkv, 3 * C, ab);
      e.bias = P + o.qkvb;
      H_TRY(h, gemm(h, ln1, 1, C, wptr(h, o.qkvw), 1, C, int(M), 3 * C, C, e));
    }
    if (kv) {
      const size_t per_layer = size_t(h->cfg.max_B) * Hh * h->kv_T * (C / Hh);
      A* kc = static_cast<A*>(h->kcache) + l * per_layer;
      A* vc = static_cast<A*>(h->vcache) + l * per_layer;
      PROF(GPT2_PROF_ATTN_FWD, 0, a * 4.0 * M * C);
      H_TRY(h, launch_kv_store<A>(qkv, B, T, C, Hh, kv->pos0, h->kv_T, kc, vc, h->st, kv->d_step));
      if (kv->decode)
        H_TRY(h, launch_attn_decode<A>(qkv, kc, vc, B, C, Hh, h->kv_T, kv->pos0 + 1, att, h->st,
                                       kv->d_step));
    }
    if (!kv || !kv->decode) {
      PROF(GPT2_PROF_ATTN_FWD, attn_flops, a * 4.0 * M * C + 4.0 * M * Hh);
      H_TRY(h, launch_attn_fwd<A>(qkv, B, T, C, Hh, att, h->alse[l], h->st));
    }
    {
      PROF(GPT2_PROF_GEMM, gemm_flops(M, C, C), a * (M * C + 1.0 * C * C) + 8.0 * M * C);
      EpiParams e = epi(EPI_RESID, nullptr, C, 0);
      e.rin = h->res[2 * l];
      e.rout = h->res[2 * l + 1];
      e.bias = P + o.projb;
      H_TRY(h, gemm(h, att, 1, C, wptr(h, o.projw), 1, C, int(M), C, C, e));
    }
    {
      PROF(GPT2_PROF_LN_FWD, 0, ln_bytes);
      H_TRY(h, launch_layernorm_fwd<A>(h->res[2 * l + 1], P + o.ln2w, P + o.ln2b, ln2, h->mu2[l],
                                       h->rs2[l], M, C, h->cfg.ln_eps, h->st));
    }
    {
      PROF(GPT2_PROF_GEMM, gemm_flops(M, F, C), a * (M * C + 1.0 * F * C + 2.0 * M * F));
      EpiParams e = epi(EPI_GELU, h->u[l], F, ab);
      e.out2 = h->g[l];
      e.bias = P + o.fcb;
      H_TRY(h, gemm(h, ln2, 1, C, wptr(h, o.fcw), 1, C, int(M), F, C, e));
    }
    {
      PROF(GPT2_PROF_GEMM, gemm_flops(M, C, F), a * (M * F + 1.0 * F * C) + 8.0 * M * C);
      EpiParams e = epi(EPI_RESID, nullptr, C, 0);
      e.rin = h->res[2 * l + 1];
      e.rout = h->res[2 * l + 2];
      e.bias = P + o.fpb;
      H_TRY(h, gemm(h, h->g[l], 1, F, wptr(h, o.fpw), 1, F, int(M), C, F, e));
    }
  }
  A* hf = static_cast<A*>(h->hf);
  {
    PROF(GPT2_PROF_LN_FWD, 0, ln_bytes);
    H_TRY(h, launch_layernorm_fwd<A>(h->res[2 * h->L], P + h->off_lnfw, P + h->off_lnfb, hf,
                                     h->muf, h->rsf, M, C, h->cfg.ln_eps, h->st));
  }
  if (d_logits) {
    // rows T-1, 2T-1, ...: the last position of each sequence (row stride T*C)
    PROF(GPT2_PROF_LMHEAD, gemm_flops(B, Vp, C), a * (double(B) * C + double(Vp) * C) + 4.0 * B * Vp);
    EpiParams e = epi(EPI_STORE, d_logits, ld_logits, 0);
    H_TRY(h, gemm(h, hf + int64_t(T - 1) * C, 1, int64_t(T) * C, wptr(h, h->off_wte), 1, C, B, Vp,
                  C, e));
    h->fwd_saved = false;
    h->fB = B;
    h->fT = T;
    return GPT2_OK;
  }
  {
    // tied head + cross-entropy: no logits are stored (see lmhead_fwd)
    PROF(GPT2_PROF_LMHEAD, gemm_flops(M, Vp, C), a * (M * C + double(Vp) * C) + 8.0 * M);
    H_TRY(h, lmhead_fwd(hf, wptr(h, h->off_wte), h->ybuf, int(M), C, Vp, h->use_bf16, h->hlse,
                        h->row_loss, h->lm_ws, h->lm_ws_bytes, h->st));
  }
  {
    PROF(GPT2_PROF_OTHER, 0, 4.0 * M);
    H_TRY(h, launch_mean(h->row_loss, M, h->d_loss, h->st));
    if (d_row_loss)
      H_CUDA(h, cudaMemcpyAsync(d_row_loss, h->row_loss, M * sizeof(float),
                                cudaMemcpyDeviceToDevice, h->st));
  }
  h->fwd_saved = save;
  h->fB = B;
  h->fT = T;
  return GPT2_OK;
}

// ------------------------------------------------------------------ backward
// Gradient buckets in the order the backward finishes them (see
// gpt2_grad_buckets): bucket L-1-l is the four matrices of layer l, one
// contiguous range of the 2-D part of the arena (qkv, proj, fc, fc-proj in
// that order); bucket L is wte and wpe (the arena's first range) and every
// vector (its last).
struct BucketRange {
  int64_t off, n;
  int b;
};
std::vector<BucketRange> bucket_plan(const gpt2_handle& t) {
  std::vector<BucketRange> r;
  for (int l = t.L - 1; l >= 0; --l) {
    const TensorInfo* q = &t.tensors[2 + 12 * l];
    const int64_t a = q[2].off, e = q[10].off + align_up(q[10].rows * q[10].cols, kAlign);
    r.push_back({a, e - a, t.L - 1 - l});
  }
  r.push_back({0, t.tensors[2 + 2].off, t.L});
  r.push_back({t.n_decay, t.n_arena - t.n_decay, t.L});
  return r;
}

// Bucket b of the gradient arena is final once the work enqueued so far on
// the handle's stream is done: start its exchange (in-library NCCL) and tell
// the caller's callback, if any.
int bucket_ready(gpt2_handle* h, int b) {
  if (h->dp_comm && h->dp_sync) {
    // the communication stream picks up here: bucket b is final on st
    H_CUDA(h, cudaEventRecord(h->ev_dp, h->st));
    H_CUDA(h, cudaStreamWaitEvent(h->st_comm, h->ev_dp, 0));
    H_TRY(h, gpt2_internal::dp_allreduce_ranges(h->dp_comm, h->dp_ranges[b], h->G, h->st_comm));
    h->dp_pending = true;
  }
  if (h->bucket_fn && !h->capturing) h->bucket_fn(h->bucket_user, b);
  return GPT2_OK;
}

template <typename A>
int backward_t(gpt2_handle* h, float grad_scale) {
  const int B = h->fB, T = h->fT;
  const int64_t M = int64_t(B) * T;
  const int C = h->C, F = h->F, Vp = h->Vp, Hh = h->H;
  const int ab = h->use_bf16;
  const double a = double(sizeof(A));
  const float* P = h->P;
  float* G = h->G;
  const int acc = h->grads_zero ? 0 : 1;
  A* hf = static_cast<A*>(h->hf);
  A* dhf = static_cast<A*>(h->dhf);
  A* dres_a = static_cast<A*>(h->dres_a);
  const float scale = grad_scale / float(M);

  {
    // tied head: dz = scale (softmax - onehot); dhf = dz W; dW += dz^T hf
    // (algorithmic work: the dH and dW contractions; the logits are recomputed)
    PROF(GPT2_PROF_LMHEAD, 2 * gemm_flops(M, Vp, C),
         a * (2.0 * M * C + double(Vp) * C) + 8.0 * double(Vp) * C);
    LmSide side;  // dW beside dH (not while profiling, so each group is timed alone)
    if (!h->prof_on) {
      side.st = h->st2;
      side.e_fork = h->ev_fork;
      side.e_join[0] = h->ev_join;
      side.e_join[1] = h->ev_join2;
      side.ws = h->ws2;
      side.ws_bytes = h->ws_bytes;
    }
    H_TRY(h, lmhead_bwd(hf, wptr(h, h->off_wte), h->ybuf, h->hlse, int(M), C, Vp, h->use_bf16,
                        scale, dhf, G + h->off_wte, acc, h->lm_ws, h->lm_ws_bytes, h->st, &side));
  }
  A* copy = ab ? dres_a : nullptr;
  const double lnb_bytes = M * C * (4.0 + 8.0 + 2.0 * a) + 8.0 * M;
  {
    PROF(GPT2_PROF_LN_BWD, 0, lnb_bytes);
    H_CUDA(h, cudaMemsetAsync(h->dres, 0, M * C * sizeof(float), h->st));
    h->defer.clear();
    // the residual gradient it leaves is the last layer's mlp.proj bias gradient
    H_TRY(h, (launch_layernorm_bwd<A, A>(dhf, h->res[2 * h->L], h->muf, h->rsf, P + h->off_lnfw,
                                          M, C, h->dres, copy, G + h->off_lnfw, G + h->off_lnfb,
                                          G + h->lo[h->L - 1].fpb, acc,
                                          h->ln_parts + 2 * h->L * h->ln_stride, h->st,
                                          &h->defer)));
  }
  A* du = static_cast<A*>(h->du);
  A* dln = static_cast<A*>(h->dln);
  A* datt = static_cast<A*>(h->datt);
  A* dqkv = static_cast<A*>(h->dqkv);
  const double attn_bwd_flops = 4.0 * B * Hh * double(T) * T * (C / Hh);
  // the attention kernels leave the attn.qkv bias column sums (bf16 tcgen05 path)
  const bool qkvb_fused = h->qkvb_parts && attn_bias_parts_written(B, T, C, Hh, h->ads);
  // Each weight-gradient GEMM (and the bias column sum beside it) is
  // independent of the input-gradient GEMM of the same layer: they run on the
  // side stream, launched after it, so that they fill its last partial wave;
  // joined back before the LayerNorm backward overwrites the bf16 dres copy.
  Side sd{h, !h->prof_on};
  for (int l = h->L - 1; l >= 0; --l) {
    const LayerOff& o = h->lo[l];
    {
      // mlp.proj: h'' = h' + g Wfp^T + b;  du = (dres Wfp) * gelu'(u)
      PROF(GPT2_PROF_GEMM, 2 * gemm_flops(M, F, C), a * (2.0 * M * C + 3.0 * M * F + F * C) + 8.0 * F * C);
      H_TRY(h, sd.fork());
      EpiParams e = epi(EPI_GELU_BWD, du, F, ab);
      e.aux = h->u[l];
      H_TRY(h, gemm(h, dres_a, 1, C, wptr(h, o.fpw), 0, F, int(M), F, C, e));
      e = epi(EPI_ACC, G + o.fpw, F, 0);
      e.accumulate = acc;
      H_TRY(h, gemm(h, dres_a, 0, C, h->g[l], 0, F, C, F, int(M), e, sd.st(), sd.ws()));
      // no join yet: the side stream runs in order, and the join before the
      // LayerNorm backward (which rewrites dres_a) also covers this GEMM
    }
    {
      // mlp.fc: u = ln2 Wfc^T + b
      PROF(GPT2_PROF_GEMM, 2 * gemm_flops(M, C, F), a * (2.0 * M * F + 2.0 * M * C + F * C) + 8.0 * F * C);
      H_TRY(h, sd.fork());
      EpiParams e = epi(EPI_STORE, dln, C, ab);
      H_TRY(h, gemm(h, du, 1, F, wptr(h, o.fcw), 0, C, int(M), C, F, e));
      e = epi(EPI_ACC, G + o.fcw, C, 0);
      e.accumulate = acc;
      H_TRY(h, gemm(h, du, 0, F, h->ln2[l], 0, C, F, C, int(M), e, sd.st(), sd.ws()));
    }
    {
      PROF(GPT2_PROF_OTHER, 0, a * M * F);
      H_TRY(h, launch_colsum<A>(du, M, F, G + o.fcb, acc, h->cs_parts + l * h->cs_stride,
                                sd.st(), &h->defer));
      H_TRY(h, sd.join());
    }
    {
      PROF(GPT2_PROF_LN_BWD, 0, lnb_bytes);
      // ... and attn.proj's bias gradient: column sums of the residual gradient
      H_TRY(h, (launch_layernorm_bwd<A, A>(dln, h->res[2 * l + 1], h->mu2[l], h->rs2[l],
                                            P + o.ln2w, M, C, h->dres, copy, G + o.ln2w,
                                            G + o.ln2b, G + o.projb, acc,
                                            h->ln_parts + (2 * l + 1) * h->ln_stride, h->st,
                                            &h->defer)));
    }
    {
      // attn.proj: h' = h + att Wp^T + b
      PROF(GPT2_PROF_GEMM, 2 * gemm_flops(M, C, C), a * (4.0 * M * C + C * C) + 8.0 * C * C);
      H_TRY(h, sd.fork());
      EpiParams e = epi(EPI_STORE, datt, C, ab);
      H_TRY(h, gemm(h, dres_a, 1, C, wptr(h, o.projw), 0, C, int(M), C, C, e));
      e = epi(EPI_ACC, G + o.projw, C, 0);
      e.accumulate = acc;
      H_TRY(h, gemm(h, dres_a, 0, C, h->att[l], 0, C, C, C, int(M), e, sd.st(), sd.ws()));
    }
    {
      PROF(GPT2_PROF_ATTN_BWD, attn_bwd_flops, a * 9.0 * M * C + 8.0 * M * Hh);
      if constexpr (std::is_same<A, bf16>::value) {
        float* qp = h->qkvb_parts ? h->qkvb_parts + l * h->qkvb_stride : nullptr;
        H_TRY(h, launch_attn_bwd_ds(datt, static_cast<A*>(h->qkv[l]), static_cast<A*>(h->att[l]),
                                    h->alse[l], B, T, C, Hh, dqkv, h->ws, h->ads, h->st, qp));
        // attn.qkv bias gradient from the kernels' per-block column sums
        if (qkvb_fused) {
          const int parts = B * attn_bias_parts(T);
          h->defer.push_back(RowSum{qp, G + o.qkvb, nullptr, nullptr, parts, 3 * C, 3 * C, acc});
        }
      } else
        H_TRY(h, launch_attn_bwd<A>(datt, static_cast<A*>(h->qkv[l]), static_cast<A*>(h->att[l]),
                                    h->alse[l], B, T, C, Hh, dqkv, h->ws, h->st));
      H_TRY(h, sd.join());  // attn.proj's weight gradient ran beside the attention backward
    }
    {
      // attn.qkv: qkv = ln1 Wqkv^T + b
      PROF(GPT2_PROF_GEMM, 2 * gemm_flops(M, C, 3 * C),
           a * (6.0 * M * C + 2.0 * M * C + 3.0 * C * C) + 12.0 * C * C);
      H_TRY(h, sd.fork());
      EpiParams e = epi(EPI_STORE, dln, C, ab);
      H_TRY(h, gemm(h, dqkv, 1, 3 * C, wptr(h, o.qkvw), 0, C, int(M), C, 3 * C, e));
      e = epi(EPI_ACC, G + o.qkvw, C, 0);
      e.accumulate = acc;
      H_TRY(h, gemm(h, dqkv, 0, 3 * C, h->ln1[l], 0, C, 3 * C, C, int(M), e, sd.st(), sd.ws()));
    }
    {
      PROF(GPT2_PROF_OTHER, 0, a * 3.0 * M * C);
      if (!qkvb_fused)
        H_TRY(h, launch_colsum<A>(dqkv, M, 3 * C, G + o.qkvb, acc,
                                  h->cs_parts + l * h->cs_stride + h->cs_qkv_off, sd.st(),
                                  &h->defer));
      H_TRY(h, sd.join());
    }
    {
      PROF(GPT2_PROF_LN_BWD, 0, lnb_bytes);
      // ... and the previous layer's mlp.proj bias gradient
      H_TRY(h, (launch_layernorm_bwd<A, A>(dln, h->res[2 * l], h->mu1[l], h->rs1[l], P + o.ln1w,
                                            M, C, h->dres, copy, G + o.ln1w, G + o.ln1b,
                                            l > 0 ? G + h->lo[l - 1].fpb : nullptr, acc,
                                            h->ln_parts + 2 * l * h->ln_stride, h->st,
                                            &h->defer)));
    }
    // layer l's weight matrices are final on st (every side-stream writer joined)
    H_TRY(h, bucket_ready(h, h->L - 1 - l));
  }
  {
    // the vector gradients: every partial buffer above, summed in one launch
    // on st (the side stream's fc-bias partials were joined into st with the
    // layer that wrote them); before the last bucket, which holds the vectors
    PROF(GPT2_PROF_OTHER, 0, 0.0);
    H_TRY(h, launch_row_sums(h->defer.data(), int(h->defer.size()), h->st));
    h->defer.clear();
  }
  {
    // embedding: both uses of the tied matrix add into one gradient [LECTURE]
    PROF(GPT2_PROF_EMBED, 0, 4.0 * M * C * 3 + 8.0 * M * C);
    H_TRY(h, launch_embed_bwd(h->xbuf, h->dres, B, T, C, h->V, G + h->off_wte, G + h->off_wpe,
                              acc, h->ws_emb, h->st));
  }
  H_TRY(h, bucket_ready(h, h->L));  // wte, wpe and every vector
  if (h->dp_pending) {  // the averaged gradients are what the next step reads
    H_CUDA(h, cudaEventRecord(h->ev_dp_join, h->st_comm));
    H_CUDA(h, cudaStreamWaitEvent(h->st, h->ev_dp_join, 0));
    h->dp_pending = false;
  }
  h->grads_zero = false;
  return GPT2_OK;
}

int validate_bt(gpt2_handle* h, int B, int T) {
  if (B < 1 || T < 1 || B > h->cfg.max_B || T > h->cfg.max_Tseq || T > h->Tmax)
    return fail(h, GPT2_ERR_ARG, "B or T outside 1..max_B / 1..max_Tseq");
  return GPT2_OK;
}

int read_loss(gpt2_handle* h, float* loss_out) {
  if (!loss_out) return GPT2_OK;
  H_CUDA(h, cudaMemcpyAsync(loss_out, h->d_loss, sizeof(float), cudaMemcpyDeviceToHost, h->st));
  H_TRY(h, check_status(h));
  return GPT2_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int gpt2_create(const gpt2_config* cfg, gpt2_handle** out) {
  if (!out) return fail(nullptr, GPT2_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg) return fail(nullptr, GPT2_ERR_ARG, "cfg is NULL");
  const gpt2_config& c = *cfg;
  const std::string bad = config_problem(c);
  if (!bad.empty()) return fail(nullptr, GPT2_ERR_ARG, bad);
  gpt2_handle* h = new gpt2_handle();
  set_shape(h, c);
  h->st = static_cast<cudaStream_t>(c.stream);
  build_layout(h);

  const int64_t M = h->Mcap, C = h->C, F = h->F, L = h->L, Vp = h->Vp;
  const size_t a = h->act_size();
  const int H = h->H;
  bool ok = true;
  auto A = [&](size_t bytes) -> void* {
    void* p = dev_alloc(h, bytes);
    if (!p) ok = false;
    return p;
  };
  const size_t arena = size_t(h->n_arena) * sizeof(float);
  h->P = static_cast<float*>(A(arena));
  h->G = static_cast<float*>(A(arena));
  h->Mo = static_cast<float*>(A(arena));
  h->Vo = static_cast<float*>(A(arena));
  if (h->use_bf16) h->Pb = static_cast<bf16*>(A(size_t(h->n_arena) * sizeof(bf16)));
  h->xbuf = static_cast<int32_t*>(A(M * sizeof(int32_t)));
  h->ybuf = static_cast<int32_t*>(A(M * sizeof(int32_t)));
  h->res.resize(2 * L + 1);
  for (auto& r : h->res) r = static_cast<float*>(A(M * C * sizeof(float)));
  h->ln1.resize(L); h->qkv.resize(L); h->att.resize(L); h->ln2.resize(L); h->u.resize(L);
  h->g.resize(L); h->mu1.resize(L); h->rs1.resize(L); h->mu2.resize(L); h->rs2.resize(L);
  h->alse.resize(L);
  for (int l = 0; l < L; ++l) {
    h->ln1[l] = A(M * C * a);
    h->qkv[l] = A(M * 3 * C * a);
    h->att[l] = A(M * C * a);
    h->ln2[l] = A(M * C * a);
    h->u[l] = A(M * F * a);
    h->g[l] = A(M * F * a);
    h->mu1[l] = static_cast<float*>(A(M * sizeof(float)));
    h->rs1[l] = static_cast<float*>(A(M * sizeof(float)));
    h->mu2[l] = static_cast<float*>(A(M * sizeof(float)));
    h->rs2[l] = static_cast<float*>(A(M * sizeof(float)));
    h->alse[l] = static_cast<float*>(A(size_t(M) * H * sizeof(float)));
  }
  h->hf = A(M * C * a);
  h->muf = static_cast<float*>(A(M * sizeof(float)));
  h->rsf = static_cast<float*>(A(M * sizeof(float)));
  h->row_loss = static_cast<float*>(A(M * sizeof(float)));
  h->hlse = static_cast<float*>(A(M * sizeof(float)));
  h->d_loss = static_cast<float*>(A(sizeof(float)));
  h->d_norm = static_cast<float*>(A(sizeof(float)));
  h->dres = static_cast<float*>(A(M * C * sizeof(float)));
  h->dres_a = h->use_bf16 ? A(M * C * a) : static_cast<void*>(h->dres);
  h->dln = A(M * C * a);
  h->datt = A(M * C * a);
  h->dqkv = A(M * 3 * C * a);
  h->du = A(M * F * a);
  h->dhf = A(M * C * a);
  h->lm_ws_bytes = lmhead_workspace(int(M), int(C), int(Vp), h->use_bf16);
  h->lm_ws = A(h->lm_ws_bytes);
  // general fp32 workspace: max of every user's need
  size_t ws = 0;
  ws = std::max(ws, layernorm_bwd_workspace(M, int(C)));
  ws = std::max(ws, colsum_workspace(M, int(std::max(F, 3 * C))));
  ws = std::max(ws, attn_bwd_workspace(c.max_B, c.max_Tseq, H));
  const int shapes[][3] = {{int(C), int(F), int(M)}, {int(F), int(C), int(M)},
                           {int(C), int(C), int(M)}, {int(3 * C), int(C), int(M)}};
  for (auto& s : shapes) ws = std::max(ws, gemm_workspace_bytes(s[0], s[1], s[2]));
  h->ws_bytes = ws;
  h->ws = static_cast<float*>(A(ws));
  h->ws2 = static_cast<float*>(A(ws));
  auto r64 = [](size_t n) { return (n + 63) / 64 * 64; };  // floats, rounded to 256 bytes
  if (h->use_bf16 && attn_tc_supported(c.max_B, c.max_Tseq, int(C), H)) {
    h->ads = static_cast<bf16*>(A(attn_tc_ds_bytes(c.max_B, c.max_Tseq, H)));
    h->qkvb_stride = r64(size_t(c.max_B) * attn_bias_parts(c.max_Tseq) * 3 * C);
    h->qkvb_parts = static_cast<float*>(A(size_t(h->L) * h->qkvb_stride * sizeof(float)));
  }
  // (every buffer starts on a 256-byte boundary: the staged kernels want 16)
  h->ln_stride = r64(layernorm_bwd_workspace(M, int(C)) / sizeof(float));
  h->ln_parts = static_cast<float*>(A(size_t(2 * h->L + 1) * h->ln_stride * sizeof(float)));
  h->cs_qkv_off = r64(colsum_workspace(M, int(F)) / sizeof(float));
  h->cs_stride = h->cs_qkv_off + r64(colsum_workspace(M, int(3 * C)) / sizeof(float));
  h->cs_parts = static_cast<float*>(A(size_t(h->L) * h->cs_stride * sizeof(float)));
  h->ws_emb = A(embed_bwd_workspace(M, int(C)));
  h->ws_norm = static_cast<double*>(A(gradnorm_workspace()));
  h->status = static_cast<DevStatus*>(A(sizeof(DevStatus)));
  h->d_cursor = static_cast<int64_t*>(A(sizeof(int64_t)));
  h->d_lr = static_cast<float*>(A(sizeof(float)));
  if (!ok) {
    free_all(h);
    delete h;
    return fail(nullptr, GPT2_ERR_OOM, "device allocation failed");
  }
  if (cudaStreamCreateWithFlags(&h->st2, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&h->ev_join2, cudaEventDisableTiming) != cudaSuccess) {
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->st2) cudaStreamDestroy(h->st2);
    free_all(h);
    delete h;
    return fail(nullptr, GPT2_ERR_CUDA, "creating the side stream failed");
  }
  cudaStream_t st = h->st;
  bool cz = cudaMemsetAsync(h->P, 0, arena, st) == cudaSuccess &&
            cudaMemsetAsync(h->G, 0, arena, st) == cudaSuccess &&
            cudaMemsetAsync(h->Mo, 0, arena, st) == cudaSuccess &&
            cudaMemsetAsync(h->Vo, 0, arena, st) == cudaSuccess &&
            cudaMemsetAsync(h->status, 0, sizeof(DevStatus), st) == cudaSuccess &&
            cudaStreamSynchronize(st) == cudaSuccess;
  if (!cz) {
    free_all(h);
    delete h;
    return fail(nullptr, GPT2_ERR_CUDA, "initialising device memory failed");
  }
  *out = h;
  return GPT2_OK;
}

int gpt2_destroy(gpt2_handle* h) {
  if (!h) return GPT2_OK;
  cudaStreamSynchronize(h->st);
  if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
  if (h->graph) cudaGraphDestroy(h->graph);
  if (h->st2) {
    cudaStreamSynchronize(h->st2);
    cudaStreamDestroy(h->st2);
  }
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->ev_join2) cudaEventDestroy(h->ev_join2);
  if (h->st_comm) {
    cudaStreamSynchronize(h->st_comm);
    cudaStreamDestroy(h->st_comm);
  }
  if (h->ev_dp) cudaEventDestroy(h->ev_dp);
  if (h->ev_dp_join) cudaEventDestroy(h->ev_dp_join);
  gpt2_internal::dp_comm_destroy(h->dp_comm);
  prof_collect(h);
  for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
  free_all(h);
  delete h;
  return GPT2_OK;
}

const char* gpt2_last_error(const gpt2_handle* h) {
  return h ? h->err.c_str() : gpt2_internal::get_error().c_str();
}

int gpt2_num_tensors(const gpt2_handle* h, int* n) {
  if (!h || !n) return GPT2_ERR_ARG;
  *n = int(h->tensors.size());
  return GPT2_OK;
}

int gpt2_tensor_info(const gpt2_handle* h, int i, const char** name, int* ndim, int64_t shape[2],
                     int* decay) {
  if (!h || i < 0 || i >= int(h->tensors.size())) return GPT2_ERR_ARG;
  const TensorInfo& t = h->tensors[i];
  if (name) *name = t.name.c_str();
  if (ndim) *ndim = t.ndim;
  if (shape) {
    shape[0] = t.rows;
    shape[1] = t.cols;
  }
  if (decay) *decay = t.decay;
  return GPT2_OK;
}

int gpt2_param_count(const gpt2_handle* h, int64_t* n) {
  if (!h || !n) return GPT2_ERR_ARG;
  int64_t s = 0;
  for (auto& t : h->tensors) s += t.rows * t.cols;
  *n = s;
  return GPT2_OK;
}

static float* arena_of(gpt2_handle* h, int which) {
  switch (which) {
    case GPT2_PARAM: return h->P;
    case GPT2_GRAD: return h->G;
    case GPT2_ADAM_M: return h->Mo;
    case GPT2_ADAM_V: return h->Vo;
  }
  return nullptr;
}

int gpt2_set_tensor(gpt2_handle* h, int i, int which, const float* src, int on_device) {
  if (!h || !src || i < 0 || i >= int(h->tensors.size())) return fail(h, GPT2_ERR_ARG, "bad tensor");
  float* base = arena_of(h, which);
  if (!base) return fail(h, GPT2_ERR_ARG, "bad selector");
  const TensorInfo& t = h->tensors[i];
  const size_t bytes = size_t(t.rows * t.cols) * sizeof(float);
  if (which == GPT2_GRAD && h->grads_zero) {
    // materialise the lazy zero before a partial write
    H_CUDA(h, cudaMemsetAsync(h->G, 0, size_t(h->n_arena) * sizeof(float), h->st));
    h->grads_zero = false;
  }
  H_CUDA(h, cudaMemcpyAsync(base + t.off, src, bytes,
                            on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, h->st));
  if (!on_device) H_CUDA(h, cudaStreamSynchronize(h->st));
  if (which == GPT2_PARAM) h->mirror_dirty = true;
  return GPT2_OK;
}

int gpt2_get_tensor(gpt2_handle* h, int i, int which, float* dst, int on_device) {
  if (!h || !dst || i < 0 || i >= int(h->tensors.size())) return fail(h, GPT2_ERR_ARG, "bad tensor");
  float* base = arena_of(h, which);
  if (!base) return fail(h, GPT2_ERR_ARG, "bad selector");
  const TensorInfo& t = h->tensors[i];
  const size_t bytes = size_t(t.rows * t.cols) * sizeof(float);
  if (which == GPT2_GRAD && h->grads_zero) {
    if (on_device)
      H_CUDA(h, cudaMemsetAsync(dst, 0, bytes, h->st));
    else
      std::memset(dst, 0, bytes);
    return GPT2_OK;
  }
  H_CUDA(h, cudaMemcpyAsync(dst, base + t.off, bytes,
                            on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost, h->st));
  if (!on_device) H_CUDA(h, cudaStreamSynchronize(h->st));
  return GPT2_OK;
}

int gpt2_get_step(const gpt2_handle* hc, int* t) {
  gpt2_handle* h = const_cast<gpt2_handle*>(hc);
  if (!h || !t) return GPT2_ERR_ARG;
  DevStatus s;
  H_CUDA(h, cudaMemcpyAsync(&s, h->status, sizeof(s), cudaMemcpyDeviceToHost, h->st));
  H_CUDA(h, cudaStreamSynchronize(h->st));
  *t = s.step;
  return GPT2_OK;
}

int gpt2_set_step(gpt2_handle* h, int t) {
  if (!h || t < 0) return fail(h, GPT2_ERR_ARG, "bad step");
  H_CUDA(h, cudaMemcpyAsync(reinterpret_cast<char*>(h->status) + offsetof(DevStatus, step), &t,
                            sizeof(int), cudaMemcpyHostToDevice, h->st));
  H_CUDA(h, cudaStreamSynchronize(h->st));
  return GPT2_OK;
}

int gpt2_batch_from_stream(gpt2_handle* h, const uint16_t* d_stream, int64_t stream_len,
                           int64_t offset, int B, int T, int32_t* d_x, int32_t* d_y) {
  if (!h || !d_stream || !d_x || !d_y || B < 1 || T < 1 || offset < 0 ||
      offset + int64_t(B) * T + 1 > stream_len)
    return fail(h, GPT2_ERR_ARG, "batch_from_stream: window outside the stream");
  H_TRY(h, launch_slice_batch(d_stream, offset, int64_t(B) * T, d_x, d_y, h->st));
  return GPT2_OK;
}

int gpt2_forward_loss(gpt2_handle* h, const int32_t* x, const int32_t* y, int B, int T,
                      int tokens_on_device, float* loss_out, float* d_row_loss) {
  if (!h || !x || !y) return fail(h, GPT2_ERR_ARG, "NULL argument");
  H_TRY(h, validate_bt(h, B, T));
  h->fwd_saved = false;
  H_TRY(h, stage_tokens(h, x, y, int64_t(B) * T, tokens_on_device));
  if (h->use_bf16)
    H_TRY(h, forward_t<bf16>(h, B, T, d_row_loss, true));
  else
    H_TRY(h, forward_t<float>(h, B, T, d_row_loss, true));
  return read_loss(h, loss_out);
}

int gpt2_backward(gpt2_handle* h, float grad_scale) {
  if (!h) return GPT2_ERR_ARG;
  if (!h->fwd_saved) return fail(h, GPT2_ERR_STATE, "backward needs a preceding forward_loss");
  if (h->use_bf16)
    H_TRY(h, backward_t<bf16>(h, grad_scale));
  else
    H_TRY(h, backward_t<float>(h, grad_scale));
  return GPT2_OK;
}

int gpt2_zero_grad(gpt2_handle* h) {
  if (!h) return GPT2_ERR_ARG;
  h->grads_zero = true;
  return GPT2_OK;
}

int gpt2_clip_adamw_step(gpt2_handle* h, float lr, float beta1, float beta2, float eps,
                         float weight_decay, float max_norm, float* grad_norm_out) {
  if (!h) return GPT2_ERR_ARG;
  if (!(beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f && eps >= 0.f && max_norm > 0.f))
    return fail(h, GPT2_ERR_ARG, "bad optimiser hyper-parameters");
  if (h->grads_zero) {
    H_CUDA(h, cudaMemsetAsync(h->G, 0, size_t(h->n_arena) * sizeof(float), h->st));
    h->grads_zero = false;
  }
  {
    PROF(GPT2_PROF_OPTIM, 14.0 * h->n_arena, (34.0 + (h->use_bf16 ? 2.0 : 0.0)) * h->n_arena);
    H_TRY(h, launch_gradnorm(h->G, h->n_arena, h->ws_norm, h->d_norm, h->st));
    H_TRY(h, launch_clip_adamw(h->P, h->G, h->Mo, h->Vo, h->Pb, h->n_arena, h->n_decay, h->d_norm,
                               h->status, lr, nullptr, beta1, beta2, eps, weight_decay, max_norm,
                               h->st));
  }
  h->mirror_dirty = false;  // the pass rewrote the bf16 mirror
  if (grad_norm_out) {
    H_CUDA(h, cudaMemcpyAsync(grad_norm_out, h->d_norm, sizeof(float), cudaMemcpyDeviceToHost,
                              h->st));
    H_TRY(h, check_status(h));
  }
  return GPT2_OK;
}

int gpt2_train_step(gpt2_handle* h, const int32_t* x, const int32_t* y, int B, int T,
                    int tokens_on_device, float lr, float beta1, float beta2, float eps,
                    float weight_decay, float max_norm, float* loss_out, float* grad_norm_out) {
  if (!h) return GPT2_ERR_ARG;
  H_TRY(h, gpt2_zero_grad(h));
  H_TRY(h, gpt2_forward_loss(h, x, y, B, T, tokens_on_device, nullptr, nullptr));
  H_TRY(h, gpt2_backward(h, 1.f));
  H_TRY(h, gpt2_clip_adamw_step(h, lr, beta1, beta2, eps, weight_decay, max_norm, nullptr));
  if (loss_out)
    H_CUDA(h, cudaMemcpyAsync(loss_out, h->d_loss, sizeof(float), cudaMemcpyDeviceToHost, h->st));
  if (grad_norm_out)
    H_CUDA(h, cudaMemcpyAsync(grad_norm_out, h->d_norm, sizeof(float), cudaMemcpyDeviceToHost,
                              h->st));
  if (loss_out || grad_norm_out) H_TRY(h, check_status(h));
  return GPT2_OK;
}

int gpt2_eval_loss(gpt2_handle* h, const int32_t* x, const int32_t* y, int B, int T,
                   int tokens_on_device, float* loss_out) {
  if (!h || !x || !y || !loss_out) return fail(h, GPT2_ERR_ARG, "NULL argument");
  H_TRY(h, validate_bt(h, B, T));
  h->fwd_saved = false;
  H_TRY(h, stage_tokens(h, x, y, int64_t(B) * T, tokens_on_device));
  if (h->use_bf16)
    H_TRY(h, forward_t<bf16>(h, B, T, nullptr, false));
  else
    H_TRY(h, forward_t<float>(h, B, T, nullptr, false));
  return read_loss(h, loss_out);
}

int gpt2_logits_last(gpt2_handle* h, const int32_t* x, int B, int T, int tokens_on_device,
                     float* logits, int64_t ld) {
  if (!h || !x || !logits) return fail(h, GPT2_ERR_ARG, "NULL argument");
  H_TRY(h, validate_bt(h, B, T));
  if (ld < h->Vp) return fail(h, GPT2_ERR_ARG, "logits_last: ld below padded_vocab");
  h->fwd_saved = false;
  // the targets buffer only feeds the embedding's id range check: give it x
  H_TRY(h, stage_tokens(h, x, x, int64_t(B) * T, tokens_on_device));
  if (h->use_bf16)
    H_TRY(h, forward_t<bf16>(h, B, T, nullptr, false, logits, ld));
  else
    H_TRY(h, forward_t<float>(h, B, T, nullptr, false, logits, ld));
  return check_status(h);
}

int gpt2_generate(gpt2_handle* h, const int32_t* prompt, int B, int T0, int n_new,
                  float temperature, int top_k, float top_p, const float* uniform,
                  int32_t* out) {
  if (!h || !prompt || !out) return fail(h, GPT2_ERR_ARG, "NULL argument");
  if (B < 1 || B > h->cfg.max_B || T0 < 1 || n_new < 0)
    return fail(h, GPT2_ERR_ARG, "generate: B outside 1..max_B, T0 < 1 or n_new < 0");
  const bool greedy = temperature == 0.f || top_k == 1;
  if (!(temperature >= 0.f) || top_k < 0 || !(top_p > 0.f && top_p <= 1.f) ||
      (!greedy && !uniform))
    return fail(h, GPT2_ERR_ARG, "generate: bad sampling settings or no uniform numbers");
  if (h->V > kSampleMaxVocab) return fail(h, GPT2_ERR_ARG, "generate: vocab_size above 53248");
  const int Wmax = std::min(h->Tmax, h->cfg.max_Tseq);
  const int64_t Ttot = int64_t(T0) + n_new;
  h->fwd_saved = false;
  if (!h->gen_logits) {
    h->gen_logits = static_cast<float*>(dev_alloc(h, size_t(h->cfg.max_B) * h->Vp * sizeof(float)));
    if (!h->gen_logits) return fail(h, GPT2_ERR_OOM, "generate: logits buffer");
  }
  H_CUDA(h, cudaMemcpy2DAsync(out, Ttot * sizeof(int32_t), prompt, T0 * sizeof(int32_t),
                              T0 * sizeof(int32_t), B, cudaMemcpyDeviceToDevice, h->st));
  for (int s = 0; s < n_new; ++s) {
    const int64_t Tc = int64_t(T0) + s;
    const int W = int(std::min<int64_t>(Tc, Wmax));
    // the window out[:, Tc-W .. Tc) as a contiguous [B, W] batch
    H_CUDA(h, cudaMemcpy2DAsync(h->xbuf, W * sizeof(int32_t), out + (Tc - W),
                                Ttot * sizeof(int32_t), W * sizeof(int32_t), B,
                                cudaMemcpyDeviceToDevice, h->st));
    H_CUDA(h, cudaMemcpyAsync(h->ybuf, h->xbuf, size_t(B) * W * sizeof(int32_t),
                              cudaMemcpyDeviceToDevice, h->st));
    if (h->use_bf16)
      H_TRY(h, forward_t<bf16>(h, B, W, nullptr, false, h->gen_logits, h->Vp));
    else
      H_TRY(h, forward_t<float>(h, B, W, nullptr, false, h->gen_logits, h->Vp));
    H_TRY(h, launch_sample(h->gen_logits, h->Vp, B, h->V, temperature, top_k, top_p,
                           greedy ? nullptr : uniform + int64_t(s) * B, out + Tc, Ttot, h->st));
  }
  return check_status(h);
}

int gpt2_generate_cached(gpt2_handle* h, const int32_t* prompt, int B, int T0, int n_new,
                         float temperature, int top_k, float top_p, const float* uniform,
                         int32_t* out) {
  if (!h || !prompt || !out) return fail(h, GPT2_ERR_ARG, "NULL argument");
  const int Tc = std::min(h->Tmax, h->cfg.max_Tseq);
  if (B < 1 || B > h->cfg.max_B || T0 < 1 || n_new < 0 || int64_t(T0) + n_new > Tc)
    return fail(h, GPT2_ERR_ARG,
                "generate_cached: B outside 1..max_B, T0 < 1, n_new < 0 or T0 + n_new above "
                "min(max_T, max_Tseq)");
  const bool greedy = temperature == 0.f || top_k == 1;
  if (!(temperature >= 0.f) || top_k < 0 || !(top_p > 0.f && top_p <= 1.f) ||
      (!greedy && !uniform))
    return fail(h, GPT2_ERR_ARG, "generate_cached: bad sampling settings or no uniform numbers");
  if (h->V > kSampleMaxVocab)
    return fail(h, GPT2_ERR_ARG, "generate_cached: vocab_size above 53248");
  if (Tc > 4096 || (h->C / h->H) > 128 || 128 % (h->C / h->H) != 0)
    return fail(h, GPT2_ERR_ARG, "generate_cached: context above 4096 or head size unsupported");
  const int64_t Ttot = int64_t(T0) + n_new;
  h->fwd_saved = false;
  if (!h->gen_logits) {
    h->gen_logits = static_cast<float*>(dev_alloc(h, size_t(h->cfg.max_B) * h->Vp * sizeof(float)));
    if (!h->gen_logits) return fail(h, GPT2_ERR_OOM, "generate: logits buffer");
  }
  if (!h->kcache) {
    const size_t bytes = size_t(h->L) * h->cfg.max_B * h->C * size_t(Tc) * h->act_size();
    h->kcache = dev_alloc(h, bytes);
    h->vcache = dev_alloc(h, bytes);
    if (!h->kcache || !h->vcache) return fail(h, GPT2_ERR_OOM, "generate_cached: KV cache");
    h->kv_T = Tc;
  }
  H_CUDA(h, cudaMemcpy2DAsync(out, Ttot * sizeof(int32_t), prompt, T0 * sizeof(int32_t),
                              T0 * sizeof(int32_t), B, cudaMemcpyDeviceToDevice, h->st));
  if (n_new == 0) return check_status(h);
  if (h->use_bf16 && h->mirror_dirty) H_TRY(h, launch_to_bf16(h->P, h->Pb, h->n_arena, h->st));
  h->mirror_dirty = false;
  // step 0: the prompt at positions 0 .. T0-1 fills the cache and gives token T0
  {
    const KvStep kv{0, false};
    H_CUDA(h, cudaMemcpy2DAsync(h->xbuf, T0 * sizeof(int32_t), out, Ttot * sizeof(int32_t),
                                T0 * sizeof(int32_t), B, cudaMemcpyDeviceToDevice, h->st));
    H_CUDA(h, cudaMemcpyAsync(h->ybuf, h->xbuf, size_t(B) * T0 * sizeof(int32_t),
                              cudaMemcpyDeviceToDevice, h->st));
    if (h->use_bf16)
      H_TRY(h, forward_t<bf16>(h, B, T0, nullptr, false, h->gen_logits, h->Vp, &kv));
    else
      H_TRY(h, forward_t<float>(h, B, T0, nullptr, false, h->gen_logits, h->Vp, &kv));
    H_TRY(h, launch_sample(h->gen_logits, h->Vp, B, h->V, temperature, top_k, top_p,
                           greedy ? nullptr : uniform, out + T0, Ttot, h->st));
  }
  if (n_new == 1) return check_status(h);
  // Steps s = 1 .. n_new-1: the token at position T0+s-1 through the block,
  // attending to the cache; s lives on the device (*gen_step) so that one
  // recorded step serves every position.
  if (!h->gen_step) {
    h->gen_step = static_cast<int*>(dev_alloc(h, sizeof(int)));
    if (!h->gen_step) return fail(h, GPT2_ERR_OOM, "generate_cached: step counter");
  }
  const int one = 1;
  H_CUDA(h, cudaMemcpyAsync(h->gen_step, &one, sizeof(int), cudaMemcpyHostToDevice, h->st));
  const KvStep kv{T0 - 1, true, h->gen_step};
  auto step = [&]() -> int {
    H_TRY(h, launch_gen_tokens(out, Ttot, B, T0 - 1, h->gen_step, h->xbuf, h->ybuf, h->st));
    if (h->use_bf16)
      H_TRY(h, forward_t<bf16>(h, B, 1, nullptr, false, h->gen_logits, h->Vp, &kv));
    else
      H_TRY(h, forward_t<float>(h, B, 1, nullptr, false, h->gen_logits, h->Vp, &kv));
    H_TRY(h, launch_sample(h->gen_logits, h->Vp, B, h->V, temperature, top_k, top_p,
                           greedy ? nullptr : uniform, out + T0, Ttot, h->st, h->gen_step,
                           int64_t(B), 1));
    H_TRY(h, launch_step_add(h->gen_step, h->st));
    return GPT2_OK;
  };
  if (h->prof_on) {  // every kernel group timed on its own: no graph
    for (int s = 1; s < n_new; ++s) H_TRY(h, step());
    return check_status(h);
  }
  // record one step on a private stream (the handle's stream may be the legacy
  // default stream, which cannot be captured), then replay it n_new-1 times
  H_CUDA(h, cudaStreamSynchronize(h->st));
  cudaStream_t user = h->st, cs = nullptr;
  H_CUDA(h, cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
  h->st = cs;
  int rc = GPT2_OK;
  cudaGraph_t g = nullptr;
  cudaError_t ec = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (ec == cudaSuccess) {
    rc = step();
    ec = cudaStreamEndCapture(cs, &g);
  }
  h->st = user;
  cudaStreamDestroy(cs);
  if (rc != GPT2_OK || ec != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    if (rc != GPT2_OK) return rc;
    return fail(h, GPT2_ERR_CUDA, std::string("generate_cached: capture failed: ") +
                                      cudaGetErrorString(ec));
  }
  cudaGraphExec_t ge = nullptr;
  cudaError_t ei = cudaGraphInstantiate(&ge, g, 0);
  cudaGraphDestroy(g);
  if (ei != cudaSuccess)
    return fail(h, GPT2_ERR_CUDA, std::string("generate_cached: graph instantiation failed: ") +
                                      cudaGetErrorString(ei));
  cudaError_t el = cudaSuccess;
  for (int s = 1; s < n_new && el == cudaSuccess; ++s) el = cudaGraphLaunch(ge, h->st);
  cudaError_t es = cudaStreamSynchronize(h->st);
  cudaGraphExecDestroy(ge);
  if (el != cudaSuccess || es != cudaSuccess)
    return fail(h, GPT2_ERR_CUDA, std::string("generate_cached: replay failed: ") +
                                      cudaGetErrorString(el != cudaSuccess ? el : es));
  return check_status(h);
}

// ---------------------------------------------------------------- stream training (graph)
// One optimizer step on consecutive windows of a device token stream, recorded
// once as a CUDA graph and replayed: zero the gradients; accum times: cut the
// window at the device cursor (x = s[o .. o+BT), y = s[o+1 .. o+BT+1]),
// advance the cursor by `stride`, forward and backward with grad_scale 1/accum;
// then the gradient norm, clip and AdamW with the learning rate read from the
// device.  Every launch is stream-ordered with no host synchronisation, which
// is what lets the step be captured; replaying it costs one graph launch
// instead of some 400 kernel launches.
namespace {
int stream_step_body(gpt2_handle* h, const uint16_t* tok, int64_t len, int64_t stride, int B,
                     int T, int accum, float beta1, float beta2, float eps, float wd,
                     float max_norm) {
  const int64_t n = int64_t(B) * T;
  h->grads_zero = true;
  const bool sync = h->dp_sync;
  for (int a = 0; a < accum; ++a) {
    h->dp_sync = sync && a == accum - 1;  // exchange after the last micro-batch only
    H_TRY(h, launch_slice_batch_cursor(tok, len, h->d_cursor, n, h->xbuf, h->ybuf, h->status,
                                       h->st));
    H_TRY(h, launch_advance_cursor(h->d_cursor, stride, h->st));
    if (h->use_bf16)
      H_TRY(h, forward_t<bf16>(h, B, T, nullptr, true));
    else
      H_TRY(h, forward_t<float>(h, B, T, nullptr, true));
    int rc = h->use_bf16 ? backward_t<bf16>(h, 1.f / float(accum))
                         : backward_t<float>(h, 1.f / float(accum));
    if (rc) {
      h->dp_sync = sync;
      return rc;
    }
  }
  h->dp_sync = sync;
  H_TRY(h, launch_gradnorm(h->G, h->n_arena, h->ws_norm, h->d_norm, h->st));
  H_TRY(h, launch_clip_adamw(h->P, h->G, h->Mo, h->Vo, h->Pb, h->n_arena, h->n_decay, h->d_norm,
                             h->status, 0.f, h->d_lr, beta1, beta2, eps, wd, max_norm, h->st));
  h->mirror_dirty = false;
  return GPT2_OK;
}
}  // namespace

int gpt2_stream_begin(gpt2_handle* h, const uint16_t* d_stream, int64_t stream_len, int64_t start,
                      int64_t stride, int B, int T, int accum, float beta1, float beta2, float eps,
                      float weight_decay, float max_norm) {
  if (!h || !d_stream) return fail(h, GPT2_ERR_ARG, "NULL argument");
  H_TRY(h, validate_bt(h, B, T));
  if (accum < 1 || start < 0 || stride < 0 || stream_len < int64_t(B) * T + 1)
    return fail(h, GPT2_ERR_ARG, "stream_begin: bad accum, start, stride or stream length");
  if (!(beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f && eps >= 0.f && max_norm > 0.f))
    return fail(h, GPT2_ERR_ARG, "bad optimiser hyper-parameters");
  if (h->prof_on) return fail(h, GPT2_ERR_STATE, "stream_begin: disable profiling first");
  if (h->graph_exec) {
    cudaGraphExecDestroy(h->graph_exec);
    h->graph_exec = nullptr;
  }
  if (h->graph) {
    cudaGraphDestroy(h->graph);
    h->graph = nullptr;
  }
  // the bf16 mirror is brought up to date now, not inside every replay
  if (h->use_bf16 && h->mirror_dirty) H_TRY(h, launch_to_bf16(h->P, h->Pb, h->n_arena, h->st));
  h->mirror_dirty = false;
  H_CUDA(h, cudaMemcpyAsync(h->d_cursor, &start, sizeof(int64_t), cudaMemcpyHostToDevice, h->st));
  H_CUDA(h, cudaStreamSynchronize(h->st));
  // Record on a private stream (the handle's stream may be the legacy default
  // stream, which cannot be captured); everything issued before is complete.
  cudaStream_t user = h->st, cs = nullptr;
  H_CUDA(h, cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
  h->st = cs;
  int rc = GPT2_OK;
  cudaGraph_t g = nullptr;
  cudaError_t ec = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (ec == cudaSuccess) {
    h->capturing = true;
    const int64_t k0 = gpt2_internal::launches();
    rc = stream_step_body(h, d_stream, stream_len, stride, B, T, accum, beta1, beta2, eps,
                          weight_decay, max_norm);
    h->graph_kernels = gpt2_internal::launches() - k0;
    h->capturing = false;
    ec = cudaStreamEndCapture(cs, &g);
  }
  h->st = user;
  cudaStreamDestroy(cs);
  if (rc != GPT2_OK) {
    if (g) cudaGraphDestroy(g);
    return rc;
  }
  if (ec != cudaSuccess)
    return fail(h, GPT2_ERR_CUDA, std::string("stream_begin: capture failed: ") +
                                      cudaGetErrorString(ec));
  h->graph = g;
  H_CUDA(h, cudaGraphInstantiate(&h->graph_exec, h->graph, 0));
  return GPT2_OK;
}

int gpt2_stream_steps(gpt2_handle* h, int n_steps, const float* lr) {
  if (!h || (n_steps > 0 && !lr)) return fail(h, GPT2_ERR_ARG, "NULL argument");
  if (!h->graph_exec) return fail(h, GPT2_ERR_STATE, "stream_steps needs stream_begin");
  for (int i = 0; i < n_steps; ++i) {
    H_CUDA(h, cudaMemcpyAsync(h->d_lr, lr + i, sizeof(float), cudaMemcpyHostToDevice, h->st));
    H_CUDA(h, cudaGraphLaunch(h->graph_exec, h->st));
    h->launches_total += 1;
  }
  return GPT2_OK;
}

int gpt2_stream_kernels(const gpt2_handle* h, int64_t* n) {
  if (!h || !n) return GPT2_ERR_ARG;
  *n = h->graph_exec ? h->graph_kernels : 0;
  return GPT2_OK;
}

int gpt2_stream_end(gpt2_handle* h, int64_t* cursor_out) {
  if (!h) return GPT2_ERR_ARG;
  if (cursor_out)
    H_CUDA(h, cudaMemcpyAsync(cursor_out, h->d_cursor, sizeof(int64_t), cudaMemcpyDeviceToHost,
                              h->st));
  H_CUDA(h, cudaStreamSynchronize(h->st));
  if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
  if (h->graph) cudaGraphDestroy(h->graph);
  h->graph_exec = nullptr;
  h->graph = nullptr;
  return check_status(h);
}

int gpt2_arena_layout(const gpt2_config* cfg, int i, char* name, int name_len, int64_t* offset,
                      int64_t* n_elems, int* n_tensors) {
  if (!cfg) return fail(nullptr, GPT2_ERR_ARG, "cfg is NULL");
  const std::string bad = config_problem(*cfg);
  if (!bad.empty()) return fail(nullptr, GPT2_ERR_ARG, bad);
  gpt2_handle t;  // host-side layout only: nothing is allocated
  set_shape(&t, *cfg);
  build_layout(&t);
  if (n_tensors) *n_tensors = int(t.tensors.size());
  if (i < 0) return GPT2_OK;
  if (i >= int(t.tensors.size())) return fail(nullptr, GPT2_ERR_ARG, "tensor index out of range");
  const TensorInfo& x = t.tensors[i];
  if (name && name_len > 0) {
    const size_t n = std::min(size_t(name_len - 1), x.name.size());
    memcpy(name, x.name.data(), n);
    name[n] = 0;
  }
  if (offset) *offset = x.off;
  if (n_elems) *n_elems = x.rows * x.cols;
  return GPT2_OK;
}

int gpt2_grad_buckets(const gpt2_config* cfg, int max_ranges, int* n_ranges, int64_t* offset,
                      int64_t* count, int* bucket) {
  if (!cfg || !n_ranges) return fail(nullptr, GPT2_ERR_ARG, "NULL argument");
  const std::string bad = config_problem(*cfg);
  if (!bad.empty()) return fail(nullptr, GPT2_ERR_ARG, bad);
  gpt2_handle t;
  set_shape(&t, *cfg);
  build_layout(&t);
  const std::vector<BucketRange> r = bucket_plan(t);
  *n_ranges = int(r.size());
  if (max_ranges < int(r.size())) return GPT2_OK;  // the count only
  for (size_t k = 0; k < r.size(); ++k) {
    if (offset) offset[k] = r[k].off;
    if (count) count[k] = r[k].n;
    if (bucket) bucket[k] = r[k].b;
  }
  return GPT2_OK;
}

int gpt2_set_bucket_callback(gpt2_handle* h, gpt2_bucket_fn fn, void* user) {
  if (!h) return GPT2_ERR_ARG;
  h->bucket_fn = fn;
  h->bucket_user = user;
  return GPT2_OK;
}

int gpt2_dp_init(gpt2_handle* h, const char* id, int rank, int world) {
  if (!h || !id) return fail(h, GPT2_ERR_ARG, "NULL argument");
  if (world < 1 || rank < 0 || rank >= world) return fail(h, GPT2_ERR_ARG, "bad rank or world");
  if (h->dp_comm) return fail(h, GPT2_ERR_STATE, "dp_init: already initialised");
  if (h->graph_exec) return fail(h, GPT2_ERR_STATE, "dp_init: end the recorded stream first");
  H_CUDA(h, cudaStreamSynchronize(h->st));
  if (!h->st_comm) {
    H_CUDA(h, cudaStreamCreateWithFlags(&h->st_comm, cudaStreamNonBlocking));
    H_CUDA(h, cudaEventCreateWithFlags(&h->ev_dp, cudaEventDisableTiming));
    H_CUDA(h, cudaEventCreateWithFlags(&h->ev_dp_join, cudaEventDisableTiming));
  }
  void* comm = nullptr;
  const int rc = gpt2_internal::dp_comm_init(&comm, id, rank, world);
  if (rc) return fail(h, rc, gpt2_internal::get_error());
  h->dp_ranges.assign(h->L + 1, {});
  for (const BucketRange& r : bucket_plan(*h)) h->dp_ranges[r.b].push_back({r.off, r.n});
  h->dp_comm = comm;
  h->dp_world = world;
  h->dp_sync = true;
  return GPT2_OK;
}

int gpt2_dp_sync(gpt2_handle* h, int on) {
  if (!h) return GPT2_ERR_ARG;
  h->dp_sync = on != 0;
  return GPT2_OK;
}

int gpt2_arena(gpt2_handle* h, int which, float** ptr, int64_t* n_elems) {
  if (!h || !ptr) return fail(h, GPT2_ERR_ARG, "NULL argument");
  float* base = arena_of(h, which);
  if (!base) return fail(h, GPT2_ERR_ARG, "bad selector");
  if (which == GPT2_GRAD && h->grads_zero) {
    H_CUDA(h, cudaMemsetAsync(h->G, 0, size_t(h->n_arena) * sizeof(float), h->st));
    h->grads_zero = false;
  }
  *ptr = base;
  if (n_elems) *n_elems = h->n_arena;
  return GPT2_OK;
}

int gpt2_profile_enable(gpt2_handle* h, int enable) {
  if (!h) return GPT2_ERR_ARG;
  h->prof_on = enable != 0;
  return GPT2_OK;
}

int gpt2_profile_reset(gpt2_handle* h) {
  if (!h) return GPT2_ERR_ARG;
  H_TRY(h, prof_collect(h));
  for (auto& c : h->cats) {
    c.launches = 0;
    c.flops = c.bytes = c.ms = 0;
  }
  h->launches_total = 0;
  return GPT2_OK;
}

int gpt2_profile_read(gpt2_handle* h, int cat, int64_t* launches, double* ms, double* flops,
                      double* bytes) {
  if (!h || cat < -1 || cat >= GPT2_PROF_NCAT) return GPT2_ERR_ARG;
  H_TRY(h, prof_collect(h));
  if (cat == -1) {
    if (launches) *launches = h->launches_total;
    if (ms) *ms = 0;
    if (flops) *flops = 0;
    if (bytes) *bytes = 0;
    return GPT2_OK;
  }
  const auto& c = h->cats[cat];
  if (launches) *launches = c.launches;
  if (ms) *ms = c.ms;
  if (flops) *flops = c.flops;
  if (bytes) *bytes = c.bytes;
  return GPT2_OK;
}

int gpt2_synchronize(gpt2_handle* h) {
  if (!h) return GPT2_ERR_ARG;
  return check_status(h);
}

}  // extern "C"
