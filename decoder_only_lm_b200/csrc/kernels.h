// Host-side launchers of the library's kernels (internal, C++ linkage).
#pragma once

#include <vector>

#include "common.cuh"

// ---------------------------------------------------------------- GEMM
// D[m,n] = epilogue(sum_k A(m,k) B(n,k)).
// A(m,k) = A[m*lda+k] (K-major) or A[k*lda+m] (MN-major); B(n,k) likewise.
enum EpiKind {
  EPI_STORE = 0,     // out = alpha*acc (+ bias[n])                  -> out type
  EPI_GELU = 1,      // u = acc + bias -> out; g = gelu(u) -> out2    (act type)
  EPI_RESID = 2,     // rout = rin + acc + bias                       (fp32)
  EPI_ACC = 3,       // out = (accumulate ? out : 0) + alpha*acc      (fp32)
  EPI_GELU_BWD = 4,  // out = acc * gelu'(aux[m,n])                   (act type)
  EPI_CE_GRAD = 5,   // out = scale*(exp(acc - lse[m]) - [n == tgt[m]]) (act type)
  EPI_LSE_PARTIAL = 6,  // per row and column tile: max and sum of exp over the tile's
                        // columns -> part_max/part_sum[m*part_ld + tile]; z[m, tgt[m]] ->
                        // tgt_logit[m] (tensor-core path only)
};

struct EpiParams {
  int kind = EPI_STORE;
  void* out = nullptr;
  int64_t ldo = 0;
  int out_bf16 = 0;        // element type of out / out2 / aux
  void* out2 = nullptr;
  const float* bias = nullptr;
  const float* rin = nullptr;
  float* rout = nullptr;
  const void* aux = nullptr;
  float alpha = 1.f;
  int accumulate = 0;
  const int32_t* tgt = nullptr;
  const float* lse = nullptr;
  float ce_scale = 0.f;
  float* part_max = nullptr;
  float* part_sum = nullptr;
  float* tgt_logit = nullptr;
  int part_ld = 0;
};

struct GemmArgs {
  const void* A; int a_kmajor; int64_t lda;
  const void* B; int b_kmajor; int64_t ldb;
  int bf16_in;  // A and B are bf16 (else fp32)
  int M, N, K;
  EpiParams ep;
  float* ws; size_t ws_bytes;  // split-K partial sums (EPI_ACC only)
};

size_t gemm_workspace_bytes(int M, int N, int K);
int gemm_launch(const GemmArgs& g, cudaStream_t st);

// ---------------------------------------------------------------- elementwise / rows
int launch_slice_batch(const uint16_t* s, int64_t off, int64_t n, int32_t* x, int32_t* y,
                       cudaStream_t st);
// x, y from the window at the device cursor *cur of a len-token stream (window_bad if outside)
int launch_slice_batch_cursor(const uint16_t* s, int64_t len, const int64_t* cur, int64_t n,
                              int32_t* x, int32_t* y, DevStatus* status, cudaStream_t st);
int launch_advance_cursor(int64_t* cur, int64_t stride, cudaStream_t st);
// positions p0 .. p0 + T - 1 with p0 = pos0 + (*d_step when d_step is given:
// a step of incremental decoding replayed from a graph)
int launch_embed_fwd(const int32_t* x, const int32_t* y, const float* wte, const float* wpe,
                     int B, int T, int C, int V, float* out, DevStatus* status, cudaStream_t st,
                     int pos0 = 0, const int* d_step = nullptr);
// dwte[x_m] += dh[m] (deterministic: sort by id, segmented sums); dwpe[t] (+)= sum_b dh[b,t].
size_t embed_bwd_workspace(int64_t M, int C);
int launch_embed_bwd(const int32_t* x, const float* dh, int B, int T, int C, int V, float* dwte,
                     float* dwpe, int wpe_accumulate, void* ws, cudaStream_t st);
template <typename OutT>
int launch_layernorm_fwd(const float* x, const float* g, const float* b, OutT* y, float* mean,
                         float* rstd, int64_t M, int C, float eps, cudaStream_t st);
// A fixed-order sum of the `parts` rows of the fp32 matrix p [parts, n]:
// column c (+)= into out0[c] (c < split), out1[c - split] (c < 2 split) or
// out2[c - 2 split].  The backward pass collects these (LayerNorm and bias
// gradient partials, each in a buffer of its own) and runs them in one launch
// at its end: only the optimizer reads the vectors they produce.
struct RowSum {
  const float* p;
  float *out0, *out1, *out2;
  int parts, n, split, accumulate;
};
int launch_row_sums(const RowSum* sums, int count, cudaStream_t st);
size_t layernorm_bwd_workspace(int64_t M, int C);
// dx (+)= LN backward; dg, db (+)= dgamma, dbeta; dsum (nullable) (+)= column
// sums of the updated dx.  With `defer`, the final sum of the partial rows in
// ws is appended there instead of launched (ws must then stay untouched until
// launch_row_sums runs the list).
template <typename DyT, typename CopyT>
int launch_layernorm_bwd(const DyT* dy, const float* x, const float* mean, const float* rstd,
                         const float* g, int64_t M, int C, float* dx, CopyT* dx_copy,
                         float* dg, float* db, float* dsum, int accumulate, float* ws,
                         cudaStream_t st, std::vector<RowSum>* defer = nullptr);
size_t colsum_workspace(int64_t M, int N);
template <typename InT>
int launch_colsum(const InT* in, int64_t M, int N, float* out, int accumulate, float* ws,
                  cudaStream_t st, std::vector<RowSum>* defer = nullptr);
// gradient norm (deterministic two-stage, double accumulation) into *norm (device)
size_t gradnorm_workspace();
int launch_gradnorm(const float* g, int64_t n, double* ws, float* norm, cudaStream_t st);
// lr_dev (nullable): learning rate read on the device instead of lr
int launch_clip_adamw(float* p, const float* g, float* m, float* v, bf16* pb, int64_t n,
                      int64_t n_decay, const float* norm, DevStatus* status, float lr,
                      const float* lr_dev, float b1, float b2, float eps, float wd, float max_norm,
                      cudaStream_t st);
int launch_to_bf16(const float* src, bf16* dst, int64_t n, cudaStream_t st);
int launch_fill(float* p, float v, int64_t n, cudaStream_t st);
// cross-entropy over a chunk of logits rows z [rows, Vp] (fp32)
int launch_ce_rows_fwd(const float* z, const int32_t* y, int rows, int Vp, float* lse,
                       float* row_loss, cudaStream_t st);
template <typename OutT>
int launch_ce_rows_bwd(const float* z, const float* lse, const int32_t* y, int rows, int Vp,
                       float scale, OutT* dz, cudaStream_t st);
int launch_mean(const float* v, int64_t n, float* out, cudaStream_t st);

// ---------------------------------------------------------------- KV-cache decoding
// K, V caches per layer: [B, H, Tc, D] of the activation type.  With d_step
// the position (and the attention length) is offset by *d_step on the device,
// so one recorded decoding step can be replayed for every position.
template <typename T>
int launch_kv_store(const T* qkv, int B, int Tn, int C, int H, int pos0, int Tc, T* kc, T* vc,
                    cudaStream_t st, const int* d_step = nullptr);
// out[b, h*D .. ] = attention of the single query row b of qkv [B, 3C] over
// cache positions 0 .. L-1 (L <= Tc, L <= 4096; a head row of D elements is
// G = D * sizeof(T) / 16 sixteen-byte vectors, G dividing 32)
template <typename T>
int launch_attn_decode(const T* qkv, const T* kc, const T* vc, int B, int C, int H, int Tc, int L,
                       T* out, cudaStream_t st, const int* d_step = nullptr);
// x[b] = y[b] = tokens[b * ld + col0 + *d_step] (the token a replayed decoding step reads)
int launch_gen_tokens(const int32_t* tokens, int64_t ld, int B, int64_t col0, const int* d_step,
                      int32_t* x, int32_t* y, cudaStream_t st);
int launch_step_add(int* d_step, cudaStream_t st);  // *d_step += 1

// ---------------------------------------------------------------- sampling
// next token of each of B rows of fp32 logits (row stride ld, first V columns):
// temperature (0 = greedy), top_k (0 = off), top_p (1 = off), uniform[b] in
// [0, 1); out[b * out_stride] (int32).  V <= kSampleMaxVocab (one row in
// shared memory, ids in 16 bits).
constexpr int kSampleMaxVocab = 53248;
size_t sample_max_vocab();
// With d_step: uniform + *d_step * u_step and out + *d_step * out_step.
int launch_sample(const float* logits, int64_t ld, int B, int V, float temperature, int top_k,
                  float top_p, const float* uniform, int32_t* out, int64_t out_stride,
                  cudaStream_t st, const int* d_step = nullptr, int64_t u_step = 0,
                  int64_t out_step = 0);

// ---------------------------------------------------------------- attention
template <typename T>
int launch_attn_fwd(const T* qkv, int B, int Tn, int C, int H, T* out, float* lse,
                    cudaStream_t st);
size_t attn_bwd_workspace(int B, int Tn, int H);
template <typename T>
int launch_attn_bwd(const T* dout, const T* qkv, const T* out, const float* lse, int B, int Tn,
                    int C, int H, T* dqkv, float* ws, cudaStream_t st);

// ---------------------------------------------------------------- tied LM head + CE
// Forward: lse[m] = logsumexp_v (h[m] . W[v]) over all Vp rows of W,
// row_loss[m] = lse[m] - h[m] . W[y[m]].  Backward: with dz = scale (softmax -
// onehot(y)): dh = dz W (overwritten), dW (+)= dz^T h.  dz exists only as a
// bounded ring of row-chunk buffers in the workspace (never the whole [M, Vp]
// once M is above one chunk).
size_t lmhead_workspace(int M, int C, int Vp, int bf16);
int lmhead_fwd(const void* h, const void* W, const int32_t* y, int M, int C, int Vp, int bf16,
               float* lse, float* row_loss, void* ws, size_t ws_bytes, cudaStream_t st);
// With side != nullptr the dW GEMM of each chunk runs on that stream (its own
// split-K workspace side_ws of ws-sized need), forked after the chunk's dz
// (event e_fork); e_join[b] is recorded after the dW GEMM that read chunk
// buffer b, and st waits on it before buffer b is rewritten and at the end.
struct LmSide {
  cudaStream_t st = nullptr;
  cudaEvent_t e_fork = nullptr, e_join[2] = {nullptr, nullptr};
  float* ws = nullptr;
  size_t ws_bytes = 0;
};
int lmhead_bwd(const void* h, const void* W, const int32_t* y, const float* lse, int M, int C,
               int Vp, int bf16, float scale, void* dh, float* dW, int dw_accumulate, void* ws,
               size_t ws_bytes, cudaStream_t st, const LmSide* side = nullptr);
bool gemm_tc_supported(const GemmArgs& g);

// device error word of the op-level calls (bounded waits)
int* device_error_word();
