// Op-level C ABI: the tied LM head + cross-entropy alone, LayerNorm,
// attention and the dense contraction, each on caller-owned device buffers
// and a caller-provided workspace, asynchronous on the caller's stream.
//
// Sources: [ZERO] "GPT training" (Zero docs): output layer (fused projection
// + cross-entropy whose [B*T, V] logits stay out of the saved graph),
// Transformer Block (LayerNorm), Attention; [LECTURE] "Andrej Karpathy:
// reproducing GPT-2 from scratch": tied head over the padded vocabulary;
// [CS336] "CS336 from scratch — pretraining" §1: cross-entropy with the row
// maximum subtracted.

#include <algorithm>
#include <string>

#include "attn_internal.h"
#include "kernels.h"

using gpt2_internal::set_error;

namespace {

__device__ int g_op_error;  // bounded-wait timeouts of op-level launches

}  // namespace

int* device_error_word() {
  static int* addr[64] = {nullptr};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_op_error) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
  }
  return addr[dev];
}

extern "C" {

int gpt2_lmhead_ce_workspace(int M, int C, int Vp, int dtype, size_t* bytes) {
  if (!bytes || M < 1 || C < 1 || Vp < 1 || (dtype != GPT2_BF16 && dtype != GPT2_F32))
    return GPT2_ERR_ARG;
  *bytes = lmhead_workspace(M, C, Vp, dtype == GPT2_BF16) + 2 * ((size_t(M) * 4 + 255) / 256 * 256);
  return GPT2_OK;
}

int gpt2_lmhead_ce(const void* hidden, const void* W, const int32_t* y, int M, int C, int Vp,
                   int V, int dtype, float grad_scale, float* d_loss, float* d_lse, void* d_dh,
                   float* d_dw, void* workspace, size_t workspace_bytes, void* stream) {
  if (!hidden || !W || !y || !d_loss || M < 1 || C < 1 || Vp < V || V < 1 ||
      (dtype != GPT2_BF16 && dtype != GPT2_F32)) {
    set_error("lmhead_ce: bad arguments");
    return GPT2_ERR_ARG;
  }
  size_t need = 0;
  gpt2_lmhead_ce_workspace(M, C, Vp, dtype, &need);
  if (!workspace || workspace_bytes < need) {
    set_error("lmhead_ce: workspace too small");
    return GPT2_ERR_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bf = dtype == GPT2_BF16;
  char* w = static_cast<char*>(workspace);
  const size_t rows = (size_t(M) * 4 + 255) / 256 * 256;
  float* lse = d_lse ? d_lse : reinterpret_cast<float*>(w);
  float* rl = reinterpret_cast<float*>(w + rows);
  void* lw = w + 2 * rows;
  const size_t lw_bytes = workspace_bytes - 2 * rows;
  int rc = lmhead_fwd(hidden, W, y, M, C, Vp, bf, lse, rl, lw, lw_bytes, st);
  if (rc) return rc;
  if (d_dh || d_dw) {
    rc = lmhead_bwd(hidden, W, y, lse, M, C, Vp, bf, grad_scale / float(M), d_dh, d_dw, 1, lw,
                    lw_bytes, st);
    if (rc) return rc;
  }
  return launch_mean(rl, M, d_loss, st);
}

int gpt2_layernorm_fwd(const float* x, const float* gamma, const float* beta, int64_t M, int C,
                       float eps, void* y, int y_dtype, float* mean, float* rstd, void* stream) {
  if (!x || !gamma || !beta || !y || M < 1 || C < 1 || C > 1024) {
    set_error("layernorm_fwd: bad arguments");
    return GPT2_ERR_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (y_dtype == GPT2_BF16)
    return launch_layernorm_fwd<bf16>(x, gamma, beta, static_cast<bf16*>(y), mean, rstd, M, C, eps, st);
  if (y_dtype == GPT2_F32)
    return launch_layernorm_fwd<float>(x, gamma, beta, static_cast<float*>(y), mean, rstd, M, C, eps, st);
  set_error("layernorm_fwd: bad dtype");
  return GPT2_ERR_ARG;
}

int gpt2_layernorm_bwd_workspace(int64_t M, int C, size_t* bytes) {
  if (!bytes || M < 1 || C < 1) return GPT2_ERR_ARG;
  *bytes = layernorm_bwd_workspace(M, C);
  return GPT2_OK;
}

int gpt2_layernorm_bwd(const void* dy, int dy_dtype, const float* x, const float* mean,
                       const float* rstd, const float* gamma, int64_t M, int C, float* dx,
                       float* dgamma, float* dbeta, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!dy || !x || !mean || !rstd || !gamma || !dx || !dgamma || !dbeta || M < 1 || C < 1 ||
      C > 1024 || !workspace || workspace_bytes < layernorm_bwd_workspace(M, C)) {
    set_error("layernorm_bwd: bad arguments or workspace too small");
    return GPT2_ERR_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  if (dy_dtype == GPT2_BF16)
    return launch_layernorm_bwd<bf16, bf16>(static_cast<const bf16*>(dy), x, mean, rstd, gamma, M,
                                            C, dx, nullptr, dgamma, dbeta, nullptr, 1, ws, st);
  if (dy_dtype == GPT2_F32)
    return launch_layernorm_bwd<float, float>(static_cast<const float*>(dy), x, mean, rstd, gamma,
                                              M, C, dx, nullptr, dgamma, dbeta, nullptr, 1, ws, st);
  set_error("layernorm_bwd: bad dtype");
  return GPT2_ERR_ARG;
}

int gpt2_attention_fwd(const void* qkv, int dtype, int B, int T, int C, int H, void* out,
                       float* lse, void* stream) {
  if (!qkv || !out || !lse || B < 1 || T < 1 || H < 1 || C % H) {
    set_error("attention_fwd: bad arguments");
    return GPT2_ERR_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == GPT2_BF16)
    return launch_attn_fwd<bf16>(static_cast<const bf16*>(qkv), B, T, C, H, static_cast<bf16*>(out), lse, st);
  if (dtype == GPT2_F32)
    return launch_attn_fwd<float>(static_cast<const float*>(qkv), B, T, C, H, static_cast<float*>(out), lse, st);
  set_error("attention_fwd: bad dtype");
  return GPT2_ERR_ARG;
}

int gpt2_attention_bwd_workspace(int B, int T, int C, int H, int dtype, size_t* bytes) {
  if (!bytes || B < 1 || T < 1 || H < 1) return GPT2_ERR_ARG;
  *bytes = attn_bwd_workspace_total(B, T, C, H, dtype == GPT2_BF16);
  return GPT2_OK;
}

int gpt2_attention_bwd(const void* dout, const void* qkv, const void* out, const float* lse,
                       int dtype, int B, int T, int C, int H, void* dqkv, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (!dout || !qkv || !out || !lse || !dqkv || B < 1 || T < 1 || H < 1 || C % H || !workspace ||
      workspace_bytes < attn_bwd_workspace_total(B, T, C, H, dtype == GPT2_BF16)) {
    set_error("attention_bwd: bad arguments or workspace too small");
    return GPT2_ERR_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  if (dtype == GPT2_BF16) {
    // the score-gradient buffer follows Delta when the workspace holds one
    const size_t delta = (attn_bwd_workspace(B, T, H) + 1023) / 1024 * 1024;
    bf16* ds = attn_bwd_workspace_total(B, T, C, H, true) > attn_bwd_workspace(B, T, H)
                   ? reinterpret_cast<bf16*>(static_cast<char*>(workspace) + delta)
                   : nullptr;
    return launch_attn_bwd_ds(static_cast<const bf16*>(dout), static_cast<const bf16*>(qkv),
                              static_cast<const bf16*>(out), lse, B, T, C, H,
                              static_cast<bf16*>(dqkv), ws, ds, st);
  }
  if (dtype == GPT2_F32)
    return launch_attn_bwd<float>(static_cast<const float*>(dout), static_cast<const float*>(qkv),
                                  static_cast<const float*>(out), lse, B, T, C, H,
                                  static_cast<float*>(dqkv), ws, st);
  set_error("attention_bwd: bad dtype");
  return GPT2_ERR_ARG;
}

int gpt2_matmul_workspace(int M, int N, int K, size_t* bytes) {
  if (!bytes || M < 1 || N < 1 || K < 1) return GPT2_ERR_ARG;
  *bytes = gemm_workspace_bytes(M, N, K);
  return GPT2_OK;
}

int gpt2_matmul(const void* A, int a_kmajor, int64_t lda, const void* B, int b_kmajor, int64_t ldb,
                int dtype, int M, int N, int K, float alpha, int accumulate, void* D, int d_dtype,
                int64_t ldd, void* workspace, size_t workspace_bytes, void* stream) {
  if (!A || !B || !D || M < 1 || N < 1 || K < 1 || (dtype != GPT2_BF16 && dtype != GPT2_F32) ||
      (accumulate && d_dtype != GPT2_F32) || ldd < N) {
    set_error("matmul: bad arguments");
    return GPT2_ERR_ARG;
  }
  EpiParams e;
  e.kind = accumulate ? EPI_ACC : EPI_STORE;
  e.out = D;
  e.ldo = ldd;
  e.alpha = alpha;
  e.accumulate = accumulate;
  e.out_bf16 = d_dtype == GPT2_BF16;
  GemmArgs g{A, a_kmajor ? 1 : 0, lda, B, b_kmajor ? 1 : 0, ldb, dtype == GPT2_BF16, M, N, K, e,
             static_cast<float*>(workspace), workspace_bytes};
  return gemm_launch(g, static_cast<cudaStream_t>(stream));
}

int gpt2_linear(int epi, const void* x, const void* w, int w_kn, const float* bias,
                const void* in, void* out, void* out2, int M, int N, int K, int dtype,
                void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !w || !out || M < 1 || N < 1 || K < 1 || (dtype != GPT2_BF16 && dtype != GPT2_F32)) {
    set_error("linear: bad arguments");
    return GPT2_ERR_ARG;
  }
  const int bf = dtype == GPT2_BF16;
  EpiParams e;
  e.ldo = N;
  e.out_bf16 = bf;
  switch (epi) {
    case GPT2_LINEAR_BIAS:
      e.kind = EPI_STORE;
      e.out = out;
      e.bias = bias;
      break;
    case GPT2_LINEAR_BIAS_GELU:
      if (!bias || !out2) {
        set_error("linear: bias+GELU needs bias and the pre-activation output");
        return GPT2_ERR_ARG;
      }
      e.kind = EPI_GELU;
      e.out = out2;  // pre-activation
      e.out2 = out;  // GELU of it
      e.bias = bias;
      break;
    case GPT2_LINEAR_RESIDUAL:
      if (!in) {
        set_error("linear: the residual epilogue needs its input");
        return GPT2_ERR_ARG;
      }
      e.kind = EPI_RESID;
      e.rin = static_cast<const float*>(in);
      e.rout = static_cast<float*>(out);
      e.bias = bias;
      e.out_bf16 = 0;
      break;
    case GPT2_LINEAR_GELU_BWD:
      if (!in || bias) {
        set_error("linear: GELU backward needs the pre-activation and no bias");
        return GPT2_ERR_ARG;
      }
      e.kind = EPI_GELU_BWD;
      e.out = out;
      e.aux = in;
      break;
    default:
      set_error("linear: unknown epilogue");
      return GPT2_ERR_ARG;
  }
  GemmArgs g{x, 1, K, w, w_kn ? 0 : 1, w_kn ? int64_t(N) : int64_t(K), bf, M, N, K, e,
             static_cast<float*>(workspace), workspace_bytes};
  return gemm_launch(g, static_cast<cudaStream_t>(stream));
}

int gpt2_sample(const float* logits, int64_t ld, int B, int V, float temperature, int top_k,
                float top_p, const float* uniform, int32_t* out, int64_t out_stride,
                void* stream) {
  const bool greedy = temperature == 0.f || top_k == 1;
  if (!logits || !out || B < 1 || V < 1 || V > kSampleMaxVocab || ld < V || out_stride < 1 ||
      !(temperature >= 0.f) || top_k < 0 || !(top_p > 0.f && top_p <= 1.f) ||
      (!greedy && !uniform)) {
    set_error("sample: bad arguments");
    return GPT2_ERR_ARG;
  }
  return launch_sample(logits, ld, B, V, temperature, top_k, top_p, uniform, out, out_stride,
                       static_cast<cudaStream_t>(stream));
}

int gpt2_launch_count(int64_t* n) {
  if (!n) return GPT2_ERR_ARG;
  *n = gpt2_internal::launches();
  return GPT2_OK;
}

int gpt2_device_error(int* code) {
  if (!code) return GPT2_ERR_ARG;
  int* w = device_error_word();
  if (!w) return GPT2_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GPT2_ERR_CUDA;
  int z = 0;
  cudaMemcpy(w, &z, sizeof(int), cudaMemcpyHostToDevice);
  *code = v ? GPT2_ERR_TIMEOUT : GPT2_OK;
  return GPT2_OK;
}

}  // extern "C"
