// Incremental decoding with a key/value cache: the keys and values of every
// position already seen are kept per layer, so a new token needs only its own
// row through the block and one query's attention over the cache.
//
// Sources: [CS336] "CS336 from scratch — pretraining" §5 text generation
// (the loop that recomputes the whole window, and the note that a KV cache
// reuses the history's computation); [ZERO] "GPT training", Attention
// (scores q.k / sqrt(D) over the positions j <= i, softmax, weighted sum of v).
//
// Cache layout (per layer, activation type T): K and V as [B, H, Tc, D], the
// row of position t of head h of sequence b at ((b H + h) Tc + t) D.

#include "kernels.h"

namespace {

// cache[b, h, pos0 + t, :] = the k (and v) of qkv row (b, t)
template <typename T>
__global__ void kv_store_kernel(const T* __restrict__ qkv, int B, int Tn, int C, int H,
                                int pos0, int Tc, T* __restrict__ kc, T* __restrict__ vc,
                                const int* __restrict__ d_step) {
  const int D = C / H;
  if (d_step) pos0 += *d_step;
  const int64_t n = int64_t(B) * Tn * C;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int c = int(e % C);
    const int64_t bt = e / C;
    const int t = int(bt % Tn), b = int(bt / Tn);
    const int h = c / D, d = c % D;
    const int64_t dst = ((int64_t(b) * H + h) * Tc + pos0 + t) * D + d;
    kc[dst] = qkv[bt * 3 * C + C + c];
    vc[dst] = qkv[bt * 3 * C + 2 * C + c];
  }
}

constexpr int kDecThreads = 128;
constexpr int kDecMaxT = 4096;  // cached positions per launch (shared scores)

// 16-byte vector of E elements of T, widened to fp32
template <typename T>
struct Vec16;
template <>
struct Vec16<float> {
  static constexpr int E = 4;
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
};
template <>
struct Vec16<bf16> {
  static constexpr int E = 8;
  static __device__ __forceinline__ void load(const bf16* p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    }
  }
};

// One CTA per (head h, sequence b): the query of the new token (its qkv row)
// against cache positions 0 .. L-1:  s_j = q.k_j / sqrt(D), p = softmax(s),
// out = sum_j p_j v_j.  A row of K or V (D elements) is read by a group of
// G = D / E lanes with 16-byte loads, so a warp covers 32 / G whole rows per
// instruction; scores go to shared memory; all reductions in a fixed order.
template <typename T>
__global__ void __launch_bounds__(kDecThreads) attn_decode_kernel(
    const T* __restrict__ qkv, const T* __restrict__ kc, const T* __restrict__ vc, int C, int H,
    int Tc, int L, T* __restrict__ out, const int* __restrict__ d_step) {
  constexpr int E = Vec16<T>::E;
  constexpr int NW = kDecThreads / 32;
  if (d_step) L += *d_step;
  __shared__ float s[kDecMaxT];
  __shared__ float red[NW];
  __shared__ float part[NW * 32 * E];  // [warp][lane] partial outputs
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int D = C / H, G = D / E, RPW = 32 / G;
  const int r = lane / G, c = lane % G;  // row within the warp's rows, 16-byte chunk
  const float scale = rsqrtf(float(D));
  float q[E];
  Vec16<T>::load(qkv + int64_t(b) * 3 * C + h * D + c * E, q);
#pragma unroll
  for (int k = 0; k < E; ++k) q[k] *= scale;
  const T* K = kc + (int64_t(b) * H + h) * Tc * D;
  const T* Vv = vc + (int64_t(b) * H + h) * Tc * D;
  // scores: rows j = (NW * i + warp) * RPW + r
  float mx = -INFINITY;
  for (int j0 = warp * RPW; j0 < L; j0 += NW * RPW) {
    const int j = j0 + r;
    float acc = 0.f;
    if (j < L) {
      float kv[E];
      Vec16<T>::load(K + int64_t(j) * D + c * E, kv);
#pragma unroll
      for (int k = 0; k < E; ++k) acc = fmaf(q[k], kv[k], acc);
    }
    for (int o = G >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (j < L) {
      if (c == 0) s[j] = acc;
      mx = fmaxf(mx, acc);
    }
  }
  mx = warp_max(mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < NW; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = tid; j < L; j += kDecThreads) {
    const float e = expf(s[j] - mx);
    s[j] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  if (lane == 0) red[warp] = sum;
  __syncthreads();  // also: every s[j] is final
  sum = red[0];
  for (int w = 1; w < NW; ++w) sum += red[w];
  // out[c E + k] = sum_j p_j v_j[c E + k], each lane over its rows
  float o[E];
#pragma unroll
  for (int k = 0; k < E; ++k) o[k] = 0.f;
  for (int j0 = warp * RPW; j0 < L; j0 += NW * RPW) {
    const int j = j0 + r;
    if (j < L) {
      float vv[E];
      Vec16<T>::load(Vv + int64_t(j) * D + c * E, vv);
      const float pj = s[j];
#pragma unroll
      for (int k = 0; k < E; ++k) o[k] = fmaf(pj, vv[k], o[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < E; ++k) part[(warp * 32 + lane) * E + k] = o[k];
  __syncthreads();
  // thread d: the RPW row groups of every warp, in order
  for (int d = tid; d < D; d += kDecThreads) {
    const int cc = d / E, k = d % E;
    float acc = 0.f;
    for (int w = 0; w < NW; ++w)
      for (int rr = 0; rr < RPW; ++rr) acc += part[(w * 32 + rr * G + cc) * E + k];
    out[int64_t(b) * C + h * D + d] = from_f32<T>(acc / sum);
  }
}

__global__ void gen_tokens_kernel(const int32_t* __restrict__ tokens, int64_t ld, int B,
                                  int64_t col0, const int* __restrict__ d_step,
                                  int32_t* __restrict__ x, int32_t* __restrict__ y) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) x[b] = y[b] = tokens[int64_t(b) * ld + col0 + *d_step];
}
__global__ void step_add_kernel(int* d_step) { *d_step += 1; }

}  // namespace

int launch_gen_tokens(const int32_t* tokens, int64_t ld, int B, int64_t col0, const int* d_step,
                      int32_t* x, int32_t* y, cudaStream_t st) {
  gen_tokens_kernel<<<(B + 127) / 128, 128, 0, st>>>(tokens, ld, B, col0, d_step, x, y);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
int launch_step_add(int* d_step, cudaStream_t st) {
  step_add_kernel<<<1, 1, 0, st>>>(d_step);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template <typename T>
int launch_kv_store(const T* qkv, int B, int Tn, int C, int H, int pos0, int Tc, T* kc, T* vc,
                    cudaStream_t st, const int* d_step) {
  const int64_t n = int64_t(B) * Tn * C;
  const int blocks = int(std::min<int64_t>(cdiv64(n, 256), 4 * int64_t(gpt2_internal::sm_count())));
  kv_store_kernel<T><<<blocks, 256, 0, st>>>(qkv, B, Tn, C, H, pos0, Tc, kc, vc, d_step);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template <typename T>
int launch_attn_decode(const T* qkv, const T* kc, const T* vc, int B, int C, int H, int Tc, int L,
                       T* out, cudaStream_t st, const int* d_step) {
  const int D = C / H;
  constexpr int E = 16 / int(sizeof(T));
  // with d_step the caller bounds L + *d_step by Tc (and kDecMaxT)
  if (L < 1 || L > kDecMaxT || L > Tc || D % E != 0 || D / E > 32 || 32 % (D / E) != 0 ||
      (C % E) != 0) {
    gpt2_internal::set_error("attention decode: cache length or head size not supported");
    return GPT2_ERR_ARG;
  }
  attn_decode_kernel<T><<<dim3(H, B), kDecThreads, 0, st>>>(qkv, kc, vc, C, H, Tc, L, out, d_step);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template int launch_kv_store<float>(const float*, int, int, int, int, int, int, float*, float*,
                                    cudaStream_t, const int*);
template int launch_kv_store<bf16>(const bf16*, int, int, int, int, int, int, bf16*, bf16*,
                                   cudaStream_t, const int*);
template int launch_attn_decode<float>(const float*, const float*, const float*, int, int, int, int,
                                       int, float*, cudaStream_t, const int*);
template int launch_attn_decode<bf16>(const bf16*, const bf16*, const bf16*, int, int, int, int,
                                      int, bf16*, cudaStream_t, const int*);
