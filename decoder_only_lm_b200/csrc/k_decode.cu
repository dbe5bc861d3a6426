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
                                int pos0, int Tc, T* __restrict__ kc, T* __restrict__ vc) {
  const int D = C / H;
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

template <typename T>
__device__ __forceinline__ float ld_f(const T* p) {
  return to_f32<T>(*p);
}

// One CTA per (head h, sequence b): the query of the new token (its qkv row)
// against cache positions 0 .. L-1:  s_j = q.k_j / sqrt(D), p = softmax(s),
// out = sum_j p_j v_j.  Scores in shared memory; fixed-order reductions.
template <typename T>
__global__ void __launch_bounds__(kDecThreads) attn_decode_kernel(
    const T* __restrict__ qkv, const T* __restrict__ kc, const T* __restrict__ vc, int C, int H,
    int Tc, int L, T* __restrict__ out) {
  __shared__ float q[256];
  __shared__ float s[kDecMaxT];
  __shared__ float red[kDecThreads / 32];
  __shared__ float part[kDecThreads];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int D = C / H;
  const float scale = rsqrtf(float(D));
  const T* qr = qkv + int64_t(b) * 3 * C + h * D;
  for (int d = tid; d < D; d += kDecThreads) q[d] = ld_f(qr + d) * scale;
  __syncthreads();
  const T* K = kc + (int64_t(b) * H + h) * Tc * D;
  const T* Vv = vc + (int64_t(b) * H + h) * Tc * D;
  float mx = -INFINITY;
  for (int j = tid; j < L; j += kDecThreads) {
    const T* kr = K + int64_t(j) * D;
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = fmaf(q[d], ld_f(kr + d), acc);
    s[j] = acc;
    mx = fmaxf(mx, acc);
  }
  mx = warp_max(mx);
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < kDecThreads / 32; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = tid; j < L; j += kDecThreads) {
    const float e = expf(s[j] - mx);
    s[j] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  if ((tid & 31) == 0) red[tid >> 5] = sum;
  __syncthreads();
  sum = red[0];
  for (int w = 1; w < kDecThreads / 32; ++w) sum += red[w];
  // out[d] = sum_j p_j v_j[d]: thread (d, slice) sums the positions j = slice mod S
  const int S = kDecThreads / D;  // position slices (D divides 128)
  const int d = tid % D, sl = tid / D;
  float acc = 0.f;
  if (sl < S)
    for (int j = sl; j < L; j += S) acc = fmaf(s[j], ld_f(Vv + int64_t(j) * D + d), acc);
  part[tid] = acc;
  __syncthreads();
  if (tid < D) {
    float o = 0.f;
    for (int k = 0; k < S; ++k) o += part[k * D + tid];
    out[int64_t(b) * C + h * D + tid] = from_f32<T>(o / sum);
  }
}

}  // namespace

template <typename T>
int launch_kv_store(const T* qkv, int B, int Tn, int C, int H, int pos0, int Tc, T* kc, T* vc,
                    cudaStream_t st) {
  const int64_t n = int64_t(B) * Tn * C;
  const int blocks = int(std::min<int64_t>(cdiv64(n, 256), 4 * int64_t(gpt2_internal::sm_count())));
  kv_store_kernel<T><<<blocks, 256, 0, st>>>(qkv, B, Tn, C, H, pos0, Tc, kc, vc);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template <typename T>
int launch_attn_decode(const T* qkv, const T* kc, const T* vc, int B, int C, int H, int Tc, int L,
                       T* out, cudaStream_t st) {
  const int D = C / H;
  if (L < 1 || L > kDecMaxT || L > Tc || D > 128 || kDecThreads % D != 0) {
    gpt2_internal::set_error("attention decode: cache length or head size not supported");
    return GPT2_ERR_ARG;
  }
  attn_decode_kernel<T><<<dim3(H, B), kDecThreads, 0, st>>>(qkv, kc, vc, C, H, Tc, L, out);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template int launch_kv_store<float>(const float*, int, int, int, int, int, int, float*, float*,
                                    cudaStream_t);
template int launch_kv_store<bf16>(const bf16*, int, int, int, int, int, int, bf16*, bf16*,
                                   cudaStream_t);
template int launch_attn_decode<float>(const float*, const float*, const float*, int, int, int, int,
                                       int, float*, cudaStream_t);
template int launch_attn_decode<bf16>(const bf16*, const bf16*, const bf16*, int, int, int, int,
                                      int, bf16*, cudaStream_t);
