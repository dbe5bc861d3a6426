// Next-token sampling over rows of logits: temperature, top-k, top-p and the
// draw, with the uniform numbers passed in.
//
// Sources: [CS336] "CS336 from scratch — pretraining" §5 text generation
// (the last position's logits divided by the temperature before the softmax,
// temperature 0 = greedy; top-p keeps the smallest set of most probable tokens
// whose cumulative probability reaches p, the token that crosses p included);
// [LECTURE] top-k (the draw restricted to the k highest-scoring tokens).
//
// One CTA of 1024 threads per row; the row's V values live in shared memory
// (first the logits, then the probabilities).  Every choice is exact and
// deterministic:
//   - probabilities p_i = exp((z_i - max z) / T) in fp32, each computed once;
//     the weight of id i is the integer w_i = rint(p_i * 2^36), so every
//     cumulative probability is an exact integer sum, whatever the order;
//   - ids are ordered by the 48-bit key (bits of p_i) << 16 | (0xFFFF - i):
//     probability first, the smaller id first among equal probabilities (all
//     keys are distinct);
//   - the top-k cut (the k-th largest key) and the top-p cut (the key at
//     which the weight summed from the top first reaches top_p times the
//     top-k weight) are found by bisection over the key space (at most 48
//     steps, one block reduction each); every thread keeps a bit mask of its
//     ids whose key is still inside the bisection interval and the count and
//     weight of its ids above it, so each step visits only the ids in play;
//   - the draw walks the kept ids in increasing id order and returns the
//     first at which the running weight exceeds u * (kept weight).

#include "kernels.h"

namespace {

constexpr int kSampleThreads = 1024;
constexpr int kSampleWarps = kSampleThreads / 32;

// ordering keys: logits (any sign) for the greedy choice, probabilities (>= 0)
__device__ __forceinline__ uint64_t logit_key(float z, int i) {
  const uint32_t b = __float_as_uint(z);
  const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (uint64_t(ord) << 16) | uint64_t(0xFFFF - i);
}
__device__ __forceinline__ uint64_t prob_key(float p, int i) {
  return (uint64_t(__float_as_uint(p)) << 16) | uint64_t(0xFFFF - i);
}

// Block reductions in a fixed order: a butterfly inside each warp (every lane
// ends with the same bits), then warp 0 over the 32 warp values.
template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, T* sh, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  if (warp == 0) {
    T w = sh[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w = op(w, __shfl_xor_sync(0xffffffffu, w, o));
    if (lane == 0) sh[kSampleWarps] = w;
  }
  __syncthreads();
  const T r = sh[kSampleWarps];
  __syncthreads();  // sh is reused by the next reduction
  return r;
}

// Two sums in one pass (same fixed order as block_reduce).
__device__ __forceinline__ void block_sum2(uint64_t& a, uint64_t& c, uint64_t* sh_a,
                                           uint64_t* sh_c) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  if (lane == 0) {
    sh_a[warp] = a;
    sh_c[warp] = c;
  }
  __syncthreads();
  if (warp == 0) {
    uint64_t x = sh_a[lane], y = sh_c[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      x += __shfl_xor_sync(0xffffffffu, x, o);
      y += __shfl_xor_sync(0xffffffffu, y, o);
    }
    if (lane == 0) {
      sh_a[kSampleWarps] = x;
      sh_c[kSampleWarps] = y;
    }
  }
  __syncthreads();
  a = sh_a[kSampleWarps];
  c = sh_c[kSampleWarps];
  __syncthreads();
}

constexpr double kWeightScale = 68719476736.0;  // 2^36

__device__ __forceinline__ uint64_t weight(float p) {
  return uint64_t(__double2ll_rn(double(p) * kWeightScale));
}

__global__ void __launch_bounds__(kSampleThreads, 1) sample_kernel(
    const float* __restrict__ logits, int64_t ld, int V, float temperature, int top_k,
    float top_p, const float* __restrict__ uniform, int32_t* __restrict__ out,
    int64_t out_stride, const int* __restrict__ d_step, int64_t u_step, int64_t out_step) {
  extern __shared__ float ps[];  // V values of this row
  if (d_step) {
    if (uniform) uniform += int64_t(*d_step) * u_step;
    out += int64_t(*d_step) * out_step;
  }
  __shared__ uint64_t sh_u[kSampleWarps + 1];
  __shared__ uint64_t sh_c[kSampleWarps + 1];
  __shared__ int sh_i[kSampleWarps + 1];
  __shared__ uint64_t warp_base[kSampleWarps];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const float* z = logits + int64_t(b) * ld;
  for (int i = tid; i < V; i += kSampleThreads) ps[i] = z[i];
  __syncthreads();

  auto umax = [](uint64_t a, uint64_t c) { return a > c ? a : c; };
  auto uadd = [](uint64_t a, uint64_t c) { return a + c; };
  auto imin = [](int a, int c) { return a < c ? a : c; };
  auto imax = [](int a, int c) { return a > c ? a : c; };

  // highest logit, the smaller id on ties
  uint64_t best = 0;
  for (int i = tid; i < V; i += kSampleThreads) best = umax(best, logit_key(ps[i], i));
  best = block_reduce(best, sh_u, umax);
  const int arg = 0xFFFF - int(best & 0xFFFFu);
  if (temperature == 0.f || top_k == 1) {
    if (tid == 0) out[int64_t(b) * out_stride] = arg;
    return;
  }
  const float zmax = ps[arg];
  __syncthreads();  // zmax read everywhere before the row is overwritten
  for (int i = tid; i < V; i += kSampleThreads) ps[i] = expf((ps[i] - zmax) / temperature);
  __syncthreads();

  // thread t holds ids t + 1024 j, j < R (R <= 64: one bit each)
  const int R = (V + kSampleThreads - 1) / kSampleThreads;
  uint64_t mine = 0;  // this thread's valid ids
  for (int j = 0; j < R; ++j)
    if (tid + j * kSampleThreads < V) mine |= uint64_t(1) << j;
  // Largest t in [lo, 2^48) with f(t) >= goal, f(t) = count (by_weight false)
  // or weight of the ids in play with key >= t, ids with key < lo excluded.
  auto bisect = [&](uint64_t lo, bool by_weight, double goal) {
    uint64_t hi = uint64_t(1) << 48;  // f(hi) = 0 < goal
    uint64_t play = mine, above = 0;  // ids with lo <= key < hi; count or weight of key >= hi
    for (int j = 0; j < R; ++j)
      if (((play >> j) & 1) && prob_key(ps[tid + j * kSampleThreads], tid + j * kSampleThreads) < lo)
        play &= ~(uint64_t(1) << j);
    while (hi - lo > 1) {
      const uint64_t mid = lo + (hi - lo) / 2;
      uint64_t ge = 0, part = above;
      for (uint64_t m = play; m; m &= m - 1) {
        const int j = __ffsll(static_cast<long long>(m)) - 1;
        const int i = tid + j * kSampleThreads;
        const float p = ps[i];
        if (prob_key(p, i) >= mid) {
          ge |= uint64_t(1) << j;
          part += by_weight ? weight(p) : 1;
        }
      }
      // ids in play at or above mid (high half) and below it (low half)
      const int n_ge = __popcll(static_cast<long long>(ge));
      uint64_t counts = (uint64_t(n_ge) << 32) | uint64_t(__popcll(static_cast<long long>(play)) - n_ge);
      block_sum2(part, counts, sh_u, sh_c);
      uint64_t left;  // ids still in play after this step
      if (double(part) >= goal) {
        lo = mid;
        play = ge;  // keys below mid leave
        left = counts >> 32;
      } else {
        hi = mid;  // keys at or above mid are always counted from now on
        for (uint64_t m = ge; m; m &= m - 1) {
          const int j = __ffsll(static_cast<long long>(m)) - 1;
          above += by_weight ? weight(ps[tid + j * kSampleThreads]) : 1;
        }
        play &= ~ge;
        left = counts & 0xFFFFFFFFu;
      }
      if (left == 1) {
        // f(lo) >= goal > f(hi) and f changes only at the one key left in
        // [lo, hi): that key is the answer
        uint64_t k = 0;
        if (play) {
          const int j = __ffsll(static_cast<long long>(play)) - 1;
          k = prob_key(ps[tid + j * kSampleThreads], tid + j * kSampleThreads);
        }
        lo = block_reduce(k, sh_u, umax);
        break;
      }
    }
    return lo;
  };
  auto weight_ge = [&](uint64_t t) {
    uint64_t m = 0;
    for (int i = tid; i < V; i += kSampleThreads)
      if (prob_key(ps[i], i) >= t) m += weight(ps[i]);
    return block_reduce(m, sh_u, uadd);
  };
  uint64_t lo = 0;  // kept: keys >= lo
  if (top_k > 0 && top_k < V) lo = bisect(0, false, double(top_k));
  if (top_p < 1.f) lo = bisect(lo, true, double(top_p) * double(weight_ge(lo)));
  const uint64_t kept = weight_ge(lo);
  const float u = fminf(fmaxf(uniform[b], 0.f), 1.f);
  const double target = double(u) * double(kept);

  // the draw in id order: thread t owns ids [tR, tR + R)
  const int i0 = tid * R, i1 = min(V, i0 + R);
  uint64_t s = 0;
  int last = -1;
  for (int i = i0; i < i1; ++i)
    if (prob_key(ps[i], i) >= lo) {
      s += weight(ps[i]);
      last = i;
    }
  uint64_t incl = s;  // inclusive scan over the warp's lanes (exact)
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh_u[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint64_t tot = sh_u[lane];
    uint64_t wi = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_base[lane] = wi - tot;
  }
  __syncthreads();
  const uint64_t base = warp_base[warp] + (incl - s);
  // the first thread whose range carries the running weight past the target
  const int owner =
      block_reduce((last >= 0 && double(base + s) > target) ? tid : kSampleThreads, sh_i, imin);
  const int last_all = block_reduce(last, sh_i, imax);  // the last kept id
  if (owner == kSampleThreads) {
    if (tid == 0) out[int64_t(b) * out_stride] = last_all;
    return;
  }
  if (tid == owner) {
    uint64_t cum = base;
    int pick = last;
    for (int i = i0; i < i1; ++i)
      if (prob_key(ps[i], i) >= lo) {
        cum += weight(ps[i]);
        if (double(cum) > target) {
          pick = i;
          break;
        }
      }
    out[int64_t(b) * out_stride] = pick;
  }
}

}  // namespace

size_t sample_max_vocab() { return kSampleMaxVocab; }

int launch_sample(const float* logits, int64_t ld, int B, int V, float temperature, int top_k,
                  float top_p, const float* uniform, int32_t* out, int64_t out_stride,
                  cudaStream_t st, const int* d_step, int64_t u_step, int64_t out_step) {
  if (B < 1 || V < 1 || V > kSampleMaxVocab) {
    gpt2_internal::set_error("sample: V outside 1..53248");
    return GPT2_ERR_ARG;
  }
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSampleMaxVocab * int(sizeof(float))) != cudaSuccess) {
      cudaGetLastError();
      gpt2_internal::set_error("sample: shared-memory size not accepted");
      return GPT2_ERR_CUDA;
    }
    attr_set = true;
  }
  sample_kernel<<<B, kSampleThreads, size_t(V) * sizeof(float), st>>>(
      logits, ld, V, temperature, top_k, top_p, uniform, out, out_stride, d_step, u_step,
      out_step);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
