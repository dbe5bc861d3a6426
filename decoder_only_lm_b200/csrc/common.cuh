// Shared device/host helpers of the GPT-2 B200 library (no model arithmetic).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/gpt2.h"

typedef __nv_bfloat16 bf16;

// Device-side status words written by kernels and read by the host when it
// synchronises.  Kernels never trap: they record and carry on.
struct DevStatus {
  int token_bad;    // an input or target id outside [0, vocab_size)
  int nonfinite;    // the gradient norm was not finite: the update was skipped
  int timeout;      // a bounded wait gave up
  int timeout_where;
  int step;         // AdamW step counter t (device copy, authoritative)
  int window_bad;   // a batch window read at a device cursor ran past its stream
  int pad[2];
};

#define GPT2_CUDA_TRY(expr)                                                        \
  do {                                                                             \
    cudaError_t e_ = (expr);                                                       \
    if (e_ != cudaSuccess) {                                                       \
      gpt2_internal::set_error(std::string(#expr) + ": " + cudaGetErrorString(e_)); \
      return GPT2_ERR_CUDA;                                                        \
    }                                                                              \
  } while (0)

#define GPT2_LAUNCH_CHECK()                                                        \
  do {                                                                             \
    cudaError_t e_ = cudaGetLastError();                                           \
    if (e_ != cudaSuccess) {                                                       \
      gpt2_internal::set_error(std::string("kernel launch: ") + cudaGetErrorString(e_)); \
      return GPT2_ERR_CUDA;                                                        \
    }                                                                              \
  } while (0)

namespace gpt2_internal {
void set_error(const std::string& msg);  // thread-local "last error" for op-level calls
const std::string& get_error();
int sm_count();                          // SMs of the current device (cached)
void count_launches(int n);              // kernels launched by this host thread
int64_t launches();
}

#define COUNT_LAUNCH(n) gpt2_internal::count_launches(n)

// ---- conversions -----------------------------------------------------------
template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// Round a float through the storage type (identity for float).
template <typename T>
__device__ __forceinline__ float round_through(float v) { return to_f32<T>(from_f32<T>(v)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// GPT-2's approximate GELU (tanh form) and its derivative.  tanhf is the CUDA
// math library's function, called, not re-derived.
__device__ __forceinline__ float gelu_tanh(float u) {
  const float k = 0.7978845608028654f, a = 0.044715f;
  return 0.5f * u * (1.f + tanhf(k * (u + a * u * u * u)));
}
__device__ __forceinline__ float gelu_tanh_grad(float u) {
  const float k = 0.7978845608028654f, a = 0.044715f;
  float t = tanhf(k * (u + a * u * u * u));
  return 0.5f * (1.f + t) + 0.5f * u * (1.f - t * t) * k * (1.f + 3.f * a * u * u);
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

static inline int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }
static inline int cdiv(int a, int b) { return (a + b - 1) / b; }
