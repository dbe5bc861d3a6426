// Attention backward for callers that cannot allocate device memory.
//
// gpt2_attention_bwd needs a caller-provided workspace for its per-row
// scratch (Delta_i = dO_i . O_i, one float per (batch, head, position)).
// Some callers cannot provide one: a host program that has handed the whole
// device to another allocator up front and runs under a fixed memory budget,
// or a latency-critical loop that must not call cudaMalloc / cudaFree because
// those calls can wait for the whole device to go idle.  This entry point
// gives them the same computation with its scratch in a fixed array that the
// library declares at file scope in device memory, so the call allocates
// nothing.  The inputs and outputs are still the caller's.

#include <mutex>
#include <string>

#include "kernels.h"

namespace {

// Largest B * H * T the fixed scratch holds: 1,048,576 rows = 4 MiB per
// device (resident on every device that loads this library, until exit).
constexpr int64_t kMaxRows = int64_t(1) << 20;

static __device__ __align__(256) float g_attn_bwd_scratch[kMaxRows];

// Device address of the scratch array on device `dev`, looked up once per
// device (host code only sees a host-side stand-in under the array's name).
float* scratch_on_device(int dev, std::string* err) {
  static std::mutex mu;
  static float* addr[64] = {nullptr};
  if (dev < 0 || dev >= 64) {
    *err = "attention_bwd_noalloc: device index out of range";
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_attn_bwd_scratch);
    if (e != cudaSuccess) {
      *err = std::string("attention_bwd_noalloc: cudaGetSymbolAddress: ") + cudaGetErrorString(e);
      return nullptr;
    }
    addr[dev] = static_cast<float*>(p);
  }
  return addr[dev];
}

}  // namespace

extern "C" int gpt2_attention_bwd_noalloc(const void* dout, const void* qkv, const void* out,
                                          const float* lse, int dtype, int B, int T, int C, int H,
                                          void* dqkv, void* stream) {
  if (!dout || !qkv || !out || !lse || !dqkv || B < 1 || T < 1 || H < 1 || C % H ||
      (dtype != GPT2_BF16 && dtype != GPT2_F32)) {
    gpt2_internal::set_error("attention_bwd_noalloc: bad arguments");
    return GPT2_ERR_ARG;
  }
  if (int64_t(B) * H * T > kMaxRows) {
    gpt2_internal::set_error(
        "attention_bwd_noalloc: B * H * T = " + std::to_string(int64_t(B) * H * T) +
        " exceeds the fixed scratch of " + std::to_string(kMaxRows) +
        " rows; use gpt2_attention_bwd with a workspace");
    return GPT2_ERR_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    gpt2_internal::set_error("attention_bwd_noalloc: no current device");
    return GPT2_ERR_CUDA;
  }
  std::string err;
  float* ws = scratch_on_device(dev, &err);
  if (!ws) {
    gpt2_internal::set_error(err);
    return GPT2_ERR_CUDA;
  }
  // Every element of the scratch that the kernels read is written first in
  // this call (Delta), so nothing has to be cleared between calls.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == GPT2_BF16)
    return launch_attn_bwd<bf16>(static_cast<const bf16*>(dout), static_cast<const bf16*>(qkv),
                                 static_cast<const bf16*>(out), lse, B, T, C, H,
                                 static_cast<bf16*>(dqkv), ws, st);
  return launch_attn_bwd<float>(static_cast<const float*>(dout), static_cast<const float*>(qkv),
                                static_cast<const float*>(out), lse, B, T, C, H,
                                static_cast<float*>(dqkv), ws, st);
}
