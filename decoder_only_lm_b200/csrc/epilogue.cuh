// Per-element epilogues of the GEMM kernels (shared by the SIMT and tcgen05
// GEMMs).  Each applies to one accumulator value acc = sum_k A(m,k) B(n,k).
#pragma once

#include "kernels.h"

template <typename T>
__device__ __forceinline__ void store_as(void* base, int64_t idx, float v) {
  reinterpret_cast<T*>(base)[idx] = from_f32<T>(v);
}
template <typename T>
__device__ __forceinline__ float load_as(const void* base, int64_t idx) {
  return to_f32<T>(reinterpret_cast<const T*>(base)[idx]);
}

// Linear layer epilogues [ZERO: OpLinearBias (bias), OpFFN (bias + GELU),
// Transformer Block (residual add)]; the cross-entropy gradient of the tied
// head [ZERO: output layer] dz = scale * (softmax(z) - onehot(y)).
template <typename OutT>
__device__ __forceinline__ void epi_apply(const EpiParams& e, int kind, int m, int n, float acc) {
  const int64_t i = int64_t(m) * e.ldo + n;
  switch (kind) {
    case EPI_STORE: {
      float v = acc * e.alpha + (e.bias ? e.bias[n] : 0.f);
      store_as<OutT>(e.out, i, v);
      break;
    }
    case EPI_GELU: {
      float u = round_through<OutT>(acc + e.bias[n]);
      store_as<OutT>(e.out, i, u);
      store_as<OutT>(e.out2, i, gelu_tanh(u));
      break;
    }
    case EPI_RESID:
      e.rout[i] = e.rin[i] + acc + (e.bias ? e.bias[n] : 0.f);
      break;
    case EPI_ACC: {
      float* o = reinterpret_cast<float*>(e.out);
      o[i] = (e.accumulate ? o[i] : 0.f) + e.alpha * acc;
      break;
    }
    case EPI_GELU_BWD:
      store_as<OutT>(e.out, i, acc * gelu_tanh_grad(load_as<OutT>(e.aux, i)));
      break;
    case EPI_CE_GRAD: {
      float p = __expf(acc - e.lse[m]);
      store_as<OutT>(e.out, i, e.ce_scale * (p - (n == e.tgt[m] ? 1.f : 0.f)));
      break;
    }
  }
}
