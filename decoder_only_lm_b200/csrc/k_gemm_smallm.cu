// Dense contraction for a handful of rows (M <= 4): the linear layers of one
// decoding step of a small batch, where every sequence contributes a single
// token, and the tied head on the last position of each sequence.
//
// Source: [ZERO] "GPT training", OpLinearBias / OpFFN / Transformer Block (the
// linear layers y = x W^T + b with their GELU and residual epilogues).
//
// D[m, n] = epilogue(sum_k A[m, k] W[n, k]) with A [M, K] and W [N, K] both
// row-major bf16 (the weight as stored).  With so few rows the work is reading
// W once: one warp per output column streams W's row n with 16-byte loads
// (eight bf16 per lane), keeps one fp32 accumulator per row of A, sums the
// lanes with a fixed butterfly, and lane m applies the layer's epilogue to
// (m, n).  Deterministic; no shared memory, no tensor cores: a few rows
// would leave almost all of a 256-row tensor-core tile empty while paying its
// fixed cost per launch.  (Measured on a decoding step of GPT-2 124M: one
// sequence 1.27 -> 0.66 ms per token; at 16 sequences re-reading A for every
// column makes this kernel slower than the tensor-core one, hence the bound.)

#include "epilogue.cuh"
#include "kernels.h"

namespace {

constexpr int kSmallMMax = 4;
constexpr int kSmallMWarps = 8;

template <int MR, typename OutT>
__global__ void __launch_bounds__(kSmallMWarps * 32) gemm_smallm_kernel(
    const bf16* __restrict__ A, int64_t lda, const bf16* __restrict__ W, int64_t ldw, int M,
    int N, int K, EpiParams ep) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * kSmallMWarps;
  for (int64_t n = int64_t(blockIdx.x) * kSmallMWarps + (threadIdx.x >> 5); n < N; n += warps) {
    const bf16* w = W + n * ldw;
    float acc[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) acc[m] = 0.f;
    for (int k = lane * 8; k < K; k += 256) {
      const uint4 wu = __ldg(reinterpret_cast<const uint4*>(w + k));
      const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wu);
      float wf[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(wh[j]);
        wf[2 * j] = f.x;
        wf[2 * j + 1] = f.y;
      }
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        if (m < M) {
          const uint4 au = __ldg(reinterpret_cast<const uint4*>(A + m * lda + k));
          const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&au);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(ah[j]);
            acc[m] = fmaf(f.x, wf[2 * j], acc[m]);
            acc[m] = fmaf(f.y, wf[2 * j + 1], acc[m]);
          }
        }
      }
    }
    float mine = 0.f;  // lane m keeps row m's total
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      float v = acc[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == m) mine = v;
    }
    if (lane < M) epi_apply<OutT>(ep, ep.kind, lane, int(n), mine);
  }
}

template <int MR, typename OutT>
int launch_smallm(const GemmArgs& g, cudaStream_t st) {
  const int64_t blocks = std::min<int64_t>((g.N + kSmallMWarps - 1) / kSmallMWarps,
                                           8 * int64_t(gpt2_internal::sm_count()));
  gemm_smallm_kernel<MR, OutT><<<int(blocks), kSmallMWarps * 32, 0, st>>>(
      static_cast<const bf16*>(g.A), g.lda, static_cast<const bf16*>(g.B), g.ldb, g.M, g.N, g.K,
      g.ep);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

}  // namespace

bool gemm_smallm_supported(const GemmArgs& g) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return g.bf16_in && g.a_kmajor && g.b_kmajor && g.M >= 1 && g.M <= kSmallMMax &&
         g.K % 8 == 0 && g.lda % 8 == 0 && g.ldb % 8 == 0 && al16(g.A) && al16(g.B) &&
         g.ep.kind != EPI_LSE_PARTIAL;
}

int gemm_smallm_launch(const GemmArgs& g, cudaStream_t st) {
  // the accumulators are unrolled for kSmallMMax rows
  const bool f32 = !g.ep.out_bf16 || g.ep.kind == EPI_RESID || g.ep.kind == EPI_ACC;
  return f32 ? launch_smallm<kSmallMMax, float>(g, st) : launch_smallm<kSmallMMax, bf16>(g, st);
}
