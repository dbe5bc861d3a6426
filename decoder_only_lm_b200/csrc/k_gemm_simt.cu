// SIMT (CUDA-core FFMA) GEMM used by the fp32 parity mode, and the shape-
// general fallback-free path for contractions the tensor-core kernel does not
// take (tiny or unaligned shapes).  128x128 block tile, 8x8 per thread,
// fp32 accumulation, any operand major-ness, fused epilogues.
//
// Split-K (EPI_ACC only, for weight gradients whose output has few tiles):
// split z writes its partial tile to ws[z]; a reduction kernel adds the
// splits in order, so the result does not depend on scheduling.

#include "epilogue.cuh"

namespace {

constexpr int BM = 128, BN = 128, BK = 16, NT = 256;

template <typename TA>
__device__ __forceinline__ void load_tile(const TA* __restrict__ X, int kmajor, int64_t ld, int r0,
                                          int R, int k0, int k1, float (*S)[BM + 4]) {
  // S[kk][r] = X(r0 + r, k0 + kk)
  for (int e = threadIdx.x; e < BM * BK; e += NT) {
    int r, kk;
    if (kmajor) {
      r = e / BK;
      kk = e % BK;
    } else {
      kk = e / BM;
      r = e % BM;
    }
    const int gr = r0 + r, gk = k0 + kk;
    float v = 0.f;
    if (gr < R && gk < k1) v = to_f32<TA>(kmajor ? X[int64_t(gr) * ld + gk] : X[int64_t(gk) * ld + gr]);
    S[kk][r] = v;
  }
}

template <typename TA, typename OutT>
__global__ void __launch_bounds__(NT) gemm_simt_kernel(const TA* __restrict__ A, int a_kmajor,
                                                       int64_t lda, const TA* __restrict__ B,
                                                       int b_kmajor, int64_t ldb, int M, int N,
                                                       int K, int k_split, EpiParams ep,
                                                       float* __restrict__ ws) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int bm = blockIdx.y * BM, bn = blockIdx.x * BN;
  const int k0 = blockIdx.z * k_split, k1 = min(K, k0 + k_split);
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int kt = k0; kt < k1; kt += BK) {
    load_tile<TA>(A, a_kmajor, lda, bm, M, kt, k1, As);
    load_tile<TA>(B, b_kmajor, ldb, bn, N, kt, k1, Bs);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = bm + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = bn + tx + 16 * j;
      if (n >= N) continue;
      if (ws)
        ws[(int64_t(blockIdx.z) * M + m) * N + n] = acc[i][j];
      else
        epi_apply<OutT>(ep, ep.kind, m, n, acc[i][j]);
    }
  }
}

// out[m,n] = (accumulate ? out : 0) + alpha * sum_z ws[z][m][n]
__global__ void splitk_reduce_kernel(const float* __restrict__ ws, int splits, int M, int N,
                                     float* __restrict__ out, int64_t ldo, float alpha,
                                     int accumulate) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= int64_t(M) * N) return;
  const int m = int(i / N), n = int(i % N);
  float acc = 0.f;
  for (int z = 0; z < splits; ++z) acc += ws[int64_t(z) * M * N + i];
  float* o = out + int64_t(m) * ldo + n;
  *o = (accumulate ? *o : 0.f) + alpha * acc;
}

int choose_splits(int M, int N, int K) {
  const int tiles = cdiv(M, BM) * cdiv(N, BN);
  const int target = 2 * gpt2_internal::sm_count();
  int s = 1;
  while (tiles * s * 2 <= target && K / (s * 2) >= 256) s *= 2;
  return s;
}

}  // namespace

size_t gemm_simt_workspace_bytes(int M, int N, int K) {
  int s = choose_splits(M, N, K);
  return s > 1 ? size_t(s) * M * N * sizeof(float) : 0;
}

int gemm_simt_launch(const GemmArgs& g, cudaStream_t st) {
  int splits = 1;
  if (g.ep.kind == EPI_ACC) {
    splits = choose_splits(g.M, g.N, g.K);
    if (size_t(splits) * g.M * g.N * sizeof(float) > g.ws_bytes || !g.ws) splits = 1;
  }
  const int k_split = splits > 1 ? cdiv(cdiv(g.K, splits), BK) * BK : g.K;
  splits = k_split > 0 ? cdiv(g.K, k_split) : 1;
  dim3 grid(cdiv(g.N, BN), cdiv(g.M, BM), splits);
  float* ws = splits > 1 ? g.ws : nullptr;
  const bool ob = g.ep.out_bf16;
  if (g.bf16_in) {
    if (ob)
      gemm_simt_kernel<bf16, bf16><<<grid, NT, 0, st>>>((const bf16*)g.A, g.a_kmajor, g.lda,
                                                        (const bf16*)g.B, g.b_kmajor, g.ldb, g.M,
                                                        g.N, g.K, k_split, g.ep, ws);
    else
      gemm_simt_kernel<bf16, float><<<grid, NT, 0, st>>>((const bf16*)g.A, g.a_kmajor, g.lda,
                                                         (const bf16*)g.B, g.b_kmajor, g.ldb, g.M,
                                                         g.N, g.K, k_split, g.ep, ws);
  } else {
    if (ob)
      gemm_simt_kernel<float, bf16><<<grid, NT, 0, st>>>((const float*)g.A, g.a_kmajor, g.lda,
                                                         (const float*)g.B, g.b_kmajor, g.ldb, g.M,
                                                         g.N, g.K, k_split, g.ep, ws);
    else
      gemm_simt_kernel<float, float><<<grid, NT, 0, st>>>((const float*)g.A, g.a_kmajor, g.lda,
                                                          (const float*)g.B, g.b_kmajor, g.ldb,
                                                          g.M, g.N, g.K, k_split, g.ep, ws);
  }
  COUNT_LAUNCH(1);
  if (ws) {
    const int64_t n = int64_t(g.M) * g.N;
    splitk_reduce_kernel<<<int(cdiv64(n, 256)), 256, 0, st>>>(
        ws, splits, g.M, g.N, reinterpret_cast<float*>(g.ep.out), g.ep.ldo, g.ep.alpha,
        g.ep.accumulate);
    COUNT_LAUNCH(1);
  }
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
