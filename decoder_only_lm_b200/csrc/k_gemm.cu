// GEMM dispatch: bf16 contractions of at most 4 rows with both operands
// K-major (the one-token-per-sequence layers of decoding) run on the
// small-M kernel; other bf16 contractions run on the tcgen05 tensor-core kernel
// when their operands meet its alignment rules (16-byte aligned bases, leading
// dimensions multiples of 8 elements); the fp32 parity mode and unaligned
// shapes run on the SIMT kernel.

#include <algorithm>

#include "kernels.h"

size_t gemm_simt_workspace_bytes(int M, int N, int K);
int gemm_simt_launch(const GemmArgs& g, cudaStream_t st);
bool gemm_tc_supported(const GemmArgs& g);
size_t gemm_tc_workspace_bytes(int M, int N, int K);
int gemm_tc_launch(const GemmArgs& g, cudaStream_t st);
bool gemm_smallm_supported(const GemmArgs& g);
int gemm_smallm_launch(const GemmArgs& g, cudaStream_t st);

size_t gemm_workspace_bytes(int M, int N, int K) {
  return std::max(gemm_simt_workspace_bytes(M, N, K), gemm_tc_workspace_bytes(M, N, K));
}

int gemm_launch(const GemmArgs& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return GPT2_OK;
  if (gemm_smallm_supported(g)) return gemm_smallm_launch(g, st);  // <= 4 rows (decoding)
  if (gemm_tc_supported(g)) return gemm_tc_launch(g, st);
  return gemm_simt_launch(g, st);
}
