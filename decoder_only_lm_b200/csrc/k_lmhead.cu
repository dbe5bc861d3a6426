// Tied LM head + mean cross-entropy, forward and backward, without holding
// the [M, Vp] logits [ZERO: output layer, fused projection + cross-entropy;
// LECTURE: tied head over the padded vocabulary; CS336 §1: the row maximum is
// subtracted before exponentiating].
//
// bf16 path (tensor cores):
//   forward  one GEMM z = h W^T over all rows whose epilogue reduces each
//            128 x 256 tile to a per-row (max, sum of exp) partial and picks
//            the target logit; a merge kernel combines the partials of a row in
//            order: lse = M + log sum_t s_t exp(m_t - M), loss = lse - z_y.
//            No logit is ever written to memory.
//   backward per chunk of kChunkBf16 rows: the recomputed logits go straight
//            from TMEM through dz = scale (exp(z - lse) - onehot) to a bf16
//            chunk buffer, then dh[chunk] = dz W (K = Vp, split along K) and
//            dW (+)= dz^T h[chunk] (fp32, one add per element and chunk, in
//            chunk order).  With kRingBf16 > 1 chunk buffers and a side stream
//            the next chunk's logits are recomputed while the previous chunk's
//            weight gradient still reads its buffer.  The live part of dz is
//            kRingBf16 x kChunkBf16 x Vp bf16 (one 2048-row chunk, 206 MB at
//            Vp = 50304), whatever the number of rows: in the graph-replayed
//            124M step this costs the same time as one buffer of all 16384 rows
//            (1.65 GB), while a ring of two 1024-row chunks was 8% slower.
// fp32 path (parity mode, CUDA cores): per chunk of <= 2048 rows, logits in an
// fp32 chunk buffer, a row kernel for lse / loss / dz, then the same two
// contractions.

#include <algorithm>

#include "kernels.h"

namespace {

constexpr int kChunkBf16 = 2048, kRingBf16 = 1, kChunkF32 = 2048;
constexpr int kTileN = 256;  // column tile of the LSE-partial tensor-core GEMM

int chunk_rows(int bf16) { return bf16 ? kChunkBf16 : kChunkF32; }
int ring(int bf16) { return bf16 ? kRingBf16 : 1; }

size_t r256(size_t b) { return (b + 255) / 256 * 256; }

struct Layout {
  size_t part, tgt, z, dz, gws, total;
};

Layout layout(int M, int C, int Vp, int bf16) {
  const int mc = std::min(chunk_rows(bf16), M);
  const int nt = cdiv(Vp, kTileN);
  Layout L{};
  L.part = bf16 ? r256(size_t(M) * nt * 4) : 0;  // each of part_max, part_sum
  L.tgt = bf16 ? r256(size_t(M) * 4) : 0;
  L.z = bf16 ? 0 : r256(size_t(mc) * Vp * 4);
  L.dz = r256(size_t(mc) * Vp * (bf16 ? 2 : 4));  // one chunk buffer (ring() of them)
  L.gws = r256(std::max({gemm_workspace_bytes(mc, Vp, C), gemm_workspace_bytes(mc, C, Vp),
                         gemm_workspace_bytes(Vp, C, mc), gemm_workspace_bytes(M, Vp, C)}));
  L.total = 2 * L.part + L.tgt + L.z + size_t(ring(bf16)) * L.dz + L.gws + 256;
  return L;
}

// One warp per row: lse = max + log(sum_t s_t exp(m_t - max)); loss = lse - z_y.
__global__ void lse_merge_kernel(const float* __restrict__ pm, const float* __restrict__ ps,
                                 int nt, const float* __restrict__ zt, int64_t M,
                                 float* __restrict__ lse, float* __restrict__ row_loss) {
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* a = pm + row * nt;
  const float* b = ps + row * nt;
  float mx = -INFINITY;
  for (int t = lane; t < nt; t += 32) mx = fmaxf(mx, a[t]);
  mx = warp_max(mx);
  float s = 0.f;
  for (int t = lane; t < nt; t += 32) s += b[t] * __expf(a[t] - mx);
  s = warp_sum(s);
  if (lane == 0) {
    const float l = mx + logf(s);
    lse[row] = l;
    row_loss[row] = l - zt[row];
  }
}

}  // namespace

size_t lmhead_workspace(int M, int C, int Vp, int bf16) { return layout(M, C, Vp, bf16).total; }

int lmhead_fwd(const void* h, const void* W, const int32_t* y, int M, int C, int Vp, int bf16,
               float* lse, float* row_loss, void* ws, size_t ws_bytes, cudaStream_t st) {
  const Layout L = layout(M, C, Vp, bf16);
  if (!ws || ws_bytes < L.total) {
    gpt2_internal::set_error("lmhead: workspace too small");
    return GPT2_ERR_ARG;
  }
  char* w = static_cast<char*>(ws);
  float* pmax = reinterpret_cast<float*>(w);
  float* psum = reinterpret_cast<float*>(w + L.part);
  float* tgt = reinterpret_cast<float*>(w + 2 * L.part);
  float* z = reinterpret_cast<float*>(w + 2 * L.part + L.tgt);
  float* gws = reinterpret_cast<float*>(w + 2 * L.part + L.tgt + L.z + ring(bf16) * L.dz);
  if (bf16) {
    EpiParams e;
    e.kind = EPI_LSE_PARTIAL;
    e.tgt = y;
    e.part_max = pmax;
    e.part_sum = psum;
    e.tgt_logit = tgt;
    e.part_ld = cdiv(Vp, kTileN);
    GemmArgs g{h, 1, C, W, 1, C, 1, M, Vp, C, e, gws, L.gws};
    if (!gemm_tc_supported(g)) {
      gpt2_internal::set_error("lmhead: bf16 operands must be 16-byte aligned with C % 8 == 0");
      return GPT2_ERR_ARG;
    }
    int rc = gemm_launch(g, st);
    if (rc) return rc;
    lse_merge_kernel<<<int(cdiv64(M, 8)), 256, 0, st>>>(pmax, psum, e.part_ld, tgt, M, lse,
                                                        row_loss);
    COUNT_LAUNCH(1);
    GPT2_LAUNCH_CHECK();
    return GPT2_OK;
  }
  for (int64_t r0 = 0; r0 < M; r0 += kChunkF32) {
    const int mc = int(std::min<int64_t>(kChunkF32, M - r0));
    EpiParams e;
    e.kind = EPI_STORE;
    e.out = z;
    e.ldo = Vp;
    GemmArgs g{static_cast<const float*>(h) + r0 * C, 1, C, W, 1, C, 0, mc, Vp, C, e, gws, L.gws};
    int rc = gemm_launch(g, st);
    if (rc) return rc;
    rc = launch_ce_rows_fwd(z, y + r0, mc, Vp, lse + r0, row_loss + r0, st);
    if (rc) return rc;
  }
  return GPT2_OK;
}

int lmhead_bwd(const void* h, const void* W, const int32_t* y, const float* lse, int M, int C,
               int Vp, int bf16, float scale, void* dh, float* dW, int dw_accumulate, void* ws,
               size_t ws_bytes, cudaStream_t st, const LmSide* side) {
  const Layout L = layout(M, C, Vp, bf16);
  if (!ws || ws_bytes < L.total) {
    gpt2_internal::set_error("lmhead: workspace too small");
    return GPT2_ERR_ARG;
  }
  char* w = static_cast<char*>(ws);
  float* z = reinterpret_cast<float*>(w + 2 * L.part + L.tgt);
  char* dz0 = w + 2 * L.part + L.tgt + L.z;
  const int nbuf = ring(bf16);
  float* gws = reinterpret_cast<float*>(dz0 + nbuf * L.dz);
  const size_t a = bf16 ? 2 : 4;
  const int chunk = chunk_rows(bf16);
  const bool par = side && side->st && dh && dW;
  int c = 0;
  for (int64_t r0 = 0; r0 < M; r0 += chunk, ++c) {
    const int mc = int(std::min<int64_t>(chunk, M - r0));
    const void* hr = static_cast<const char*>(h) + r0 * C * int64_t(a);
    void* dz = dz0 + (c % nbuf) * L.dz;
    // the weight gradient of the chunk that last used this buffer (side
    // stream) has finished reading it; dH of that chunk ran before on st
    if (par && c >= nbuf) GPT2_CUDA_TRY(cudaStreamWaitEvent(st, side->e_join[c % nbuf], 0));
    int rc;
    if (bf16) {
      EpiParams e;
      e.kind = EPI_CE_GRAD;
      e.out = dz;
      e.ldo = Vp;
      e.out_bf16 = 1;
      e.lse = lse + r0;
      e.tgt = y + r0;
      e.ce_scale = scale;
      GemmArgs g{hr, 1, C, W, 1, C, 1, mc, Vp, C, e, gws, L.gws};
      rc = gemm_launch(g, st);
    } else {
      EpiParams e;
      e.kind = EPI_STORE;
      e.out = z;
      e.ldo = Vp;
      GemmArgs g{hr, 1, C, W, 1, C, 0, mc, Vp, C, e, gws, L.gws};
      rc = gemm_launch(g, st);
      if (!rc)
        rc = launch_ce_rows_bwd<float>(z, lse + r0, y + r0, mc, Vp, scale, static_cast<float*>(dz),
                                       st);
    }
    if (rc) return rc;
    if (par) {  // dz of this chunk complete: dW may start beside dH
      GPT2_CUDA_TRY(cudaEventRecord(side->e_fork, st));
      GPT2_CUDA_TRY(cudaStreamWaitEvent(side->st, side->e_fork, 0));
    }
    if (dh) {
      EpiParams e;
      e.kind = EPI_STORE;
      e.out = static_cast<char*>(dh) + r0 * C * int64_t(a);
      e.ldo = C;
      e.out_bf16 = bf16;
      GemmArgs g{dz, 1, Vp, W, 0, C, bf16, mc, C, Vp, e, gws, L.gws};
      rc = gemm_launch(g, st);
      if (rc) return rc;
    }
    if (dW) {
      // chunks add into dW one after the other (stream order): deterministic
      EpiParams e;
      e.kind = EPI_ACC;
      e.out = dW;
      e.ldo = C;
      e.accumulate = (dw_accumulate || r0 > 0) ? 1 : 0;
      GemmArgs g{dz, 0, Vp, hr, 0, C, bf16, Vp, C, mc, e, par ? side->ws : gws,
                 par ? side->ws_bytes : L.gws};
      rc = gemm_launch(g, par ? side->st : st);
      if (rc) return rc;
      if (par) GPT2_CUDA_TRY(cudaEventRecord(side->e_join[c % nbuf], side->st));
    }
  }
  // the side stream runs in order: its last weight-gradient GEMM done means all are
  if (par && c > 0) GPT2_CUDA_TRY(cudaStreamWaitEvent(st, side->e_join[(c - 1) % nbuf], 0));
  return GPT2_OK;
}
