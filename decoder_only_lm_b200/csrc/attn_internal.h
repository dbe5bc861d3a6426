// Attention backward with kept score gradients: internal entry points of
// k_attn_tc.cu / k_attn_simt.cu beside the ones in kernels.h.
#pragma once

#include <cstddef>

#include "kernels.h"

// tcgen05 kernels apply: bf16, head size 64, B * T rows addressable
bool attn_tc_supported(int B, int T, int C, int H);
// bytes of the bf16 score-gradient buffer of the tcgen05 backward: dS^T in
// 128 x 128 tiles, one per (key block, query block) of the causal triangle of
// every (batch, head)
size_t attn_tc_ds_bytes(int B, int T, int H);
// launch_attn_bwd<bf16> with a score-gradient buffer `ds` (16-byte aligned,
// attn_tc_ds_bytes): the dK/dV kernel keeps dS^T there and dQ is one
// contraction over it instead of a second recomputation of S, P and dP.
// ds == nullptr, or a shape the tcgen05 kernels do not take, gives
// launch_attn_bwd<bf16>.  ws holds B * H * T floats (Delta), as there.
// With bias_part (B * attn_bias_parts(T) rows of 3C floats) the kernels also
// leave per-block column sums of dqkv there (when they keep dS; the return
// value of attn_bias_parts_written() says whether they did).
int launch_attn_bwd_ds(const bf16* dout, const bf16* qkv, const bf16* out, const float* lse, int B,
                       int Tn, int C, int H, bf16* dqkv, float* ws, bf16* ds, cudaStream_t st,
                       float* bias_part = nullptr);
// row blocks of 128 per sequence: the partial rows per batch element
int attn_bias_parts(int T);
// whether launch_attn_bwd_ds with these arguments writes the partial sums
bool attn_bias_parts_written(int B, int T, int C, int H, const bf16* ds);
// workspace of gpt2_attention_bwd: Delta (rounded up to 1 KB), then, for bf16
// on the tcgen05 path, the score-gradient buffer
size_t attn_bwd_workspace_total(int B, int T, int C, int H, bool bf16_path);
