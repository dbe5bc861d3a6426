// Causal multi-head attention on CUDA cores (fp32 parity mode and any head
// size), flash style: the [T, T] scores are never stored; the forward keeps a
// running max / sum per query row and saves the row log-normaliser, the
// backward recomputes probabilities from it [ZERO: Attention, OpFlashAttention
// recomputes scores in the backward; LECTURE: flash attention, causal mask].
//
// Layout: qkv [B, T, 3C] with q | k | v and head h on channels [hD, (h+1)D);
// out [B, T, C]; lse [B, H, T].  Backward: dkdv kernel (one thread per key)
// and dq kernel (one thread per query) both recompute p_ij, so no two threads
// add into the same element and the result is deterministic.

#include "attn_internal.h"
#include "kernels.h"

namespace {

constexpr int QB = 64;   // queries per block in the forward, one per thread
constexpr int QBB = 32;  // keys / queries per block in the backward (shared memory)

template <typename T, int D>
__global__ void __launch_bounds__(QB) attn_fwd_kernel(const T* __restrict__ qkv, int Tn, int C,
                                                      int H, T* __restrict__ out,
                                                      float* __restrict__ lse) {
  __shared__ float Ks[QB][D + 1];
  __shared__ float Vs[QB][D + 1];
  const int b = blockIdx.z, h = blockIdx.y, qb = blockIdx.x;
  const int i = qb * QB + threadIdx.x;
  const int64_t row_stride = 3 * int64_t(C);
  const T* base = qkv + int64_t(b) * Tn * row_stride + h * D;
  const float scale = rsqrtf(float(D));
  float q[D], o[D];
  float mrun = -INFINITY, l = 0.f;
  if (i < Tn) {
#pragma unroll
    for (int d = 0; d < D; ++d) q[d] = to_f32<T>(base[int64_t(i) * row_stride + d]) * scale;
  }
#pragma unroll
  for (int d = 0; d < D; ++d) o[d] = 0.f;
  for (int kb = 0; kb <= qb; ++kb) {
    __syncthreads();
    for (int e = threadIdx.x; e < QB * D; e += QB) {
      const int r = e / D, d = e % D;
      const int j = kb * QB + r;
      float kv = 0.f, vv = 0.f;
      if (j < Tn) {
        kv = to_f32<T>(base[int64_t(j) * row_stride + C + d]);
        vv = to_f32<T>(base[int64_t(j) * row_stride + 2 * C + d]);
      }
      Ks[r][d] = kv;
      Vs[r][d] = vv;
    }
    __syncthreads();
    if (i < Tn) {
      const int rmax = min(QB, i - kb * QB + 1);  // keys j <= i only
      for (int r = 0; r < rmax; ++r) {
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) s = fmaf(q[d], Ks[r][d], s);
        const float mn = fmaxf(mrun, s);
        const float corr = expf(mrun - mn);
        const float p = expf(s - mn);
        l = l * corr + p;
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] = fmaf(p, Vs[r][d], o[d] * corr);
        mrun = mn;
      }
    }
  }
  if (i < Tn) {
    const float inv = 1.f / l;
    T* orow = out + (int64_t(b) * Tn + i) * C + h * D;
#pragma unroll
    for (int d = 0; d < D; ++d) orow[d] = from_f32<T>(o[d] * inv);
    lse[(int64_t(b) * H + h) * Tn + i] = mrun + logf(l);
  }
}

// Delta_i = sum_d dout_i,d * out_i,d   ([B, H, T], fp32)
template <typename T>
__global__ void attn_delta_kernel(const T* __restrict__ dout, const T* __restrict__ out, int B,
                                  int Tn, int C, int H, float* __restrict__ delta) {
  const int64_t idx = blockIdx.x * int64_t(blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const int64_t nrows = int64_t(B) * H * Tn;
  if (idx >= nrows) return;
  const int i = int(idx % Tn);
  const int h = int((idx / Tn) % H);
  const int b = int(idx / (int64_t(Tn) * H));
  const int D = C / H;
  const int64_t off = (int64_t(b) * Tn + i) * C + h * D;
  float s = 0.f;
  for (int d = lane; d < D; d += 32) s += to_f32<T>(dout[off + d]) * to_f32<T>(out[off + d]);
  s = warp_sum(s);
  if (lane == 0) delta[idx] = s;
}

// Delta for head size 64, bf16: eight lanes per (b, t, h) row, h fastest, so
// a warp's 16-byte loads cover four consecutive 128-byte head slices of dO
// and of O (512 contiguous bytes each); the eight partial dot products are
// summed with three shuffles.
__global__ void attn_delta64_kernel(const bf16* __restrict__ dout, const bf16* __restrict__ out,
                                    int B, int Tn, int C, int H, float* __restrict__ delta) {
  const int64_t idx = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 3;  // row
  const int part = threadIdx.x & 7;
  if (idx >= int64_t(B) * Tn * H) return;  // whole 8-lane groups leave together
  const int h = int(idx % H);
  const int64_t bt = idx / H;  // b * T + t
  const int b = int(bt / Tn), t = int(bt % Tn);
  const uint4 ua = *reinterpret_cast<const uint4*>(dout + bt * C + h * 64 + part * 8);
  const uint4 ub = *reinterpret_cast<const uint4*>(out + bt * C + h * 64 + part * 8);
  const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&ua);
  const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&ub);
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 fa = __bfloat1622float2(ha[j]), fb = __bfloat1622float2(hb[j]);
    s += fa.x * fb.x + fa.y * fb.y;
  }
  const unsigned grp = 0xffu << (threadIdx.x & 24);  // this row's eight lanes
  s += __shfl_xor_sync(grp, s, 4);
  s += __shfl_xor_sync(grp, s, 2);
  s += __shfl_xor_sync(grp, s, 1);
  if (part == 0) delta[(int64_t(b) * H + h) * Tn + t] = s;
}

// One thread per key j: dv_j = sum_{i>=j} p_ij do_i, dk_j = sum_{i>=j} ds_ij q_i / sqrt(D)
template <typename T, int D>
__global__ void __launch_bounds__(QBB) attn_dkdv_kernel(const T* __restrict__ dout,
                                                       const T* __restrict__ qkv,
                                                       const float* __restrict__ lse,
                                                       const float* __restrict__ delta, int Tn,
                                                       int C, int H, T* __restrict__ dqkv) {
  __shared__ float Qs[QBB][D + 1];
  __shared__ float Os[QBB][D + 1];  // dout rows
  __shared__ float Kmine[QBB][D + 1];
  __shared__ float Vmine[QBB][D + 1];
  __shared__ float Ls[QBB], Ds[QBB];
  const int b = blockIdx.z, h = blockIdx.y, kb = blockIdx.x;
  const int j = kb * QBB + threadIdx.x;
  const int64_t rs = 3 * int64_t(C);
  const T* base = qkv + int64_t(b) * Tn * rs + h * D;
  const T* dbase = dout + int64_t(b) * Tn * C + h * D;
  const float scale = rsqrtf(float(D));
  for (int e = threadIdx.x; e < QBB * D; e += QBB) {
    const int r = e / D, d = e % D;
    const int jj = kb * QBB + r;
    Kmine[r][d] = jj < Tn ? to_f32<T>(base[int64_t(jj) * rs + C + d]) : 0.f;
    Vmine[r][d] = jj < Tn ? to_f32<T>(base[int64_t(jj) * rs + 2 * C + d]) : 0.f;
  }
  float dk[D], dv[D];
#pragma unroll
  for (int d = 0; d < D; ++d) dk[d] = dv[d] = 0.f;
  const int nqb = (Tn + QBB - 1) / QBB;
  for (int qb = kb; qb < nqb; ++qb) {
    __syncthreads();
    for (int e = threadIdx.x; e < QBB * D; e += QBB) {
      const int r = e / D, d = e % D;
      const int i = qb * QBB + r;
      Qs[r][d] = i < Tn ? to_f32<T>(base[int64_t(i) * rs + d]) : 0.f;
      Os[r][d] = i < Tn ? to_f32<T>(dbase[int64_t(i) * C + d]) : 0.f;
    }
    if (threadIdx.x < QBB) {
      const int i = qb * QBB + threadIdx.x;
      Ls[threadIdx.x] = i < Tn ? lse[(int64_t(b) * H + h) * Tn + i] : 0.f;
      Ds[threadIdx.x] = i < Tn ? delta[(int64_t(b) * H + h) * Tn + i] : 0.f;
    }
    __syncthreads();
    if (j < Tn) {
      for (int r = 0; r < QBB; ++r) {
        const int i = qb * QBB + r;
        if (i < j || i >= Tn) continue;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          s = fmaf(Qs[r][d], Kmine[threadIdx.x][d], s);
          dp = fmaf(Os[r][d], Vmine[threadIdx.x][d], dp);
        }
        const float p = expf(s * scale - Ls[r]);
        const float ds = p * (dp - Ds[r]);
#pragma unroll
        for (int d = 0; d < D; ++d) {
          dv[d] = fmaf(p, Os[r][d], dv[d]);
          dk[d] = fmaf(ds * scale, Qs[r][d], dk[d]);
        }
      }
    }
  }
  if (j < Tn) {
    T* drow = dqkv + (int64_t(b) * Tn + j) * rs + h * D;
#pragma unroll
    for (int d = 0; d < D; ++d) {
      drow[C + d] = from_f32<T>(dk[d]);
      drow[2 * C + d] = from_f32<T>(dv[d]);
    }
  }
}

// One thread per query i: dq_i = sum_{j<=i} ds_ij k_j / sqrt(D)
template <typename T, int D>
__global__ void __launch_bounds__(QBB) attn_dq_kernel(const T* __restrict__ dout,
                                                     const T* __restrict__ qkv,
                                                     const float* __restrict__ lse,
                                                     const float* __restrict__ delta, int Tn,
                                                     int C, int H, T* __restrict__ dqkv) {
  __shared__ float Ks[QBB][D + 1];
  __shared__ float Vs[QBB][D + 1];
  __shared__ float Omine[QBB][D + 1];
  const int b = blockIdx.z, h = blockIdx.y, qb = blockIdx.x;
  const int i = qb * QBB + threadIdx.x;
  const int64_t rs = 3 * int64_t(C);
  const T* base = qkv + int64_t(b) * Tn * rs + h * D;
  const T* dbase = dout + int64_t(b) * Tn * C + h * D;
  const float scale = rsqrtf(float(D));
  float q[D], dq[D];
  float L = 0.f, Dl = 0.f;
  if (i < Tn) {
#pragma unroll
    for (int d = 0; d < D; ++d) q[d] = to_f32<T>(base[int64_t(i) * rs + d]);
    L = lse[(int64_t(b) * H + h) * Tn + i];
    Dl = delta[(int64_t(b) * H + h) * Tn + i];
  }
  for (int e = threadIdx.x; e < QBB * D; e += QBB) {
    const int r = e / D, d = e % D;
    const int ii = qb * QBB + r;
    Omine[r][d] = ii < Tn ? to_f32<T>(dbase[int64_t(ii) * C + d]) : 0.f;
  }
#pragma unroll
  for (int d = 0; d < D; ++d) dq[d] = 0.f;
  for (int kb = 0; kb <= qb; ++kb) {
    __syncthreads();
    for (int e = threadIdx.x; e < QBB * D; e += QBB) {
      const int r = e / D, d = e % D;
      const int j = kb * QBB + r;
      Ks[r][d] = j < Tn ? to_f32<T>(base[int64_t(j) * rs + C + d]) : 0.f;
      Vs[r][d] = j < Tn ? to_f32<T>(base[int64_t(j) * rs + 2 * C + d]) : 0.f;
    }
    __syncthreads();
    if (i < Tn) {
      const int rmax = min(QBB, i - kb * QBB + 1);
      for (int r = 0; r < rmax; ++r) {
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          s = fmaf(q[d], Ks[r][d], s);
          dp = fmaf(Omine[threadIdx.x][d], Vs[r][d], dp);
        }
        const float p = expf(s * scale - L);
        const float ds = p * (dp - Dl);
#pragma unroll
        for (int d = 0; d < D; ++d) dq[d] = fmaf(ds * scale, Ks[r][d], dq[d]);
      }
    }
  }
  if (i < Tn) {
    T* drow = dqkv + (int64_t(b) * Tn + i) * rs + h * D;
#pragma unroll
    for (int d = 0; d < D; ++d) drow[d] = from_f32<T>(dq[d]);
  }
}

template <typename T, int D>
void fwd_d(const T* qkv, int B, int Tn, int C, int H, T* out, float* lse, cudaStream_t st) {
  dim3 grid(cdiv(Tn, QB), H, B);
  attn_fwd_kernel<T, D><<<grid, QB, 0, st>>>(qkv, Tn, C, H, out, lse);
  COUNT_LAUNCH(1);
}

template <typename T, int D>
void bwd_d(const T* dout, const T* qkv, const float* lse, const float* delta, int B, int Tn, int C,
           int H, T* dqkv, cudaStream_t st) {
  dim3 grid(cdiv(Tn, QBB), H, B);
  attn_dkdv_kernel<T, D><<<grid, QBB, 0, st>>>(dout, qkv, lse, delta, Tn, C, H, dqkv);
  COUNT_LAUNCH(1);
  attn_dq_kernel<T, D><<<grid, QBB, 0, st>>>(dout, qkv, lse, delta, Tn, C, H, dqkv);
  COUNT_LAUNCH(1);
}

}  // namespace

template <typename T>
int launch_attn_simt_fwd(const T* qkv, int B, int Tn, int C, int H, T* out, float* lse,
                         cudaStream_t st) {
  switch (C / H) {
    case 16: fwd_d<T, 16>(qkv, B, Tn, C, H, out, lse, st); break;
    case 32: fwd_d<T, 32>(qkv, B, Tn, C, H, out, lse, st); break;
    case 64: fwd_d<T, 64>(qkv, B, Tn, C, H, out, lse, st); break;
    default:
      gpt2_internal::set_error("attention: head size must be 16, 32 or 64 on this path");
      return GPT2_ERR_ARG;
  }
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

size_t attn_bwd_workspace(int B, int Tn, int H) { return size_t(B) * H * Tn * sizeof(float); }

template <typename T>
int launch_attn_simt_bwd(const T* dout, const T* qkv, const T* out, const float* lse, int B, int Tn,
                         int C, int H, T* dqkv, float* ws, cudaStream_t st) {
  const int64_t rows = int64_t(B) * H * Tn;
  attn_delta_kernel<T><<<int(cdiv64(rows, 8)), 256, 0, st>>>(dout, out, B, Tn, C, H, ws);
  COUNT_LAUNCH(1);
  switch (C / H) {
    case 16: bwd_d<T, 16>(dout, qkv, lse, ws, B, Tn, C, H, dqkv, st); break;
    case 32: bwd_d<T, 32>(dout, qkv, lse, ws, B, Tn, C, H, dqkv, st); break;
    case 64: bwd_d<T, 64>(dout, qkv, lse, ws, B, Tn, C, H, dqkv, st); break;
    default:
      gpt2_internal::set_error("attention: head size must be 16, 32 or 64 on this path");
      return GPT2_ERR_ARG;
  }
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template int launch_attn_simt_fwd<float>(const float*, int, int, int, int, float*, float*,
                                         cudaStream_t);
template int launch_attn_simt_fwd<bf16>(const bf16*, int, int, int, int, bf16*, float*,
                                        cudaStream_t);
template int launch_attn_simt_bwd<float>(const float*, const float*, const float*, const float*,
                                         int, int, int, int, float*, float*, cudaStream_t);
template int launch_attn_simt_bwd<bf16>(const bf16*, const bf16*, const bf16*, const float*, int,
                                        int, int, int, bf16*, float*, cudaStream_t);

// Dispatch: bf16 with head size 64 runs on the tcgen05 kernels (k_attn_tc.cu);
// fp32 (the parity mode) and other head sizes run on the kernels above.
int launch_attn_tc_fwd(const bf16* qkv, int B, int T, int C, int H, bf16* out, float* lse,
                       cudaStream_t st);
int launch_attn_tc_bwd(const bf16* dout, const bf16* qkv, const float* lse, const float* delta,
                       int B, int T, int C, int H, bf16* dqkv, bf16* ds, float* bias_part,
                       cudaStream_t st);

template <>
int launch_attn_fwd<float>(const float* qkv, int B, int Tn, int C, int H, float* out, float* lse,
                           cudaStream_t st) {
  return launch_attn_simt_fwd<float>(qkv, B, Tn, C, H, out, lse, st);
}
template <>
int launch_attn_fwd<bf16>(const bf16* qkv, int B, int Tn, int C, int H, bf16* out, float* lse,
                          cudaStream_t st) {
  if (attn_tc_supported(B, Tn, C, H)) return launch_attn_tc_fwd(qkv, B, Tn, C, H, out, lse, st);
  return launch_attn_simt_fwd<bf16>(qkv, B, Tn, C, H, out, lse, st);
}
template <>
int launch_attn_bwd<float>(const float* dout, const float* qkv, const float* out, const float* lse,
                           int B, int Tn, int C, int H, float* dqkv, float* ws, cudaStream_t st) {
  return launch_attn_simt_bwd<float>(dout, qkv, out, lse, B, Tn, C, H, dqkv, ws, st);
}
int attn_bias_parts(int T) { return int(cdiv64(T, 128)); }
bool attn_bias_parts_written(int B, int T, int C, int H, const bf16* ds) {
  return ds && H >= 1 && C % H == 0 && attn_tc_supported(B, T, C, H);
}
int launch_attn_bwd_ds(const bf16* dout, const bf16* qkv, const bf16* out, const float* lse, int B,
                       int Tn, int C, int H, bf16* dqkv, float* ws, bf16* ds, cudaStream_t st,
                       float* bias_part) {
  if (!attn_tc_supported(B, Tn, C, H))
    return launch_attn_simt_bwd<bf16>(dout, qkv, out, lse, B, Tn, C, H, dqkv, ws, st);
  const int64_t rows = int64_t(B) * H * Tn;
  attn_delta64_kernel<<<int(cdiv64(rows * 8, 256)), 256, 0, st>>>(dout, out, B, Tn, C, H, ws);
  COUNT_LAUNCH(1);
  return launch_attn_tc_bwd(dout, qkv, lse, ws, B, Tn, C, H, dqkv, ds, bias_part, st);
}
template <>
int launch_attn_bwd<bf16>(const bf16* dout, const bf16* qkv, const bf16* out, const float* lse,
                          int B, int Tn, int C, int H, bf16* dqkv, float* ws, cudaStream_t st) {
  return launch_attn_bwd_ds(dout, qkv, out, lse, B, Tn, C, H, dqkv, ws, nullptr, st);
}
size_t attn_bwd_workspace_total(int B, int T, int C, int H, bool bf16_path) {
  const size_t delta = attn_bwd_workspace(B, T, H);
  if (!bf16_path || H < 1 || C % H || !attn_tc_supported(B, T, C, H)) return delta;
  return (delta + 1023) / 1024 * 1024 + attn_tc_ds_bytes(B, T, H);
}
