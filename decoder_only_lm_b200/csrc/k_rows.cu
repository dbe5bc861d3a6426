// Memory-bound kernels of the training step: batch slicing, embedding
// forward/backward, LayerNorm forward/backward, bias-gradient column sums,
// cross-entropy rows, gradient norm and the fused clip+AdamW pass.
//
// Sources: [CH28] "Chapter 28: data, evaluation and recovery" §28.3 (B*T+1
// slicing); [ZERO] "GPT training" (Zero docs): Embedding, Transformer Block
// (pre-LN), output layer; [CS336] "CS336 from scratch — pretraining" §1
// cross-entropy (max subtracted), §2 AdamW (bias correction folded into the
// step size, decay before the update) and gradient clipping
// (min(1, c/(n+1e-6))); [LECTURE] "Andrej Karpathy: reproducing GPT-2 from
// scratch": tied head gradients add, decay on matrices only, fused AdamW.
//
// All reductions are in a fixed order (no floating-point atomics), so two runs
// on the same inputs give identical bits.

#include <algorithm>

#include "kernels.h"
#include "tc_common.cuh"

namespace {

constexpr int kThreads = 256;

// ------------------------------------------------------------ batch slicing
// The window at the device cursor *cur; a window that would run past the
// stream (len tokens) is not read: its ids become 0 and window_bad is set,
// which skips the optimizer update and is reported by the next status read.
__global__ void slice_batch_cursor_kernel(const uint16_t* __restrict__ s, int64_t len,
                                          const int64_t* __restrict__ cur, int64_t n,
                                          int32_t* __restrict__ x, int32_t* __restrict__ y,
                                          DevStatus* status) {
  const int64_t off = *cur;
  const bool ok = off >= 0 && off + n + 1 <= len;
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  if (!ok) {
    if (i == 0) atomicExch(&status->window_bad, 1);
    x[i] = 0;
    y[i] = 0;
    return;
  }
  x[i] = int32_t(s[off + i]);
  y[i] = int32_t(s[off + i + 1]);
}
__global__ void advance_cursor_kernel(int64_t* cur, int64_t stride) { *cur += stride; }

__global__ void slice_batch_kernel(const uint16_t* __restrict__ s, int64_t off, int64_t n,
                                   int32_t* __restrict__ x, int32_t* __restrict__ y) {
  int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i < n) {
    x[i] = int32_t(s[off + i]);
    y[i] = int32_t(s[off + i + 1]);
  }
}

// ------------------------------------------------------------ embedding
// out[m, :] = wte[x_m, :] + wpe[t_m, :] in fp32; ids outside [0, V) are
// recorded in the status word and read as id 0 so no access leaves the table.
__global__ void embed_fwd_kernel(const int32_t* __restrict__ x, const int32_t* __restrict__ y,
                                 const float* __restrict__ wte, const float* __restrict__ wpe,
                                 int T, int C, int V, int64_t M, float* __restrict__ out,
                                 DevStatus* status, int pos0, const int* __restrict__ d_step) {
  int64_t m = blockIdx.x;
  if (m >= M) return;
  int id = x[m];
  if (threadIdx.x == 0) {
    int yy = y ? y[m] : 0;
    if (id < 0 || id >= V || yy < 0 || yy >= V) atomicExch(&status->token_bad, 1);
  }
  if (id < 0 || id >= V) id = 0;
  const int t = pos0 + (d_step ? *d_step : 0) + int(m % T);
  const float* a = wte + int64_t(id) * C;
  const float* b = wpe + int64_t(t) * C;
  float* o = out + m * C;
  if ((C & 3) == 0) {
    for (int c = threadIdx.x * 4; c < C; c += blockDim.x * 4) {
      float4 u = *reinterpret_cast<const float4*>(a + c);
      float4 w = *reinterpret_cast<const float4*>(b + c);
      *reinterpret_cast<float4*>(o + c) = make_float4(u.x + w.x, u.y + w.y, u.z + w.z, u.w + w.w);
    }
  } else {
    for (int c = threadIdx.x; c < C; c += blockDim.x) o[c] = a[c] + b[c];
  }
}

// Embedding backward, deterministic:
//  1. keys_m = (x_m << 32) | m, padded with ~0 to a power of two, bitonic-sorted
//     (ties impossible: m is unique), so equal ids are grouped in index order;
//  2. pieces: every run of equal ids inside an aligned group of 32 sorted
//     entries is summed (rows of dh in index order) into piece[first entry];
//  3. every run start adds its pieces (stride 32) in order into dwte[id].
constexpr int kSortChunk = 2048;  // keys sorted in shared memory by one block
constexpr int kPiece = 32;

__device__ __forceinline__ void cmp_swap(uint64_t& a, uint64_t& b, bool up) {
  if ((a > b) == up) {
    uint64_t t = a;
    a = b;
    b = t;
  }
}

__global__ void make_keys_kernel(const int32_t* __restrict__ x, int64_t M, int64_t Mp, int V,
                                 uint64_t* __restrict__ keys) {
  int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= Mp) return;
  if (i < M) {
    int id = x[i];
    if (id < 0 || id >= V) id = 0;  // recorded by the forward; keep accesses in range
    keys[i] = (uint64_t(uint32_t(id)) << 32) | uint64_t(i);
  } else {
    keys[i] = ~uint64_t(0);
  }
}

// Stages k = 2 .. min(kSortChunk, Mp) of the bitonic network inside one chunk,
// directions taken from the global index.  `k_from` > 2 restarts at a merge
// level (then only the j < kSortChunk steps of level k_from are done).
__global__ void bitonic_chunk_kernel(uint64_t* __restrict__ keys, int64_t Mp, int64_t k_only) {
  __shared__ uint64_t s[kSortChunk];
  const int64_t base = int64_t(blockIdx.x) * kSortChunk;
  const int n = int(min64(kSortChunk, Mp));
  for (int i = threadIdx.x; i < n; i += blockDim.x) s[i] = keys[base + i];
  __syncthreads();
  int64_t k_lo = 2, k_hi = n;
  if (k_only) k_lo = k_hi = k_only;
  for (int64_t k = k_lo; k <= k_hi; k <<= 1) {
    for (int j = int(min64(k >> 1, n >> 1)); j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < n / 2; t += blockDim.x) {
        int i = 2 * j * (t / j) + (t % j);
        int64_t gi = base + i;
        cmp_swap(s[i], s[i + j], (gi & k) == 0);
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) keys[base + i] = s[i];
}

__global__ void bitonic_global_kernel(uint64_t* __restrict__ keys, int64_t Mp, int64_t j,
                                      int64_t k) {
  int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (t >= Mp / 2) return;
  int64_t i = 2 * j * (t / j) + (t % j);
  uint64_t a = keys[i], b = keys[i + j];
  bool up = (i & k) == 0;
  if ((a > b) == up) {
    keys[i] = b;
    keys[i + j] = a;
  }
}

__global__ void embed_pieces_kernel(const uint64_t* __restrict__ keys, const float* __restrict__ dh,
                                    int64_t M, int C, float* __restrict__ piece) {
  const int64_t r0 = int64_t(blockIdx.x) * kPiece;
  const int64_t r1 = min64(M, r0 + kPiece);
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float acc = 0.f;
    int64_t start = r0;
    uint32_t cur = uint32_t(keys[r0] >> 32);
    for (int64_t r = r0; r < r1; ++r) {
      uint64_t kk = keys[r];
      uint32_t id = uint32_t(kk >> 32);
      if (id != cur) {
        piece[start * C + c] = acc;
        acc = 0.f;
        start = r;
        cur = id;
      }
      acc += dh[int64_t(uint32_t(kk)) * C + c];
    }
    piece[start * C + c] = acc;
  }
}

__global__ void embed_runs_kernel(const uint64_t* __restrict__ keys, const float* __restrict__ piece,
                                  int64_t M, int C, float* __restrict__ dwte) {
  const int64_t r0 = int64_t(blockIdx.x) * kPiece;
  const int64_t r1 = min64(M, r0 + kPiece);
  for (int64_t r = r0; r < r1; ++r) {
    const uint32_t id = uint32_t(keys[r] >> 32);
    if (r > 0 && uint32_t(keys[r - 1] >> 32) == id) continue;  // not a run start
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      float acc = piece[r * C + c];
      for (int64_t q = (r / kPiece + 1) * kPiece; q < M && uint32_t(keys[q] >> 32) == id; q += kPiece)
        acc += piece[q * C + c];
      dwte[int64_t(id) * C + c] += acc;
    }
  }
}

// dwpe[t, c] (+)= sum_b dh[b, t, c]
__global__ void embed_wpe_kernel(const float* __restrict__ dh, int B, int T, int C,
                                 float* __restrict__ dwpe, int accumulate) {
  int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= int64_t(T) * C) return;
  float acc = 0.f;
  for (int b = 0; b < B; ++b) acc += dh[int64_t(b) * T * C + i];
  dwpe[i] = accumulate ? dwpe[i] + acc : acc;
}

// ------------------------------------------------------------ LayerNorm
constexpr int kLnMaxPerLane = 32;  // C <= 1024

template <typename OutT>
__global__ void layernorm_fwd_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                     const float* __restrict__ b, OutT* __restrict__ y,
                                     float* __restrict__ mean, float* __restrict__ rstd,
                                     int64_t M, int C, float eps) {
  const int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* xr = x + row * C;
  float v[kLnMaxPerLane];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxPerLane; ++i) {
    int c = lane + 32 * i;
    v[i] = c < C ? xr[c] : 0.f;
    s += v[i];
  }
  const float mu = warp_sum(s) / float(C);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxPerLane; ++i) {
    int c = lane + 32 * i;
    float d = c < C ? v[i] - mu : 0.f;
    q += d * d;
  }
  const float rs = rsqrtf(warp_sum(q) / float(C) + eps);
  OutT* yr = y + row * C;
#pragma unroll
  for (int i = 0; i < kLnMaxPerLane; ++i) {
    int c = lane + 32 * i;
    if (c < C) yr[c] = from_f32<OutT>((v[i] - mu) * rs * g[c] + b[c]);
  }
  if (lane == 0) {
    if (mean) mean[row] = mu;
    if (rstd) rstd[row] = rs;
  }
}

// One block = 8 warps; each warp takes rows row0 + warp, row0 + warp + 8, ...
// (kLnRowsPerBlock rows per block).  dx is ADDED to `dx` (the residual-stream
// gradient) and, when dx_copy is given, the new dx is also stored rounded to
// CopyT.  Column partials of dgamma/dbeta go to ws[block][2C].
constexpr int kLnRowsPerBlock = 64;

template <typename DyT, typename CopyT>
__global__ void layernorm_bwd_kernel(const DyT* __restrict__ dy, const float* __restrict__ x,
                                     const float* __restrict__ mean, const float* __restrict__ rstd,
                                     const float* __restrict__ g, int64_t M, int C,
                                     float* __restrict__ dx, CopyT* __restrict__ dx_copy,
                                     float* __restrict__ ws) {
  __shared__ float red[8][2][kLnMaxPerLane * 32 / 8];  // reused per column slice
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  float pg[kLnMaxPerLane], pb[kLnMaxPerLane];
#pragma unroll
  for (int i = 0; i < kLnMaxPerLane; ++i) pg[i] = pb[i] = 0.f;
  const int64_t row0 = int64_t(blockIdx.x) * kLnRowsPerBlock;
  for (int rr = warp; rr < kLnRowsPerBlock; rr += 8) {
    const int64_t row = row0 + rr;
    if (row >= M) break;
    const float mu = mean[row], rs = rstd[row];
    float xh[kLnMaxPerLane], dyv[kLnMaxPerLane];
    float a = 0.f, bsum = 0.f;
#pragma unroll
    for (int i = 0; i < kLnMaxPerLane; ++i) {
      int c = lane + 32 * i;
      if (c < C) {
        xh[i] = (x[row * C + c] - mu) * rs;
        dyv[i] = to_f32<DyT>(dy[row * C + c]);
        float dxh = dyv[i] * g[c];
        a += dxh;
        bsum += dxh * xh[i];
        pg[i] += dyv[i] * xh[i];
        pb[i] += dyv[i];
      } else {
        xh[i] = dyv[i] = 0.f;
      }
    }
    a = warp_sum(a) / float(C);
    bsum = warp_sum(bsum) / float(C);
#pragma unroll
    for (int i = 0; i < kLnMaxPerLane; ++i) {
      int c = lane + 32 * i;
      if (c < C) {
        float dxh = dyv[i] * g[c];
        float nv = dx[row * C + c] + rs * (dxh - a - xh[i] * bsum);
        dx[row * C + c] = nv;
        if (dx_copy) dx_copy[row * C + c] = from_f32<CopyT>(nv);
      }
    }
  }
  // Reduce the 8 warps' column partials in a fixed order, 128 columns at a time.
  float* out = ws + int64_t(blockIdx.x) * 2 * C;
#pragma unroll
  for (int i0 = 0; i0 < kLnMaxPerLane; i0 += 4) {
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      red[warp][0][i * 32 + lane] = pg[i0 + i];
      red[warp][1][i * 32 + lane] = pb[i0 + i];
    }
    __syncthreads();
    if (threadIdx.x < 128) {
      const int i = threadIdx.x / 32, l = threadIdx.x & 31;
      const int c = l + 32 * (i0 + i);
      if (c < C) {
        float sg = 0.f, sb = 0.f;
        for (int w = 0; w < 8; ++w) {
          sg += red[w][0][threadIdx.x];
          sb += red[w][1][threadIdx.x];
        }
        out[c] = sg;
        out[C + c] = sb;
      }
    }
  }
}

// out[c] (+)= sum over `parts` rows of ws[., c], in order.
__global__ void reduce_partials_kernel(const float* __restrict__ ws, int parts, int n,
                                       float* __restrict__ out, int accumulate) {
  int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n) return;
  float acc = 0.f;
  for (int p = 0; p < parts; ++p) acc += ws[int64_t(p) * n + c];
  out[c] = accumulate ? out[c] + acc : acc;
}

__global__ void reduce_ln_partials_kernel(const float* __restrict__ ws, int parts, int C,
                                          float* __restrict__ dg, float* __restrict__ db,
                                          int accumulate) {
  int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= 2 * C) return;
  float acc = 0.f;
  for (int p = 0; p < parts; ++p) acc += ws[int64_t(p) * 2 * C + c];
  float* o = c < C ? dg + c : db + (c - C);
  *o = accumulate ? *o + acc : acc;
}

// Vectorised LayerNorm for C = 128 * NV, one warp per row: lane l owns the
// float4 column groups 4l + 128i of the row.
template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&v)[4]) {
  float4 f = *reinterpret_cast<const float4*>(p);
  v[0] = f.x;
  v[1] = f.y;
  v[2] = f.z;
  v[3] = f.w;
}
template <>
__device__ __forceinline__ void load4<bf16>(const bf16* p, float (&v)[4]) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
  float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
  v[0] = a.x;
  v[1] = a.y;
  v[2] = b.x;
  v[3] = b.y;
}
template <typename T>
__device__ __forceinline__ void store4(T* p, const float (&v)[4]);
template <>
__device__ __forceinline__ void store4<float>(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16* p, const float (&v)[4]) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// Rows reach shared memory by bulk copies.  A block is kLnWarps warps and
// the grid is persistent (a few blocks per SM); warp w of the grid takes rows
// w, w + W, w + 2W, ... (W warps in the grid) and keeps a ring of S row
// buffers of its own, each filled by one bulk copy S rows ahead of the row
// it computes, so every warp has several rows of HBM reads in flight while
// it reduces and writes the current one.  A wait that expires sets the error
// word; the warp then computes nothing more but waits (bounded) for the
// copies it has issued before it leaves.
constexpr int kLnWarps = 8;
constexpr int kLnMaxBlocks = 1024;  // grid cap (the backward's partial rows)

// per-warp ring: S mbarriers and S stage buffers of `stage` bytes
struct LnRing {
  uint32_t bar0, buf0;
  uint8_t* buf;
  int S;
  uint32_t stage;
  __device__ uint32_t bar(int64_t k) const { return bar0 + 8u * uint32_t(k % S); }
  __device__ uint32_t parity(int64_t k) const { return uint32_t((k / S) & 1); }
  __device__ uint8_t* at(int64_t k) const { return buf + uint32_t(k % S) * stage; }
  __device__ uint32_t at_s(int64_t k) const { return buf0 + uint32_t(k % S) * stage; }
};
// shared memory: kLnWarps * S barriers (padded to 128 bytes), then the
// stage buffers [warp][stage]
__host__ __device__ constexpr size_t ln_bar_bytes(int S) {
  return (size_t(kLnWarps) * S * 8 + 127) / 128 * 128;
}
__device__ __forceinline__ LnRing ln_ring(uint8_t* smem, int S, uint32_t stage, int warp,
                                          int lane) {
  LnRing r;
  r.S = S;
  r.stage = stage;
  r.bar0 = tc::smem_u32(smem) + uint32_t(warp * S * 8);
  r.buf = smem + ln_bar_bytes(S) + size_t(warp) * S * stage;
  r.buf0 = tc::smem_u32(r.buf);
  if (lane == 0) {
    for (int i = 0; i < S; ++i) tc::mbar_init(r.bar0 + 8u * i, 1);
    tc::fence_mbar_init();
  }
  __syncwarp();
  return r;
}
// waits (bounded) for the copies of rows [from, to) of the ring
__device__ __forceinline__ void ln_drain(const LnRing& r, int64_t from, int64_t to, int* err,
                                         int where) {
  for (int64_t k = from; k < to; ++k) tc::mbar_wait(r.bar(k), r.parity(k), err, where);
}

template <int NV, typename OutT>
__global__ void __launch_bounds__(kLnWarps * 32) layernorm_fwd_staged_kernel(
    const float* __restrict__ x, const float* __restrict__ g, const float* __restrict__ b,
    OutT* __restrict__ y, float* __restrict__ mean, float* __restrict__ rstd, int64_t M,
    float eps, int S, int* err) {
  constexpr int C = NV * 128;
  constexpr uint32_t RB = C * 4;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t W = int64_t(gridDim.x) * kLnWarps;
  const int64_t w0 = int64_t(blockIdx.x) * kLnWarps + warp;
  const int64_t nk = w0 < M ? (M - 1 - w0) / W + 1 : 0;  // rows of this warp
  const LnRing ring = ln_ring(smem, S, RB, warp, lane);
  auto issue = [&](int64_t k) {
    tc::mbar_expect_tx(ring.bar(k), RB);
    tc::bulk_load_1d(ring.at_s(k), x + (w0 + k * W) * C, RB, ring.bar(k));
  };
  if (lane == 0)
    for (int64_t k = 0; k < nk && k < S; ++k) issue(k);
  float gg[NV][4], bb[NV][4];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    load4<float>(g + 4 * lane + 128 * i, gg[i]);
    load4<float>(b + 4 * lane + 128 * i, bb[i]);
  }
  int64_t k = 0;
  for (; k < nk; ++k) {
    if (!__all_sync(0xffffffffu, tc::mbar_wait(ring.bar(k), ring.parity(k), err, 41))) break;
    const float* xr = reinterpret_cast<const float*>(ring.at(k));
    float v[NV][4];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      load4<float>(xr + 4 * lane + 128 * i, v[i]);
      sum += (v[i][0] + v[i][1]) + (v[i][2] + v[i][3]);
    }
    const float mu = warp_sum(sum) / float(C);  // every lane's reads are done
    if (lane == 0 && k + S < nk) issue(k + S);
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float dd = v[i][j] - mu;
        q += dd * dd;
      }
    const float rs = rsqrtf(warp_sum(q) / float(C) + eps);
    const int64_t row = w0 + k * W;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      float o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = (v[i][j] - mu) * rs * gg[i][j] + bb[i][j];
      store4<OutT>(y + row * C + 4 * lane + 128 * i, o);
    }
    if (lane == 0) {
      if (mean) mean[row] = mu;
      if (rstd) rstd[row] = rs;
    }
  }
  if (k < nk) ln_drain(ring, k, k + S < nk ? k + S : nk, err, 42);
}

// LayerNorm backward, C = 128 * NV: dx is ADDED to `dx` (the residual-stream
// gradient) and, when dx_copy is given, the new dx is also stored rounded to
// CopyT.  A stage holds the row's x, dx and dy.  Each warp keeps its column
// partials of dgamma, dbeta and (want_sum) of the updated dx in registers; at
// the end the block's warps are summed in warp order and the block's partial
// goes to ws[block][parts][C] (parts = 2 or 3).
template <int NV, typename DyT, typename CopyT>
__global__ void __launch_bounds__(kLnWarps * 32, 1) layernorm_bwd_staged_kernel(
    const DyT* __restrict__ dy, const float* __restrict__ x, const float* __restrict__ mean,
    const float* __restrict__ rstd, const float* __restrict__ g, int64_t M,
    float* __restrict__ dx, CopyT* __restrict__ dx_copy, float* __restrict__ ws, int want_sum,
    int S, int* err) {
  constexpr int C = NV * 128;
  constexpr uint32_t RB = C * 4, DB = C * sizeof(DyT), ST = 2 * RB + DB;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t W = int64_t(gridDim.x) * kLnWarps;
  const int64_t w0 = int64_t(blockIdx.x) * kLnWarps + warp;
  const int64_t nk = w0 < M ? (M - 1 - w0) / W + 1 : 0;
  const LnRing ring = ln_ring(smem, S, ST, warp, lane);
  auto issue = [&](int64_t k) {
    const int64_t row = w0 + k * W;
    const uint32_t s = ring.at_s(k), bar = ring.bar(k);
    tc::mbar_expect_tx(bar, ST);
    tc::bulk_load_1d(s, x + row * C, RB, bar);
    tc::bulk_load_1d(s + RB, dx + row * C, RB, bar);
    tc::bulk_load_1d(s + 2 * RB, dy + row * C, DB, bar);
  };
  if (lane == 0)
    for (int64_t k = 0; k < nk && k < S; ++k) issue(k);
  float gam[NV][4], pg[NV][4], pb[NV][4], ps[NV][4];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    load4<float>(g + 4 * lane + 128 * i, gam[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) pg[i][j] = pb[i][j] = ps[i][j] = 0.f;
  }
  float mu = 0.f, rs = 0.f;
  if (nk > 0) {
    mu = mean[w0];
    rs = rstd[w0];
  }
  int64_t k = 0;
  for (; k < nk; ++k) {
    const int64_t row = w0 + k * W;
    float mu_n = 0.f, rs_n = 0.f;  // the next row's statistics, loaded early
    if (k + 1 < nk) {
      mu_n = mean[row + W];
      rs_n = rstd[row + W];
    }
    if (!__all_sync(0xffffffffu, tc::mbar_wait(ring.bar(k), ring.parity(k), err, 43))) break;
    const float* xr = reinterpret_cast<const float*>(ring.at(k));
    const float* dxr = xr + C;
    const DyT* dyr = reinterpret_cast<const DyT*>(xr + 2 * C);
    float a = 0.f, bsum = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = 4 * lane + 128 * i;
      float xh[4], d[4];
      load4<float>(xr + c, xh);
      load4<DyT>(dyr + c, d);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xh[j] = (xh[j] - mu) * rs;
        const float dxh = d[j] * gam[i][j];
        a += dxh;
        bsum += dxh * xh[j];
        pg[i][j] += d[j] * xh[j];
        pb[i][j] += d[j];
      }
    }
    a = warp_sum(a) / float(C);
    bsum = warp_sum(bsum) / float(C);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = 4 * lane + 128 * i;
      float xh[4], d[4], cur[4];
      load4<float>(xr + c, xh);
      load4<DyT>(dyr + c, d);
      load4<float>(dxr + c, cur);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xh[j] = (xh[j] - mu) * rs;
        cur[j] += rs * (d[j] * gam[i][j] - a - xh[j] * bsum);
        ps[i][j] += cur[j];
      }
      store4<float>(dx + row * C + c, cur);
      if (dx_copy) store4<CopyT>(dx_copy + row * C + c, cur);
    }
    __syncwarp();  // every lane has read the stage
    if (lane == 0 && k + S < nk) issue(k + S);
    mu = mu_n;
    rs = rs_n;
  }
  if (k < nk) ln_drain(ring, k, k + S < nk ? k + S : nk, err, 44);
  // the block's column partials, summed over its warps in warp order; the
  // stage buffers are free now (every copy has landed)
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem + ln_bar_bytes(S));  // [kLnWarps][C]
  const int parts = want_sum ? 3 : 2;
  float* out = ws + int64_t(blockIdx.x) * parts * C;
  for (int part = 0; part < parts; ++part) {
#pragma unroll
    for (int i = 0; i < NV; ++i)
      store4<float>(red + warp * C + 4 * lane + 128 * i,
                    part == 0 ? pg[i] : part == 1 ? pb[i] : ps[i]);
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kLnWarps; ++w) t += red[w * C + c];
      out[part * C + c] = t;
    }
    __syncthreads();
  }
}

// out[c] (+)= sum_p ws[p][c] for c < n (c >= split goes to out1[c - split],
// c >= 2 split to out2[c - 2 split]),
// in a fixed order: 8 interleaved row slices per column, then the 8 slices.
__device__ __forceinline__ void reduce_rows_body(const float* __restrict__ ws, int parts, int n,
                                                 float* __restrict__ out0,
                                                 float* __restrict__ out1, int split,
                                                 int accumulate, float* __restrict__ out2) {
  __shared__ float sh[8][33];
  const int cx = threadIdx.x & 31, ry = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + cx;
  float acc = 0.f;
  if (c < n)
    for (int p = ry; p < parts; p += 8) acc += ws[int64_t(p) * n + c];
  sh[ry][cx] = acc;
  __syncthreads();
  if (ry == 0 && c < n) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += sh[k][cx];
    float* o = c < split ? out0 + c : c < 2 * split ? out1 + (c - split) : out2 + (c - 2 * split);
    *o = accumulate ? *o + t : t;
  }
}
__global__ void __launch_bounds__(256) reduce_rows_kernel(const float* __restrict__ ws, int parts,
                                                          int n, float* __restrict__ out0,
                                                          float* __restrict__ out1, int split,
                                                          int accumulate,
                                                          float* __restrict__ out2 = nullptr) {
  reduce_rows_body(ws, parts, n, out0, out1, split, accumulate, out2);
}
// Up to kRowSumMax such sums in one launch: blockIdx.y picks the sum, the
// same arithmetic in the same order as reduce_rows_kernel.
constexpr int kRowSumMax = 64;
struct RowSumBatch {
  RowSum s[kRowSumMax];
};
__global__ void __launch_bounds__(256) reduce_rows_batch_kernel(const __grid_constant__ RowSumBatch b) {
  const RowSum& r = b.s[blockIdx.y];
  if (int(blockIdx.x) * 32 >= r.n) return;  // the whole block: this sum has fewer columns
  reduce_rows_body(r.p, r.parts, r.n, r.out0, r.out1, r.split, r.accumulate, r.out2);
}

// ------------------------------------------------------------ bias-gradient column sums
constexpr int kColRows = 256;  // rows per partial

template <typename InT>
__global__ void colsum_partial_kernel(const InT* __restrict__ in, int64_t M, int N,
                                      float* __restrict__ ws) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const int64_t r0 = int64_t(blockIdx.y) * kColRows;
  const int64_t r1 = min64(M, r0 + kColRows);
  float acc = 0.f;
  for (int64_t r = r0; r < r1; ++r) acc += to_f32<InT>(in[r * N + n]);
  ws[int64_t(blockIdx.y) * N + n] = acc;
}

// ------------------------------------------------------------ cross-entropy rows
// lse_r = max_v z + log sum_v exp(z - max);  row_loss_r = lse_r - z[r, y_r].
__global__ void ce_rows_fwd_kernel(const float* __restrict__ z, const int32_t* __restrict__ y,
                                   int Vp, float* __restrict__ lse, float* __restrict__ row_loss) {
  __shared__ float sh[32];
  const int r = blockIdx.x;
  const float* zr = z + int64_t(r) * Vp;
  float mx = -INFINITY;
  for (int v = threadIdx.x; v < Vp; v += blockDim.x) mx = fmaxf(mx, zr[v]);
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x / 32] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < blockDim.x / 32 ? sh[threadIdx.x] : -INFINITY;
    t = warp_max(t);
    if (threadIdx.x == 0) sh[0] = t;
  }
  __syncthreads();
  mx = sh[0];
  __syncthreads();
  float s = 0.f;
  for (int v = threadIdx.x; v < Vp; v += blockDim.x) s += expf(zr[v] - mx);
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < int(blockDim.x / 32); ++w) t += sh[w];
    float l = mx + logf(t);
    lse[r] = l;
    row_loss[r] = l - zr[y[r]];
  }
}

template <typename OutT>
__global__ void ce_rows_bwd_kernel(const float* __restrict__ z, const float* __restrict__ lse,
                                   const int32_t* __restrict__ y, int Vp, float scale,
                                   OutT* __restrict__ dz) {
  const int r = blockIdx.x;
  const float* zr = z + int64_t(r) * Vp;
  OutT* dr = dz + int64_t(r) * Vp;
  const float l = lse[r];
  const int t = y[r];
  for (int v = threadIdx.x; v < Vp; v += blockDim.x)
    dr[v] = from_f32<OutT>(scale * (expf(zr[v] - l) - (v == t ? 1.f : 0.f)));
}

// out = mean of v[0..n), fixed order (one block).
__global__ void mean_kernel(const float* __restrict__ v, int64_t n, float* __restrict__ out) {
  __shared__ double sh[kThreads];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) acc += double(v[i]);
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = float(sh[0] / double(n));
}

// ------------------------------------------------------------ gradient norm, clip + AdamW
constexpr int kNormBlocks = 1024;

__global__ void sumsq_kernel(const float* __restrict__ g, int64_t n, double* __restrict__ ws) {
  __shared__ double sh[kThreads];
  const int64_t chunk = (n + kNormBlocks - 1) / kNormBlocks;
  const int64_t a = int64_t(blockIdx.x) * chunk, e = min64(n, a + chunk);
  double acc = 0.0;
  for (int64_t i = a + threadIdx.x; i < e; i += blockDim.x) {
    float v = g[i];
    acc += double(v) * double(v);
  }
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) ws[blockIdx.x] = sh[0];
}

__global__ void norm_finalize_kernel(const double* __restrict__ ws, float* __restrict__ norm) {
  __shared__ double sh[kNormBlocks];
  for (int i = threadIdx.x; i < kNormBlocks; i += blockDim.x) sh[i] = ws[i];
  __syncthreads();
  for (int s = kNormBlocks / 2; s > 0; s >>= 1) {
    for (int i = threadIdx.x; i < s; i += blockDim.x) sh[i] += sh[i + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) norm[0] = float(sqrt(sh[0]));
}

// One fused pass.  Elements [0, n_decay) belong to 2-D tensors (decayed).
// Every thread reads the same status and norm, so either all of them update
// or none does; the step counter is advanced by step_advance_kernel.
__global__ void clip_adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                  float* __restrict__ m, float* __restrict__ v,
                                  bf16* __restrict__ pb, int64_t n, int64_t n_decay,
                                  const float* __restrict__ norm, const DevStatus* __restrict__ st,
                                  float lr_arg, const float* __restrict__ lr_dev, float b1,
                                  float b2, float eps, float wd, float max_norm) {
  const float nrm = *norm;
  const float lr = lr_dev ? *lr_dev : lr_arg;  // lr_dev: set on the device between graph replays
  if (st->token_bad || st->window_bad || !isfinite(nrm)) return;
  const int t = st->step + 1;
  const float s = fminf(1.f, max_norm / (nrm + 1e-6f));
  const float alpha = lr * sqrtf(1.f - powf(b2, float(t))) / (1.f - powf(b1, float(t)));
  const float dec = 1.f - lr * wd;
  const int64_t n4 = n / 4;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    float4 P = reinterpret_cast<float4*>(p)[i];
    float4 G = reinterpret_cast<const float4*>(g)[i];
    float4 Mo = reinterpret_cast<float4*>(m)[i];
    float4 Vo = reinterpret_cast<float4*>(v)[i];
    const float d = (i * 4 < n_decay) ? dec : 1.f;  // n_decay is a multiple of 4
    float* pp = &P.x;
    float* gg = &G.x;
    float* mm = &Mo.x;
    float* vv = &Vo.x;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float gk = s * gg[k];
      mm[k] = b1 * mm[k] + (1.f - b1) * gk;
      vv[k] = b2 * vv[k] + (1.f - b2) * gk * gk;
      pp[k] = pp[k] * d;
      pp[k] -= alpha * mm[k] / (sqrtf(vv[k]) + eps);
    }
    reinterpret_cast<float4*>(p)[i] = P;
    reinterpret_cast<float4*>(m)[i] = Mo;
    reinterpret_cast<float4*>(v)[i] = Vo;
    if (pb) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(P.x, P.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(P.z, P.w);
      reinterpret_cast<__nv_bfloat162*>(pb)[2 * i] = lo;
      reinterpret_cast<__nv_bfloat162*>(pb)[2 * i + 1] = hi;
    }
  }
}

__global__ void step_advance_kernel(const float* __restrict__ norm, DevStatus* st) {
  if (st->token_bad || st->window_bad) return;
  if (!isfinite(*norm)) {
    st->nonfinite = 1;
    return;
  }
  st->step += 1;
}

__global__ void to_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

__global__ void fill_kernel(float* __restrict__ p, float v, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x)
    p[i] = v;
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  int cap = gpt2_internal::sm_count() * 8;
  return int(max64(1, min64(b, cap)));
}

int64_t next_pow2(int64_t n) {
  int64_t p = 1;
  while (p < n) p <<= 1;
  return p;
}

}  // namespace

// ============================================================ launchers

int launch_slice_batch_cursor(const uint16_t* s, int64_t len, const int64_t* cur, int64_t n,
                              int32_t* x, int32_t* y, DevStatus* status, cudaStream_t st) {
  if (n <= 0) return GPT2_OK;
  slice_batch_cursor_kernel<<<int(cdiv64(n, kThreads)), kThreads, 0, st>>>(s, len, cur, n, x, y,
                                                                          status);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_advance_cursor(int64_t* cur, int64_t stride, cudaStream_t st) {
  advance_cursor_kernel<<<1, 1, 0, st>>>(cur, stride);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_slice_batch(const uint16_t* s, int64_t off, int64_t n, int32_t* x, int32_t* y,
                       cudaStream_t st) {
  if (n <= 0) return GPT2_OK;
  slice_batch_kernel<<<int(cdiv64(n, kThreads)), kThreads, 0, st>>>(s, off, n, x, y);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_embed_fwd(const int32_t* x, const int32_t* y, const float* wte, const float* wpe, int B,
                     int T, int C, int V, float* out, DevStatus* status, cudaStream_t st,
                     int pos0, const int* d_step) {
  const int64_t M = int64_t(B) * T;
  embed_fwd_kernel<<<int(M), 192, 0, st>>>(x, y, wte, wpe, T, C, V, M, out, status, pos0, d_step);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

size_t embed_bwd_workspace(int64_t M, int C) {
  int64_t Mp = max64(next_pow2(M), 2);
  return size_t(Mp) * sizeof(uint64_t) + size_t(M) * C * sizeof(float) + 256;
}

int launch_embed_bwd(const int32_t* x, const float* dh, int B, int T, int C, int V, float* dwte,
                     float* dwpe, int wpe_accumulate, void* ws, cudaStream_t st) {
  const int64_t M = int64_t(B) * T;
  const int64_t Mp = max64(next_pow2(M), 2);
  uint64_t* keys = reinterpret_cast<uint64_t*>(ws);
  float* piece = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) +
                                          ((size_t(Mp) * sizeof(uint64_t) + 255) / 256) * 256);
  make_keys_kernel<<<int(cdiv64(Mp, kThreads)), kThreads, 0, st>>>(x, M, Mp, V, keys);
  COUNT_LAUNCH(1);
  const int nchunks = int(max64(1, Mp / kSortChunk));
  bitonic_chunk_kernel<<<nchunks, 1024, 0, st>>>(keys, Mp, 0);
  COUNT_LAUNCH(1);
  for (int64_t k = 2 * kSortChunk; k <= Mp; k <<= 1) {
    for (int64_t j = k >> 1; j >= kSortChunk; j >>= 1) {
      bitonic_global_kernel<<<int(cdiv64(Mp / 2, kThreads)), kThreads, 0, st>>>(keys, Mp, j, k);
      COUNT_LAUNCH(1);
    }
    bitonic_chunk_kernel<<<nchunks, 1024, 0, st>>>(keys, Mp, k);
    COUNT_LAUNCH(1);
  }
  const int nb = int(cdiv64(M, kPiece));
  embed_pieces_kernel<<<nb, std::min(C, 256), 0, st>>>(keys, dh, M, C, piece);
  COUNT_LAUNCH(1);
  embed_runs_kernel<<<nb, std::min(C, 256), 0, st>>>(keys, piece, M, C, dwte);
  COUNT_LAUNCH(1);
  embed_wpe_kernel<<<int(cdiv64(int64_t(T) * C, kThreads)), kThreads, 0, st>>>(dh, B, T, C, dwpe,
                                                                               wpe_accumulate);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Launch shape of a staged LayerNorm kernel: S stages of `stage` bytes per
// warp, a grid of as many blocks as fit on the device at once (at most one
// per kLnWarps rows and kLnMaxBlocks).
struct LnLaunch {
  int S = 0, grid = 0;
  size_t smem = 0;
};
template <typename K>
int ln_launch_shape(K kernel, int64_t M, uint32_t stage, size_t budget, LnLaunch& L) {
  L.S = int(std::min<size_t>(4, std::max<size_t>(2, budget / (size_t(kLnWarps) * stage))));
  L.smem = ln_bar_bytes(L.S) + size_t(kLnWarps) * L.S * stage;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L.smem)) !=
      cudaSuccess) {
    cudaGetLastError();
    gpt2_internal::set_error("layernorm: shared-memory size not accepted");
    return GPT2_ERR_CUDA;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kLnWarps * 32, L.smem) !=
          cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  L.grid = int(std::min<int64_t>({cdiv64(M, kLnWarps),
                                  int64_t(per_sm) * gpt2_internal::sm_count(),
                                  int64_t(kLnMaxBlocks)}));
  return GPT2_OK;
}

template <typename OutT>
int launch_layernorm_fwd(const float* x, const float* g, const float* b, OutT* y, float* mean,
                         float* rstd, int64_t M, int C, float eps, cudaStream_t st) {
  if (C > kLnMaxPerLane * 32) {
    gpt2_internal::set_error("layernorm: C above 1024");
    return GPT2_ERR_ARG;
  }
  if (M <= 0) return GPT2_OK;
  // the staged kernels move whole rows by bulk copies and float4 accesses
  const bool aligned = al16(x) && al16(g) && al16(b) && al16(y);
  switch (aligned ? C : -1) {
#define LNF(NV)                                                                              \
  case NV * 128: {                                                                         \
    auto k = layernorm_fwd_staged_kernel<NV, OutT>;                                         \
    LnLaunch L;                                                                            \
    const int rc = ln_launch_shape(k, M, NV * 128 * 4, 96 * 1024, L);                      \
    if (rc) return rc;                                                                     \
    k<<<L.grid, kLnWarps * 32, L.smem, st>>>(x, g, b, y, mean, rstd, M, eps, L.S,           \
                                            device_error_word());                          \
    break;                                                                                 \
  }
    LNF(1) LNF(2) LNF(3) LNF(4) LNF(5) LNF(6) LNF(7) LNF(8)
#undef LNF
    default:
      layernorm_fwd_kernel<OutT><<<int(cdiv64(M, 8)), 256, 0, st>>>(x, g, b, y, mean, rstd, M, C,
                                                                    eps);
  }
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
template int launch_layernorm_fwd<float>(const float*, const float*, const float*, float*, float*,
                                         float*, int64_t, int, float, cudaStream_t);
template int launch_layernorm_fwd<bf16>(const float*, const float*, const float*, bf16*, float*,
                                        float*, int64_t, int, float, cudaStream_t);

size_t layernorm_bwd_workspace(int64_t M, int C) {
  // staged kernel: one [dgamma | dbeta | column sums of dx] row per block;
  // generic kernel (also taken by unaligned views): [dgamma | dbeta] per 64
  // rows, then the column-sum partials
  const int64_t staged = (C % 128 == 0 && C <= 1024)
                             ? std::min<int64_t>(cdiv64(M, kLnWarps), kLnMaxBlocks) * 3 * C
                             : 0;
  const int64_t generic = cdiv64(M, kLnRowsPerBlock) * 2 * C;
  return std::max({size_t(staged) * sizeof(float), size_t(generic) * sizeof(float),
                   colsum_workspace(M, C)});
}

template <typename DyT, typename CopyT>
int launch_layernorm_bwd(const DyT* dy, const float* x, const float* mean, const float* rstd,
                         const float* g, int64_t M, int C, float* dx, CopyT* dx_copy, float* dg,
                         float* db, float* dsum, int accumulate, float* ws, cudaStream_t st,
                         std::vector<RowSum>* defer) {
  if (C > kLnMaxPerLane * 32) {
    gpt2_internal::set_error("layernorm: C above 1024");
    return GPT2_ERR_ARG;
  }
  if (C % 128 == 0 && C <= 1024 && al16(dy) && al16(x) && al16(g) && al16(dx) &&
      al16(dx_copy) && al16(ws)) {
    int nb = 0;  // blocks, one partial row of ws each
    if (M > 0) {
      switch (C / 128) {
#define LNB(NV)                                                                              \
  case NV: {                                                                               \
    auto k = layernorm_bwd_staged_kernel<NV, DyT, CopyT>;                                  \
    LnLaunch L;                                                                            \
    const int rc =                                                                         \
        ln_launch_shape(k, M, NV * 128 * (8 + uint32_t(sizeof(DyT))), 200 * 1024, L);      \
    if (rc) return rc;                                                                     \
    k<<<L.grid, kLnWarps * 32, L.smem, st>>>(dy, x, mean, rstd, g, M, dx, dx_copy, ws,      \
                                            dsum != nullptr, L.S, device_error_word());    \
    nb = L.grid;                                                                           \
    break;                                                                                 \
  }
        LNB(1) LNB(2) LNB(3) LNB(4) LNB(5) LNB(6) LNB(7) LNB(8)
#undef LNB
      }
      COUNT_LAUNCH(1);
    }
    const int n = (dsum ? 3 : 2) * C;
    if (defer) {
      defer->push_back(RowSum{ws, dg, db, dsum, nb, n, C, accumulate});
    } else {
      reduce_rows_kernel<<<cdiv(n, 32), 256, 0, st>>>(ws, nb, n, dg, db, C, accumulate, dsum);
      COUNT_LAUNCH(1);
    }
  } else {
    const int nb = int(cdiv64(M, kLnRowsPerBlock));
    if (nb > 0) {
      layernorm_bwd_kernel<DyT, CopyT><<<nb, 256, 0, st>>>(dy, x, mean, rstd, g, M, C, dx,
                                                           dx_copy, ws);
      COUNT_LAUNCH(1);
    }
    // ws rows hold [dgamma | dbeta]; both halves are reduced in one pass
    reduce_ln_partials_kernel<<<cdiv(2 * C, 256), 256, 0, st>>>(ws, nb, C, dg, db, accumulate);
    COUNT_LAUNCH(1);
    if (dsum && M == 0) {  // no rows: the column sums are zero
      reduce_partials_kernel<<<cdiv(C, 256), 256, 0, st>>>(ws, 0, C, dsum, accumulate);
      COUNT_LAUNCH(1);
    } else if (dsum) {  // column sums of the updated dx (same stream: ws is free again)
      const int rc = launch_colsum<float>(dx, M, C, dsum, accumulate, ws, st);
      if (rc) return rc;
    }
  }
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
template int launch_layernorm_bwd<float, float>(const float*, const float*, const float*,
                                                const float*, const float*, int64_t, int, float*,
                                                float*, float*, float*, float*, int, float*,
                                                cudaStream_t, std::vector<RowSum>*);
template int launch_layernorm_bwd<bf16, bf16>(const bf16*, const float*, const float*, const float*,
                                              const float*, int64_t, int, float*, bf16*, float*,
                                              float*, float*, int, float*, cudaStream_t,
                                              std::vector<RowSum>*);
template int launch_layernorm_bwd<float, bf16>(const float*, const float*, const float*,
                                               const float*, const float*, int64_t, int, float*,
                                               bf16*, float*, float*, float*, int, float*, cudaStream_t,
                                               std::vector<RowSum>*);

// Column sums over a slab of kColRows rows, 16 bytes per lane and row: a block
// of 32 lanes x 8 row slices covers 32*VEC columns; lanes of a warp read one
// contiguous 32*16-byte row segment; the 8 slices are combined in shared
// memory in a fixed order.  Requires N % VEC == 0 and 16-byte aligned rows.
template <typename InT>
__global__ void __launch_bounds__(256) colsum_vec_kernel(const InT* __restrict__ in, int64_t M,
                                                         int N, float* __restrict__ ws) {
  constexpr int VEC = 16 / int(sizeof(InT));
  __shared__ float sh[8][32 * VEC];
  const int lane = threadIdx.x & 31, ry = threadIdx.x >> 5;
  const int n0 = (blockIdx.x * 32 + lane) * VEC;
  const int64_t r0 = int64_t(blockIdx.y) * kColRows;
  const int64_t r1 = min64(M, r0 + kColRows);
  float acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
  if (n0 < N) {
#pragma unroll 4
    for (int64_t r = r0 + ry; r < r1; r += 8) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(in + r * N + n0));
      if constexpr (VEC == 8) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(h2[q]);
          acc[2 * q] += f.x;
          acc[2 * q + 1] += f.y;
        }
      } else {
        acc[0] += __uint_as_float(u.x);
        acc[1] += __uint_as_float(u.y);
        acc[2] += __uint_as_float(u.z);
        acc[3] += __uint_as_float(u.w);
      }
    }
  }
#pragma unroll
  for (int v = 0; v < VEC; ++v) sh[ry][lane * VEC + v] = acc[v];
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * VEC; c += 256) {
    const int n = blockIdx.x * 32 * VEC + c;
    if (n >= N) continue;
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += sh[k][c];
    ws[int64_t(blockIdx.y) * N + n] = t;
  }
}

size_t colsum_workspace(int64_t M, int N) { return size_t(cdiv64(M, kColRows)) * N * sizeof(float); }

template <typename InT>
int launch_colsum(const InT* in, int64_t M, int N, float* out, int accumulate, float* ws,
                  cudaStream_t st, std::vector<RowSum>* defer) {
  const int parts = int(cdiv64(M, kColRows));
  constexpr int VEC = 16 / int(sizeof(InT));
  if (N % VEC == 0 && (reinterpret_cast<uintptr_t>(in) & 15) == 0) {
    dim3 grid(cdiv(N, 32 * VEC), parts);
    colsum_vec_kernel<InT><<<grid, 256, 0, st>>>(in, M, N, ws);
    COUNT_LAUNCH(1);
    if (defer) {
      defer->push_back(RowSum{ws, out, nullptr, nullptr, parts, N, N, accumulate});
    } else {
      reduce_rows_kernel<<<cdiv(N, 32), 256, 0, st>>>(ws, parts, N, out, nullptr, N, accumulate);
      COUNT_LAUNCH(1);
    }
  } else {
    dim3 grid(cdiv(N, kThreads), parts);
    colsum_partial_kernel<InT><<<grid, kThreads, 0, st>>>(in, M, N, ws);
    COUNT_LAUNCH(1);
    reduce_partials_kernel<<<cdiv(N, kThreads), kThreads, 0, st>>>(ws, parts, N, out, accumulate);
    COUNT_LAUNCH(1);
  }
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
template int launch_colsum<float>(const float*, int64_t, int, float*, int, float*, cudaStream_t,
                                  std::vector<RowSum>*);
template int launch_colsum<bf16>(const bf16*, int64_t, int, float*, int, float*, cudaStream_t,
                                 std::vector<RowSum>*);

int launch_row_sums(const RowSum* sums, int count, cudaStream_t st) {
  for (int i0 = 0; i0 < count; i0 += kRowSumMax) {
    const int k = std::min(kRowSumMax, count - i0);
    RowSumBatch b{};
    int max_n = 0;
    for (int i = 0; i < k; ++i) {
      b.s[i] = sums[i0 + i];
      max_n = std::max(max_n, b.s[i].n);
    }
    if (max_n <= 0) continue;
    reduce_rows_batch_kernel<<<dim3(cdiv(max_n, 32), k), 256, 0, st>>>(b);
    COUNT_LAUNCH(1);
    GPT2_LAUNCH_CHECK();
  }
  return GPT2_OK;
}

size_t gradnorm_workspace() { return kNormBlocks * sizeof(double); }

int launch_gradnorm(const float* g, int64_t n, double* ws, float* norm, cudaStream_t st) {
  sumsq_kernel<<<kNormBlocks, kThreads, 0, st>>>(g, n, ws);
  COUNT_LAUNCH(1);
  norm_finalize_kernel<<<1, 1024, 0, st>>>(ws, norm);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_clip_adamw(float* p, const float* g, float* m, float* v, bf16* pb, int64_t n,
                      int64_t n_decay, const float* norm, DevStatus* status, float lr,
                      const float* lr_dev, float b1, float b2, float eps, float wd, float max_norm,
                      cudaStream_t st) {
  if ((n & 3) || (n_decay & 3)) {
    gpt2_internal::set_error("clip_adamw: arena sizes must be multiples of 4");
    return GPT2_ERR_ARG;
  }
  clip_adamw_kernel<<<grid_for(n / 4, kThreads), kThreads, 0, st>>>(
      p, g, m, v, pb, n, n_decay, norm, status, lr, lr_dev, b1, b2, eps, wd, max_norm);
  COUNT_LAUNCH(1);
  step_advance_kernel<<<1, 1, 0, st>>>(norm, status);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_ce_rows_fwd(const float* z, const int32_t* y, int rows, int Vp, float* lse,
                       float* row_loss, cudaStream_t st) {
  if (rows <= 0) return GPT2_OK;
  ce_rows_fwd_kernel<<<rows, 512, 0, st>>>(z, y, Vp, lse, row_loss);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template <typename OutT>
int launch_ce_rows_bwd(const float* z, const float* lse, const int32_t* y, int rows, int Vp,
                       float scale, OutT* dz, cudaStream_t st) {
  if (rows <= 0) return GPT2_OK;
  ce_rows_bwd_kernel<OutT><<<rows, 512, 0, st>>>(z, lse, y, Vp, scale, dz);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
template int launch_ce_rows_bwd<float>(const float*, const float*, const int32_t*, int, int, float,
                                       float*, cudaStream_t);
template int launch_ce_rows_bwd<bf16>(const float*, const float*, const int32_t*, int, int, float,
                                      bf16*, cudaStream_t);

int launch_mean(const float* v, int64_t n, float* out, cudaStream_t st) {
  mean_kernel<<<1, kThreads, 0, st>>>(v, n, out);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_to_bf16(const float* src, bf16* dst, int64_t n, cudaStream_t st) {
  if (n <= 0) return GPT2_OK;
  to_bf16_kernel<<<grid_for(n, kThreads), kThreads, 0, st>>>(src, dst, n);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_fill(float* p, float v, int64_t n, cudaStream_t st) {
  if (n <= 0) return GPT2_OK;
  fill_kernel<<<grid_for(n, kThreads), kThreads, 0, st>>>(p, v, n);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
