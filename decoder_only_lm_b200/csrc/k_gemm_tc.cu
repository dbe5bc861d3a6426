// Tensor-core GEMM for sm_100a: tcgen05.mma (kind::f16, bf16 operands, fp32
// accumulation in TMEM) fed by TMA, with the linear-layer epilogues fused.
//
//   D[m,n] = epilogue( sum_k A(m,k) B(n,k) )
//
// Design
//   - persistent CTAs (one per SM), static round-robin over output tiles of
//     128 x BN (BN = 256 or 128), m fastest so co-resident CTAs share B tiles;
//   - warp-specialised: warp 0 issues TMA loads (one elected lane), warp 1
//     issues tcgen05.mma (one elected lane), warp 2 owns the TMEM allocation,
//     warps 4-7 and 8-11 (two warpgroups, one per accumulator) drain the
//     accumulator with tcgen05.ld and run the epilogue; for epilogues with an
//     input (residual, GELU input) lane 0 of warp 2 / 3 issues the TMA copies
//     of warpgroup 0 / 1;
//   - STAGES-deep shared-memory ring of (A, B) k-blocks of 64 elements with
//     128-byte swizzle, full/empty mbarriers; two TMEM accumulators so the
//     epilogue of tile i overlaps the MMAs of tile i+1;
//   - operands may be K-major (rows of K contiguous) or MN-major (rows of M or
//     N contiguous: the weight-gradient and transposed-weight contractions of
//     the backward pass), described to the MMA by the smem descriptors;
//   - split-K for weight gradients with few output tiles: split s writes its
//     partial tile to a workspace, a reduction adds the splits in order;
//   - every mbarrier wait is bounded by a global-timer budget: on expiry the
//     kernel records a timeout in the error word, every role leaves its loop,
//     in-flight copies and MMAs are waited for (again bounded) and TMEM is
//     freed before the CTA exits.  No trap, no unbounded spin.
//
// No TMA multicast is used anywhere (each CTA loads its own tiles).

#include <cuda.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "epilogue.cuh"
#include "tc_common.cuh"

using namespace tc;

namespace {

// A tile of the output is 256 x BN, computed by a pair of CTAs (a cluster of
// two): CTA r of the pair owns rows 128 r .. 128 r + 127 of the tile, holds
// those rows of A and columns BN/2 r .. BN/2 r + BN/2 - 1 of B in its shared
// memory, and receives its 128 accumulator rows in its own TMEM.
constexpr int BM = 128;         // rows per CTA
constexpr int BM2 = 2 * BM;     // rows per tile (CTA pair)
constexpr int UMMA_K = 16;
constexpr int kThreads = 384;  // warps 0-3: TMA, MMA, TMEM, idle; 4-7 and 8-11: epilogue

constexpr int kSmemLimit = 232448;  // opt-in dynamic shared memory per block

template <int EPI>
__host__ __device__ constexpr bool epi_has_input() {
  return EPI == EPI_RESID || EPI == EPI_GELU_BWD;
}
// k-block stages of the operand pipeline: epilogues with an input stream
// keep more shared memory for their chunk buffers
template <int EPI>
__host__ __device__ constexpr int tc_stages(bool te) {
  return !te ? 5 : epi_has_input<EPI>() ? 4 : 5;
}
// Shared memory: [STAGES x (A, B) k-block ring | epilogue area | barriers].
// With the TMA epilogue (TE) the area is a set of 8 KB chunk buffers; GEMMs
// whose epilogue reads an input (residual, GELU input) give up one k-block
// stage for more buffers so that more input bytes are in flight.
template <int BN, bool TE, int EPI>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;        // this CTA's 128 rows of A
  static constexpr int B_BYTES = (BN / 2) * BK * 2;  // this CTA's BN/2 rows of B
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = tc_stages<EPI>(TE);
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 512;
  static constexpr int STAGE_ROW = 36;  // fp32 per staged accumulator row (32 + 4 pad)
  // chunk buffers per epilogue warpgroup (two warpgroups, at most 8 each)
  static constexpr int NBUF_WG =
      TE ? ((kSmemLimit - 1024 - BAR_BYTES - STAGES * STAGE) / 16384 > 8
                ? 8
                : (kSmemLimit - 1024 - BAR_BYTES - STAGES * STAGE) / 16384)
         : 0;
  static constexpr int WG_BYTES = TE ? NBUF_WG * 8192 : BM * STAGE_ROW * 4;
  static constexpr int EPI_BYTES = 2 * WG_BYTES;
  static constexpr int SMEM = STAGES * STAGE + EPI_BYTES + BAR_BYTES + 1024;
  static_assert(SMEM <= kSmemLimit, "shared memory");
  static_assert(!TE || NBUF_WG >= 4, "epilogue buffers");
};

struct TcParams {
  int M, N, K;
  int a_mn, b_mn;
  int tiles_m, tiles_n, splits, kb_per_split, num_kb, total_tiles;  // tiles of BM2 x BN
  int n_fast;  // tile order: 1 = column tiles vary fastest (A panels read once)
  EpiParams ep;
  float* ws;
  int* err;
};

// Output tile, column tile and K split of linear tile index t.  Consecutive
// tiles (processed at the same time by neighbouring CTA pairs) share the
// panel of the larger operand, which is then read from memory once: rows of
// A when n_fast, columns of B otherwise.
__device__ __forceinline__ void tile_coords(const TcParams& p, int t, int& tm, int& tn, int& sp) {
  const int mn = p.tiles_m * p.tiles_n;
  sp = t / mn;
  const int r = t - sp * mn;
  if (p.n_fast) {
    tn = r % p.tiles_n;
    tm = r / p.tiles_n;
  } else {
    tm = r % p.tiles_m;
    tn = r / p.tiles_m;
  }
}

// Instruction descriptor: kind::f16, bf16 A and B, fp32 D, M = 256 (pair), N = BN.
template <int BN>
__device__ __forceinline__ uint32_t gemm_idesc(int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(BN >> 3) << 17) | (uint32_t(BM2 >> 4) << 24);
}

// ------------------------------------------------------------ vector helpers
template <typename T, int W>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[W]);
template <typename T, int W>
__device__ __forceinline__ void store_vec(T* p, const float (&v)[W]);
template <>
__device__ __forceinline__ void load_vec<float, 4>(const float* p, float (&v)[4]) {
  const float4 f = *reinterpret_cast<const float4*>(p);
  v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
template <>
__device__ __forceinline__ void store_vec<float, 4>(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void load_vec<bf16, 8>(const bf16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(h[q]);
    v[2 * q] = f.x;
    v[2 * q + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void store_vec<bf16, 8>(bf16* p, const float (&v)[8]) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
    w[q] = *reinterpret_cast<uint32_t*>(&t);
  }
  *reinterpret_cast<uint4*>(p) = u;
}
template <>
__device__ __forceinline__ void load_vec<float, 8>(const float* p, float (&v)[8]) {
#pragma unroll
  for (int j = 0; j < 8; j += 4) {
    const float4 f = *reinterpret_cast<const float4*>(p + j);
    v[j] = f.x; v[j + 1] = f.y; v[j + 2] = f.z; v[j + 3] = f.w;
  }
}
template <>
__device__ __forceinline__ void store_vec<float, 8>(float* p, const float (&v)[8]) {
#pragma unroll
  for (int j = 0; j < 8; j += 4)
    *reinterpret_cast<float4*>(p + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
}
template <>
__device__ __forceinline__ void load_vec<bf16, 4>(const bf16* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
template <>
__device__ __forceinline__ void store_vec<bf16, 4>(bf16* p, const float (&v)[4]) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
  __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
template <int W>
__device__ __forceinline__ void load_bias(const float* b, int n, float (&v)[W]) {
#pragma unroll
  for (int j = 0; j < W; j += 4) {
    const float4 f = *reinterpret_cast<const float4*>(b + n + j);
    v[j] = f.x; v[j + 1] = f.y; v[j + 2] = f.z; v[j + 3] = f.w;
  }
}

// The epilogue op on W consecutive columns n .. n+W-1 of row m, s = the
// accumulators (all W columns in range, 16-byte aligned addresses).
template <int EPI, typename OutT, int W>
__device__ __forceinline__ void epi_vec(const EpiParams& e, int m, int n, float (&s)[W]) {
  const int64_t i = int64_t(m) * e.ldo + n;
  if (EPI == EPI_STORE) {
    if (e.bias) {
      float b[W];
      load_bias<W>(e.bias, n, b);
#pragma unroll
      for (int j = 0; j < W; ++j) s[j] = s[j] * e.alpha + b[j];
    } else {
#pragma unroll
      for (int j = 0; j < W; ++j) s[j] *= e.alpha;
    }
    store_vec<OutT, W>(reinterpret_cast<OutT*>(e.out) + i, s);
  } else if (EPI == EPI_GELU) {
    float b[W];
    load_bias<W>(e.bias, n, b);
#pragma unroll
    for (int j = 0; j < W; ++j) s[j] = round_through<OutT>(s[j] + b[j]);
    store_vec<OutT, W>(reinterpret_cast<OutT*>(e.out) + i, s);
#pragma unroll
    for (int j = 0; j < W; ++j) s[j] = gelu_tanh(s[j]);
    store_vec<OutT, W>(reinterpret_cast<OutT*>(e.out2) + i, s);
  } else if (EPI == EPI_RESID) {
    float r[W];
    load_vec<float, W>(e.rin + i, r);
    if (e.bias) {
      float b[W];
      load_bias<W>(e.bias, n, b);
#pragma unroll
      for (int j = 0; j < W; ++j) r[j] += b[j];
    }
#pragma unroll
    for (int j = 0; j < W; ++j) s[j] += r[j];
    store_vec<float, W>(e.rout + i, s);
  } else if (EPI == EPI_ACC) {
    float* o = reinterpret_cast<float*>(e.out) + i;
    if (e.accumulate) {
      float r[W];
      load_vec<float, W>(o, r);
#pragma unroll
      for (int j = 0; j < W; ++j) s[j] = r[j] + e.alpha * s[j];
    } else {
#pragma unroll
      for (int j = 0; j < W; ++j) s[j] *= e.alpha;
    }
    store_vec<float, W>(o, s);
  } else if (EPI == EPI_GELU_BWD) {
    float u[W];
    load_vec<OutT, W>(reinterpret_cast<const OutT*>(e.aux) + i, u);
#pragma unroll
    for (int j = 0; j < W; ++j) s[j] *= gelu_tanh_grad(u[j]);
    store_vec<OutT, W>(reinterpret_cast<OutT*>(e.out) + i, s);
  } else if (EPI == EPI_CE_GRAD) {
    const float l = e.lse[m];
    const int t = e.tgt[m];
#pragma unroll
    for (int j = 0; j < W; ++j) s[j] = e.ce_scale * (__expf(s[j] - l) - (n + j == t ? 1.f : 0.f));
    store_vec<OutT, W>(reinterpret_cast<OutT*>(e.out) + i, s);
  }
}

// named barrier of one epilogue warpgroup (ids 1 and 2)
__device__ __forceinline__ void epi_bar(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

// Store phase of one staged 128 x 32 chunk: W consecutive columns per item,
// items spread so that a warp covers whole row segments (coalesced).  All of
// a thread's global loads (residual, accumulator, GELU input) are issued
// before any of its stores, so their latencies overlap.
template <int EPI, typename OutT, int W>
__device__ __forceinline__ void epi_store_chunk(const TcParams& p, const float* S, int stage_row,
                                                int e, int m0, int n0, int sp) {
  constexpr int SEGS = 32 / W;  // segments per row; 128 rows x SEGS items, SEGS per thread
  constexpr bool kLoadF32 = (EPI == EPI_RESID || EPI == EPI_ACC);
  constexpr bool kLoadAux = (EPI == EPI_GELU_BWD);
  const EpiParams& ep = p.ep;
  float s[SEGS][W], r[SEGS][W];
  bool full[SEGS], live[SEGS];
#pragma unroll
  for (int k = 0; k < SEGS; ++k) {
    const int item = e + 128 * k;
    const int row = item / SEGS, seg = item % SEGS;
    const int m = m0 + row, n = n0 + seg * W;
    live[k] = m < p.M && n < p.N;
    full[k] = live[k] && n + W <= p.N;
#pragma unroll
    for (int j = 0; j < W; j += 4) {
      const float4 f = *reinterpret_cast<const float4*>(S + row * stage_row + seg * W + j);
      s[k][j] = f.x; s[k][j + 1] = f.y; s[k][j + 2] = f.z; s[k][j + 3] = f.w;
    }
    if (!p.ws && full[k]) {
      const int64_t i = int64_t(m) * ep.ldo + n;
      if (kLoadF32 && (EPI == EPI_RESID || ep.accumulate))
        load_vec<float, W>((EPI == EPI_RESID ? ep.rin : reinterpret_cast<const float*>(ep.out)) + i,
                           r[k]);
      if (kLoadAux) load_vec<OutT, W>(reinterpret_cast<const OutT*>(ep.aux) + i, r[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < SEGS; ++k) {
    if (!live[k]) continue;
    const int item = e + 128 * k;
    const int row = item / SEGS, seg = item % SEGS;
    const int m = m0 + row, n = n0 + seg * W;
    if (p.ws) {
      float* w = p.ws + (int64_t(sp) * p.M + m) * p.N + n;
      if (full[k] && W == 4 && (p.N & 3) == 0) {
        *reinterpret_cast<float4*>(w) = make_float4(s[k][0], s[k][1], s[k][2], s[k][3]);
      } else {
        for (int j = 0; j < W; ++j)
          if (n + j < p.N) w[j] = s[k][j];
      }
      continue;
    }
    if (!full[k]) {
      for (int j = 0; j < W; ++j)
        if (n + j < p.N) epi_apply<OutT>(ep, EPI, m, n + j, s[k][j]);
      continue;
    }
    const int64_t i = int64_t(m) * ep.ldo + n;
    if (EPI == EPI_RESID) {
      if (ep.bias) {
        float b[W];
        load_bias<W>(ep.bias, n, b);
#pragma unroll
        for (int j = 0; j < W; ++j) r[k][j] += b[j];
      }
#pragma unroll
      for (int j = 0; j < W; ++j) s[k][j] += r[k][j];
      store_vec<float, W>(ep.rout + i, s[k]);
    } else if (EPI == EPI_ACC) {
#pragma unroll
      for (int j = 0; j < W; ++j) s[k][j] = (ep.accumulate ? r[k][j] : 0.f) + ep.alpha * s[k][j];
      store_vec<float, W>(reinterpret_cast<float*>(ep.out) + i, s[k]);
    } else if (EPI == EPI_GELU_BWD) {
#pragma unroll
      for (int j = 0; j < W; ++j) s[k][j] *= gelu_tanh_grad(r[k][j]);
      store_vec<OutT, W>(reinterpret_cast<OutT*>(ep.out) + i, s[k]);
    } else {
      epi_vec<EPI, OutT, W>(ep, m, n, s[k]);
    }
  }
}

// ------------------------------------------------------------ TMA epilogue
// GELU of the bf16 tensor-core path with tanh from the hardware tanh.approx
// instruction (relative error about 2^-11, below the bf16 rounding of the
// stored activation) [ZERO: OpFFN; the tanh form of GELU].
__device__ __forceinline__ float tanh_hw(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x from the hardware ex2.approx instruction (exp(x) = 2^(x log2 e)).
__device__ __forceinline__ float ex2_hw(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;
// The GELU epilogues two columns per packed instruction (fma/mul/add.f32x2).
// With z = k (u + a u^3) and t = tanh z:  GELU(u) = u/2 (1 + t),
// GELU'(u) = (1 + t)/2 + u/2 (1 - t^2) k (1 + 3 a u^2).
constexpr float kGeluK = 0.7978845608028654f;  // sqrt(2 / pi)
constexpr float kGeluKA = kGeluK * 0.044715f;
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// pre = bf16(v + b) (the stored pre-activation), act = bf16(GELU(pre)): the
// activation is taken of the rounded value, the one the backward reads.
__device__ __forceinline__ void gelu_chunk32(const float (&v)[32], const float (&b)[32],
                                             uint32_t (&pre)[16], uint32_t (&act)[16]) {
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    float x0 = v[j], x1 = v[j + 1];
    add2(x0, x1, b[j], b[j + 1]);
    const uint32_t pk = bf16x2_bits(x0, x1);
    pre[j >> 1] = pk;
    const float u0 = __uint_as_float(pk << 16), u1 = __uint_as_float(pk & 0xffff0000u);
    float s0 = u0, s1 = u1, z0, z1;
    mul2(s0, s1, u0, u1);
    fma2(z0, z1, s0, s1, kGeluKA, kGeluKA, kGeluK, kGeluK);
    mul2(z0, z1, u0, u1);
    const float t0 = tanh_hw(z0), t1 = tanh_hw(z1);
    float h0 = u0, h1 = u1, g0, g1;
    mul2(h0, h1, 0.5f, 0.5f);
    fma2(g0, g1, h0, h1, t0, t1, h0, h1);
    act[j >> 1] = bf16x2_bits(g0, g1);
  }
}
// (d0, d1) *= GELU'(u0, u1)
__device__ __forceinline__ void gelu_bwd_pair(float& d0, float& d1, float u0, float u1) {
  float s0 = u0, s1 = u1, z0, z1, q0, q1, m0, m1, g0, g1;
  mul2(s0, s1, u0, u1);
  fma2(z0, z1, s0, s1, kGeluKA, kGeluKA, kGeluK, kGeluK);
  mul2(z0, z1, u0, u1);
  const float t0 = tanh_hw(z0), t1 = tanh_hw(z1);
  fma2(q0, q1, s0, s1, 3.f * kGeluKA, 3.f * kGeluKA, kGeluK, kGeluK);  // k (1 + 3 a u^2)
  fma2(m0, m1, t0, t1, t0, t1, -1.f, -1.f);                            // t^2 - 1
  float r0 = u0, r1 = u1;
  mul2(r0, r1, -0.5f, -0.5f);
  mul2(r0, r1, m0, m1);  // u/2 (1 - t^2)
  mul2(r0, r1, q0, q1);
  add2(r0, r1, 0.5f, 0.5f);
  fma2(g0, g1, t0, t1, 0.5f, 0.5f, r0, r1);
  mul2(d0, d1, g0, g1);
}

// Chunks of the TMA epilogue: 128 rows x 64 bytes (32 bf16 or 16 fp32
// columns) per 8 KB buffer in the 64-byte swizzle of the tensor map: the
// 16-byte unit u of row r sits at r*64 + 16*(u ^ ((r >> 1) & 3)), so the
// row-per-thread accesses of a warp are free of bank conflicts.
template <int EPI, typename OutT, int NBUF>
struct TeCfg {
  static constexpr int CW = 64 / int(sizeof(OutT));
  static constexpr int ARR = EPI == EPI_GELU ? 2 : 1;  // buffers per chunk
  static constexpr int SLOTS = NBUF / ARR;
  static constexpr bool HAS_IN = epi_has_input<EPI>();
  // bulk groups that may still be reading their buffers when a chunk is
  // done (with an input: when the issuer takes the next chunk)
  static constexpr int WAITN = HAS_IN ? 1 : (SLOTS - 2 < 6 ? SLOTS - 2 : 6);
  static_assert(SLOTS >= 2 && SLOTS <= 8 && WAITN >= 0, "epilogue slots");
};
// tcgen05.ld of CW (32 or 16) accumulator columns without waiting; the
// registers are valid after tmem_wait_cols(r), which names them so that no
// use is scheduled before the wait.
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld32_async(taddr, r);
}
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_cols(uint32_t (&r)[32]) { tmem_wait_ld(r); }
__device__ __forceinline__ void tmem_wait_cols(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
}
__device__ __forceinline__ int swz64(int row, int u) {
  return row * 64 + ((u ^ ((row >> 1) & 3)) << 4);
}
template <typename T>
__device__ __forceinline__ void row_put(uint8_t* buf, int r, const float (&v)[64 / sizeof(T)]);
template <>
__device__ __forceinline__ void row_put<bf16>(uint8_t* buf, int r, const float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint4 w;
    uint32_t* x = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 t = __floats2bfloat162_rn(v[8 * u + 2 * q], v[8 * u + 2 * q + 1]);
      x[q] = *reinterpret_cast<uint32_t*>(&t);
    }
    *reinterpret_cast<uint4*>(buf + swz64(r, u)) = w;
  }
}
template <>
__device__ __forceinline__ void row_put<float>(uint8_t* buf, int r, const float (&v)[16]) {
#pragma unroll
  for (int u = 0; u < 4; ++u)
    *reinterpret_cast<float4*>(buf + swz64(r, u)) =
        make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
}
// a row of 32 bf16 already packed in pairs
__device__ __forceinline__ void row_put_bits(uint8_t* buf, int r, const uint32_t (&x)[16]) {
#pragma unroll
  for (int u = 0; u < 4; ++u)
    *reinterpret_cast<uint4*>(buf + swz64(r, u)) =
        make_uint4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
}
template <typename T>
__device__ __forceinline__ void row_get(const uint8_t* buf, int r, float (&v)[64 / sizeof(T)]);
template <>
__device__ __forceinline__ void row_get<bf16>(const uint8_t* buf, int r, float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint4 w = *reinterpret_cast<const uint4*>(buf + swz64(r, u));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(h[q]);
      v[8 * u + 2 * q] = f.x;
      v[8 * u + 2 * q + 1] = f.y;
    }
  }
}
template <>
__device__ __forceinline__ void row_get<float>(const uint8_t* buf, int r, float (&v)[16]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float4 f = *reinterpret_cast<const float4*>(buf + swz64(r, u));
    v[4 * u] = f.x; v[4 * u + 1] = f.y; v[4 * u + 2] = f.z; v[4 * u + 3] = f.w;
  }
}
// bias[n0 .. n0+CW-1], zero past column N
template <int CW>
__device__ __forceinline__ void bias_chunk(const float* bias, int n0, int N, float (&b)[CW]) {
  if (n0 + CW <= N) {
#pragma unroll
    for (int j = 0; j < CW; j += 4) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(bias + n0 + j));
      b[j] = f.x; b[j + 1] = f.y; b[j + 2] = f.z; b[j + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < CW; ++j) b[j] = n0 + j < N ? bias[n0 + j] : 0.f;
  }
}

// The epilogue op on one chunk of a row: v holds CW accumulator columns of
// row e of this CTA's half-tile (first column n0); inputs (residual, GELU
// input) are read from, and the results written to, the chunk's swizzled
// buffer(s) at b0.
template <int EPI, typename OutT, int CW>
__device__ __forceinline__ void chunk_apply(const TcParams& p, uint8_t* b0, int e, int n0,
                                            float (&v)[CW], float row_l, int row_t) {
  const EpiParams& ep = p.ep;
  if constexpr (EPI == EPI_RESID || EPI == EPI_GELU_BWD) {
    float r[CW];
    row_get<OutT>(b0, e, r);
    if constexpr (EPI == EPI_RESID) {
      if (ep.bias) {
        float bb[CW];
        bias_chunk<CW>(ep.bias, n0, p.N, bb);
#pragma unroll
        for (int j = 0; j < CW; ++j) r[j] += bb[j];
      }
#pragma unroll
      for (int j = 0; j < CW; ++j) v[j] += r[j];
    } else {
#pragma unroll
      for (int j = 0; j < CW; j += 2) gelu_bwd_pair(v[j], v[j + 1], r[j], r[j + 1]);
    }
    row_put<OutT>(b0, e, v);
  } else if constexpr (EPI == EPI_GELU) {
    static_assert(CW == 32, "bf16 GELU chunks");
    float bb[CW];
    bias_chunk<CW>(ep.bias, n0, p.N, bb);
    uint32_t pre[CW / 2], act[CW / 2];
    gelu_chunk32(v, bb, pre, act);
    row_put_bits(b0, e, pre);
    row_put_bits(b0 + 8192, e, act);
  } else if constexpr (EPI == EPI_STORE) {
    if (ep.bias) {
      float bb[CW];
      bias_chunk<CW>(ep.bias, n0, p.N, bb);
#pragma unroll
      for (int j = 0; j < CW; ++j) v[j] = v[j] * ep.alpha + bb[j];
    } else {
#pragma unroll
      for (int j = 0; j < CW; ++j) v[j] *= ep.alpha;
    }
    row_put<OutT>(b0, e, v);
  } else if constexpr (EPI == EPI_ACC) {
    if (!p.ws) {  // split partial sums stay raw (alpha applied by the reduction)
#pragma unroll
      for (int j = 0; j < CW; ++j) v[j] *= ep.alpha;
    }
    row_put<OutT>(b0, e, v);
  } else if constexpr (EPI == EPI_CE_GRAD) {
    const float cs = ep.ce_scale;
    if (cs > 0.f) {  // cs 2^x = 2^(x + log2 cs): one packed fma and one ex2 per element
      const float b = log2f(cs) - row_l * kLog2e;
#pragma unroll
      for (int j = 0; j < CW; j += 2) {
        float a0, a1;
        fma2(a0, a1, v[j], v[j + 1], kLog2e, kLog2e, b, b);
        v[j] = ex2_hw(a0);
        v[j + 1] = ex2_hw(a1);
      }
    } else {
      const float l2 = row_l * kLog2e;
#pragma unroll
      for (int j = 0; j < CW; ++j) v[j] = cs * ex2_hw(fmaf(v[j], kLog2e, -l2));
    }
    if (row_t >= n0 && row_t < n0 + CW) {  // the target column: - scale
#pragma unroll
      for (int j = 0; j < CW; ++j)
        if (n0 + j == row_t) v[j] -= cs;
    }
    row_put<OutT>(b0, e, v);
  }
}

// Barriers of the TMA epilogue (offsets in tb, one per slot and warpgroup):
// in[s] the chunk's input landed (TMA transaction count), rdy[s] the chunk is
// written (4 warp arrivals, epilogues with an input only).
constexpr int kEpiIn = 4, kEpiRdy = 20, kTmemSlot = 36;

// The pair-local tiles of warpgroup wg (wg, wg+2, ...).
struct EpiTiles {
  int pair, npairs, wg, my_tiles;
  __device__ EpiTiles(const TcParams& p, int wg_) : wg(wg_) {
    pair = int(blockIdx.x) >> 1;
    npairs = int(gridDim.x) >> 1;
    const int pair_tiles = pair < p.total_tiles ? (p.total_tiles - 1 - pair) / npairs + 1 : 0;
    my_tiles = pair_tiles > wg ? (pair_tiles - wg + 1) / 2 : 0;
  }
  __device__ int tile(int j) const { return pair + (wg + 2 * j) * npairs; }
};

// Epilogue warpgroup with TMA stores, for the epilogues without an input:
// thread e owns row 128 r + e of the pair's tile (CTA rank r, TMEM lane e).
// Per chunk it loads CW accumulator columns, applies the epilogue op, writes
// the row into the swizzled buffer, and after one named barrier a single
// thread issues the TMA store (for gradient accumulation the TMA reduce-add:
// one fp32 add per element, so the result does not depend on timing).
// Out-of-range rows and columns of edge tiles are clipped by the tensor map.
template <int BN, int EPI, typename OutT, int NBUF>
__device__ __forceinline__ void epilogue_tma(const TcParams& p, const CUtensorMap* mo,
                                             const CUtensorMap* mo2, uint8_t* ebuf, uint64_t* tb,
                                             uint32_t tmem_base, int wg) {
  using T = TeCfg<EPI, OutT, NBUF>;
  static_assert(!T::HAS_IN, "epilogues with an input use epilogue_tma_split");
  constexpr int CW = T::CW, NCH = BN / CW, SL = T::SLOTS;
  const int e = threadIdx.x - 128 - 128 * wg;
  const int bar_id = 1 + wg;
  const int q = e >> 5;  // TMEM lanes 32q .. 32q+31
  const bool leader = e == 0;
  const uint32_t eb = smem_u32(ebuf);
  const int rank = int(cluster_ctarank());
  auto tfull = [&](int a) { return smem_u32(tb + a); };
  // the even CTA's accumulator-empty barrier (its MMA issuer waits on it)
  auto tempty_pair = [&](int a) { return mapa_shared(smem_u32(tb + 2 + a), 0); };
  const EpiTiles et(p, wg);
  // A wait that expires (error word set) poisons the thread: later waits are
  // skipped but every thread still runs the same sequence of named barriers,
  // so no warp is left waiting at one.
  int g = 0;  // chunks done by this warpgroup
  bool ok = true;
  for (int j = 0; j < et.my_tiles; ++j) {
    const int t_local = wg + 2 * j;
    int tm, tn, sp;
    tile_coords(p, et.tile(j), tm, tn, sp);
    const int acc = wg;
    const int m0 = tm * BM2 + rank * BM;  // first row of this CTA's half
    const int m = m0 + e;
    // the row's log-sum-exp and target are fetched while the MMAs still run
    float row_l = 0.f;
    int row_t = -1;
    if (EPI == EPI_CE_GRAD && m < p.M) {
      row_l = p.ep.lse[m];
      row_t = p.ep.tgt[m];
    }
    if (ok) ok = mbar_wait(tfull(acc), (t_local >> 1) & 1, p.err, 4);
    tc_fence_after();
    const uint32_t tbase = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
    // the accumulator columns of chunk c+1 are loaded while chunk c is processed
    uint32_t rn[CW];
    tmem_ld_cols(tbase, rn);
    tmem_wait_cols(rn);
#pragma unroll 1
    for (int c = 0; c < NCH; ++c, ++g) {
      const int slot = g % SL;
      const int n0 = tn * BN + c * CW;
      float v[CW];
#pragma unroll
      for (int jj = 0; jj < CW; ++jj) v[jj] = __uint_as_float(rn[jj]);
      if (c + 1 < NCH) {
        tmem_ld_cols(tbase + uint32_t((c + 1) * CW), rn);
      } else if (leader) {
        // every thread's TMEM loads completed before the previous chunk's
        // barrier: the accumulator is drained, the pair's MMA may reuse it
        mbar_arrive_cluster(tempty_pair(acc));
      }
      chunk_apply<EPI, OutT, CW>(p, ebuf + slot * T::ARR * 8192, e, n0, v, row_l, row_t);
      fence_proxy_async();
      if (c + 1 < NCH) tmem_wait_cols(rn);
      if (c + 2 == NCH) tc_fence_before();  // last TMEM load of the tile waited for
      if (leader) bulk_wait_read<T::WAITN>();
      epi_bar(bar_id);
      if (leader) {
        const uint32_t src = eb + slot * T::ARR * 8192;
        if (EPI == EPI_ACC && p.ws)  // split sp's partial: rows sp * M .. of [splits * M, N]
          tma_store_2d(mo, src, n0, m0 + sp * p.M);
        else if (EPI == EPI_ACC && p.ep.accumulate)
          tma_reduce_add_2d(mo, src, n0, m0);
        else
          tma_store_2d(mo, src, n0, m0);
        if (EPI == EPI_GELU) tma_store_2d(mo2, src + 8192, n0, m0);
        bulk_commit();
      }
    }
  }
  if (leader) bulk_wait_all();
}

// Epilogue with an input (residual add, GELU backward), split in two roles
// per warpgroup wg so that no TMA issue and no named barrier sits on the
// warpgroup's per-chunk path:
//   - the 128 threads of the warpgroup (thread e owns row 128 r + e of the
//     pair's tile) wait for the chunk's input, load CW accumulator columns,
//     apply the op, write the row over the input in the chunk's buffer, and
//     each warp signals "chunk written" (rdy);
//   - one issuer thread (lane 0 of warp 2 + wg, epilogue_issuer) issues the
//     chunk's TMA store and, once that store has read the buffer, fetches
//     the input of a later chunk into it.
template <int BN, int EPI, typename OutT, int NBUF>
__device__ __forceinline__ void epilogue_tma_split(const TcParams& p, uint8_t* ebuf, uint64_t* tb,
                                                   uint32_t tmem_base, int wg) {
  using T = TeCfg<EPI, OutT, NBUF>;
  static_assert(T::HAS_IN && T::ARR == 1, "epilogues with an input");
  constexpr int CW = T::CW, NCH = BN / CW, SL = T::SLOTS;
  const int e = threadIdx.x - 128 - 128 * wg;
  const int lane = e & 31;
  const int q = e >> 5;  // TMEM lanes 32q .. 32q+31
  auto tfull = [&](int a) { return smem_u32(tb + a); };
  auto tempty_pair = [&](int a) { return mapa_shared(smem_u32(tb + 2 + a), 0); };
  auto inb = [&](int s) { return smem_u32(tb + kEpiIn + 8 * wg + s); };
  auto rdy = [&](int s) { return smem_u32(tb + kEpiRdy + 8 * wg + s); };
  const EpiTiles et(p, wg);
  // an expired wait (error word set) skips later waits; every arrival still happens
  int g = 0;
  bool ok = true;
  for (int j = 0; j < et.my_tiles; ++j) {
    const int t_local = wg + 2 * j;
    int tm, tn, sp;
    tile_coords(p, et.tile(j), tm, tn, sp);
    const int acc = wg;
    if (ok) ok = mbar_wait(tfull(acc), (t_local >> 1) & 1, p.err, 4);
    tc_fence_after();
    const uint32_t tbase = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
    // this warp's TMEM loads of the tile are complete: one of the pair's 8
    // arrivals that let the MMA reuse the accumulator
    auto drained = [&]() {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_pair(acc));
    };
    uint32_t rn[CW];
    tmem_ld_cols(tbase, rn);
    tmem_wait_cols(rn);
    if (NCH == 1) drained();
#pragma unroll 1
    for (int c = 0; c < NCH; ++c, ++g) {
      const int slot = g % SL;
      float v[CW];
#pragma unroll
      for (int jj = 0; jj < CW; ++jj) v[jj] = __uint_as_float(rn[jj]);
      if (c + 1 < NCH) tmem_ld_cols(tbase + uint32_t((c + 1) * CW), rn);
      if (ok) ok = mbar_wait(inb(slot), uint32_t((g / SL) & 1), p.err, 7);
      chunk_apply<EPI, OutT, CW>(p, ebuf + slot * 8192, e, tn * BN + c * CW, v, 0.f, -1);
      // this thread's rows are written (generic proxy) before the store reads
      // them (async proxy); the warp's arrival follows all its lanes' fences
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(rdy(slot));
      if (c + 1 < NCH) {
        tmem_wait_cols(rn);
        if (c + 2 == NCH) drained();  // the tile's last TMEM load has completed
      }
    }
  }
}

// The issuer thread of warpgroup wg's chunks (epilogue_tma_split).  One
// store group may still be reading its buffer when the next chunk is taken;
// the input of chunk g + SLOTS - 1 goes into the buffer that chunk g - 1's
// store has just released.
template <int BN, int EPI, typename OutT, int NBUF>
__device__ __forceinline__ void epilogue_issuer(const TcParams& p, const CUtensorMap* mo,
                                                const CUtensorMap* mi, uint8_t* ebuf, uint64_t* tb,
                                                int wg) {
  using T = TeCfg<EPI, OutT, NBUF>;
  static_assert(T::HAS_IN && T::ARR == 1, "epilogues with an input");
  constexpr int CW = T::CW, NCH = BN / CW, SL = T::SLOTS, W = T::WAITN;
  const int rank = int(cluster_ctarank());
  const uint32_t eb = smem_u32(ebuf);
  auto inb = [&](int s) { return smem_u32(tb + kEpiIn + 8 * wg + s); };
  auto rdy = [&](int s) { return smem_u32(tb + kEpiRdy + 8 * wg + s); };
  const EpiTiles et(p, wg);
  const int total_chunks = et.my_tiles * NCH;
  // global coordinates of chunk gc: column n0, first row m0 of this CTA's half
  auto coords = [&](int gc, int& n0, int& m0) {
    int tm, tn, sp;
    tile_coords(p, et.tile(gc / NCH), tm, tn, sp);
    n0 = tn * BN + (gc % NCH) * CW;
    m0 = tm * BM2 + rank * BM;
  };
  int next_load = 0;  // next chunk whose input is to be fetched
  auto issue_load = [&]() {
    int n0, m0;
    coords(next_load, n0, m0);
    const int slot = next_load % SL;
    mbar_expect_tx(inb(slot), 8192);
    tma_load_2d(eb + slot * 8192, mi, inb(slot), n0, m0);
    ++next_load;
  };
  while (next_load < min(SL, total_chunks)) issue_load();  // every buffer starts free
  bool ok = true;
  for (int g = 0; g < total_chunks; ++g) {
    if (ok) ok = mbar_wait(rdy(g % SL), uint32_t((g / SL) & 1), p.err, 9);
    int n0, m0;
    coords(g, n0, m0);
    tma_store_2d(mo, eb + (g % SL) * 8192, n0, m0);
    bulk_commit();
    bulk_wait_read<W>();  // the stores of chunks <= g - W have read their buffers
    if (g >= W && next_load < total_chunks) issue_load();
  }
  bulk_wait_all();
  // after an expired wait some fetched inputs may never have been waited
  // for: let the last one of each buffer land before the CTA exits
  for (int gc = max(0, next_load - SL); gc < next_load; ++gc)
    mbar_wait(inb(gc % SL), uint32_t((gc / SL) & 1), p.err, 8);
}

template <int BN, int EPI, typename OutT, bool TE>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tma_a,
                   const __grid_constant__ CUtensorMap tma_b,
                   const __grid_constant__ CUtensorMap tma_o,
                   const __grid_constant__ CUtensorMap tma_o2,
                   const __grid_constant__ CUtensorMap tma_i, const TcParams p) {
  using Cfg = TcCfg<BN, TE, EPI>;
  constexpr int S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // [stages | epilogue area | barriers]; both CTAs of the pair use the same
  // offsets, which the pair's MMA and its multicast commits rely on
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * Cfg::STAGE + Cfg::EPI_BYTES);
  static_assert((2 * S + kTmemSlot + 1) * 8 <= Cfg::BAR_BYTES, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + kTmemSlot);
  const uint32_t sbase = smem_u32(smem);
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + S + s); };
  auto tfull = [&](int a) { return smem_u32(bars + 2 * S + a); };
  auto tempty = [&](int a) { return smem_u32(bars + 2 * S + 2 + a); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const int pair = int(blockIdx.x) >> 1, npairs = int(gridDim.x) >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);   // even CTA: its producer's arrive + both CTAs' bytes
      mbar_init(empty(s), 1);  // the pair's MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);   // the pair's MMA commit
      // even CTA: the epilogue arrivals of both CTAs (one per warp when the
      // epilogue has an input and TMA stores, else one per warpgroup)
      mbar_init(tempty(a), (TE && epi_has_input<EPI>()) ? 8 : 2);
    }
    for (int s = 0; s < 16; ++s) {  // TMA epilogue slots of both warpgroups
      mbar_init(smem_u32(bars + 2 * S + kEpiIn + s), 1);
      mbar_init(smem_u32(bars + 2 * S + kEpiRdy + s), 4);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 2) tmem_alloc_pair(smem_u32(tmem_slot), Cfg::TMEM_COLS);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    // Loads this CTA's half of A (rows 128 rank ..) and of B (rows BN/2 rank ..)
    // into its own ring; completion is counted on the even CTA's full barrier,
    // whose expected byte count (both halves) the even CTA's producer posts.
    const uint32_t full0 = mapa_shared(full(0), 0);
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    for (int tile = pair; tile < p.total_tiles && ok; tile += npairs) {
      int tm, tn, sp;
      tile_coords(p, tile, tm, tn, sp);
      const int kb0 = sp * p.kb_per_split, kb1 = min(p.num_kb, kb0 + p.kb_per_split);
      const int ma = tm * BM2 + int(rank) * BM, nb = tn * BN + int(rank) * (BN / 2);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1, p.err, 1)) {
          ok = false;
          break;
        }
        if (rank == 0) mbar_expect_tx(full(stage), 2 * Cfg::STAGE);
        const uint32_t fb = full0 + uint32_t(stage * 8);
        const uint32_t sa = sbase + stage * Cfg::STAGE, sb = sa + Cfg::A_BYTES;
        const int k0 = kb * BK;
        if (!p.a_mn) {
          tma_load_2d_pair(sa, &tma_a, fb, k0, ma);
        } else {
          tma_load_2d_pair(sa, &tma_a, fb, ma, k0);
          tma_load_2d_pair(sa + BK * 128, &tma_a, fb, ma + 64, k0);
        }
        if (!p.b_mn) {
          tma_load_2d_pair(sb, &tma_b, fb, k0, nb);
        } else {
#pragma unroll
          for (int j = 0; j < BN / 128; ++j)
            tma_load_2d_pair(sb + j * BK * 128, &tma_b, fb, nb + 64 * j, k0);
        }
        ++issued;
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    // the MMA has consumed (so the copies have landed in) the last issued stages
    for (int q = 1; q <= min(issued, S); ++q) {
      const int idx = issued - q;
      mbar_wait(empty(idx % S), uint32_t((idx / S) & 1), p.err, 5);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------ MMA issuer (even CTA)
    const uint32_t idesc = gemm_idesc<BN>(p.a_mn, p.b_mn);
    // descriptors of stage 0, k-slice 0; a stage is STAGE bytes further, a
    // 16-element k-slice +2 (K-major) or +128 (MN-major) in the address field
    const uint64_t a0 = p.a_mn ? desc_mnmajor(sbase, 0) : desc_kmajor(sbase, 0);
    const uint64_t b0 = p.b_mn ? desc_mnmajor(sbase + Cfg::A_BYTES, 0)
                               : desc_kmajor(sbase + Cfg::A_BYTES, 0);
    const uint64_t a_k = p.a_mn ? 128 : 2, b_k = p.b_mn ? 128 : 2;
    int stage = 0;
    uint32_t phase = 0;
    int t_local = 0;
    bool ok = true;
    for (int tile = pair; tile < p.total_tiles && ok; tile += npairs, ++t_local) {
      int tm, tn, sp;
      tile_coords(p, tile, tm, tn, sp);
      const int kb0 = sp * p.kb_per_split, kb1 = min(p.num_kb, kb0 + p.kb_per_split);
      const int acc = t_local & 1;
      // arrivals of both CTAs' epilogues (release at cluster scope)
      if (!mbar_wait_cluster(tempty(acc), ((t_local >> 1) & 1) ^ 1, p.err, 2)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + uint32_t(acc * BN);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full(stage), phase, p.err, 3)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = desc_offset(a0, stage * Cfg::STAGE);
        const uint64_t bd = desc_offset(b0, stage * Cfg::STAGE);
        if (kb == kb0)  // the tile's first MMA overwrites the accumulator
          umma_pair_i<0>(d, ad, bd, idesc);
        else
          umma_pair_i<1>(d, ad, bd, idesc);
#pragma unroll
        for (int k = 1; k < BK / UMMA_K; ++k) umma_pair_i<1>(d, ad + k * a_k, bd + k * b_k, idesc);
        umma_commit_pair(empty(stage), 3);  // frees the stage in both CTAs
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      umma_commit_pair(tfull(acc), 3);  // both halves of the accumulator ready
    }
    // all issued MMAs complete before TMEM is released
    if (t_local > 0) {
      const int last = t_local - 1;
      mbar_wait(tfull(last & 1), uint32_t((last >> 1) & 1), p.err, 6);
    }
  } else if ((warp == 2 || warp == 3) && lane == 0 && TE && epi_has_input<EPI>()) {
    // ------------------------------------------------ TMA issuer of epilogue warpgroup warp - 2
    const int wg = warp - 2;
    if constexpr (TE && epi_has_input<EPI>())
      epilogue_issuer<BN, EPI, OutT, Cfg::NBUF_WG>(
          p, &tma_o, &tma_i, smem + S * Cfg::STAGE + wg * Cfg::WG_BYTES, bars + 2 * S, wg);
  } else if (warp >= 4 && TE) {
    // ------------------------------------------------ epilogue warpgroup (TMA stores)
    const int wg = (warp - 4) >> 2;  // warpgroup wg drains accumulator wg
    uint8_t* ebuf = smem + S * Cfg::STAGE + wg * Cfg::WG_BYTES;
    if constexpr (TE && epi_has_input<EPI>())
      epilogue_tma_split<BN, EPI, OutT, Cfg::NBUF_WG>(p, ebuf, bars + 2 * S, tmem_base, wg);
    else if constexpr (TE)
      epilogue_tma<BN, EPI, OutT, Cfg::NBUF_WG>(p, &tma_o, &tma_o2, ebuf, bars + 2 * S, tmem_base,
                                                wg);
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue warpgroup
    // TMEM phase: thread e (= row 128 rank + e of the tile, TMEM lane e)
    // loads 32 accumulator columns and stages them in shared memory; store
    // phase: the 128 threads apply the epilogue op to row segments and write
    // them coalesced.
    // Warpgroup wg (warps 4-7 or 8-11) drains accumulator wg: the pair's
    // local tiles wg, wg+2, ...
    const int wg = (warp - 4) >> 2;
    const int bar_id = 1 + wg;
    const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
    const int e = threadIdx.x - 128 - 128 * wg;
    float* stg = reinterpret_cast<float*>(smem + S * Cfg::STAGE + wg * Cfg::WG_BYTES);
    constexpr int SR = Cfg::STAGE_ROW;
    const uint32_t tempty0 = mapa_shared(tempty(0), 0);
    bool ok = true;
    for (int t_local = wg, tile = pair + wg * npairs; tile < p.total_tiles;
         t_local += 2, tile += 2 * npairs) {
      int tm, tn, sp;
      tile_coords(p, tile, tm, tn, sp);
      const int acc = wg;
      const int m0 = tm * BM2 + int(rank) * BM;
      // an expired wait (error word set) skips later waits, never the barriers
      if (ok) ok = mbar_wait(tfull(acc), (t_local >> 1) & 1, p.err, 4);
      tc_fence_after();
      const int m_row = m0 + e;
      int row_tgt = -1;
      if (EPI == EPI_LSE_PARTIAL && m_row < p.M) row_tgt = p.ep.tgt[m_row];
      float run_m = -INFINITY, run_s = 0.f, zt = 0.f;
      bool has_t = false;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        __syncwarp();
        float v[32];
        tmem_ld32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN + c0), v);
        const int n0 = tn * BN + c0;
        if (EPI == EPI_LSE_PARTIAL) {
          if (m_row >= p.M || n0 >= p.N) continue;
          // running max / sum of exp over this tile's valid columns
          const bool whole = n0 + 32 <= p.N;
          float cm = -INFINITY;
          if (whole) {
#pragma unroll
            for (int j = 0; j < 32; ++j) cm = fmaxf(cm, v[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < p.N) cm = fmaxf(cm, v[j]);
          }
          const float nm = fmaxf(run_m, cm);
          const float nml = nm * kLog2e;
          float sacc = 0.f;
          if (whole) {
#pragma unroll
            for (int j = 0; j < 32; ++j) sacc += ex2_hw(fmaf(v[j], kLog2e, -nml));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < p.N) sacc += ex2_hw(fmaf(v[j], kLog2e, -nml));
          }
          run_s = run_s * ex2_hw((run_m - nm) * kLog2e) + sacc;
          run_m = nm;
          if (row_tgt >= n0 && row_tgt < n0 + 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j == row_tgt) zt = v[j];
            has_t = true;
          }
          continue;
        }
        if (n0 >= p.N) continue;  // uniform over the warpgroup
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(stg + e * SR + j) =
              make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        epi_bar(bar_id);
        if (p.ws || sizeof(OutT) == 4)
          epi_store_chunk<EPI, OutT, 4>(p, stg, SR, e, m0, n0, sp);
        else
          epi_store_chunk<EPI, OutT, 8>(p, stg, SR, e, m0, n0, sp);
        epi_bar(bar_id);
      }
      if (EPI == EPI_LSE_PARTIAL && m_row < p.M) {
        p.ep.part_max[int64_t(m_row) * p.ep.part_ld + tn] = run_m;
        p.ep.part_sum[int64_t(m_row) * p.ep.part_ld + tn] = run_s;
        if (has_t) p.ep.tgt_logit[m_row] = zt;
      }
      // all 128 threads' TMEM loads done: one arrival for this CTA's half
      tc_fence_before();
      epi_bar(bar_id);
      if (e == 0) mbar_arrive_cluster(tempty0 + uint32_t(acc * 8));
    }
  }
  // neither CTA leaves (freeing shared memory and TMEM that the pair's MMA,
  // commits and arrivals address) before both are done
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
}

// Split-K reduction, splits added in order, then the GEMM's epilogue on the
// sum (this kernel: every kind; the vectorised one below: EPI_STORE and
// EPI_ACC):
//   EPI_ACC:   out = (accumulate ? out : 0) + alpha * sum_z ws[z]      (fp32)
//   EPI_STORE: out = alpha * sum_z ws[z] + bias[n]                    (OutT)
template <typename OutT>
__global__ void tc_splitk_reduce_kernel(const float* __restrict__ ws, int splits, int M, int N,
                                        EpiParams e) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= int64_t(M) * N) return;
  const int m = int(i / N), n = int(i % N);
  float acc = 0.f;
  for (int z = 0; z < splits; ++z) acc += ws[int64_t(z) * M * N + i];
  epi_apply<OutT>(e, e.kind, m, n, acc);  // the GEMM's own epilogue on the summed value
}

// Same reduction, four columns per thread (N and ldo multiples of 4), rows
// strided over blockIdx.y.
template <typename OutT>
__global__ void tc_splitk_reduce4_kernel(const float* __restrict__ ws, int splits, int M, int N,
                                         EpiParams e) {
  const int n = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (n >= N) return;
  const int64_t plane = int64_t(M) * N;
  for (int m = blockIdx.y; m < M; m += gridDim.y) {
    const int64_t i = int64_t(m) * N + n;
    float4 a = *reinterpret_cast<const float4*>(ws + i);
    for (int z = 1; z < splits; ++z) {
      const float4 b = *reinterpret_cast<const float4*>(ws + z * plane + i);
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    const int64_t o = int64_t(m) * e.ldo + n;
    if (e.kind == EPI_ACC) {
      float4* out = reinterpret_cast<float4*>(reinterpret_cast<float*>(e.out) + o);
      float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e.accumulate) r = *out;
      *out = make_float4(r.x + e.alpha * a.x, r.y + e.alpha * a.y, r.z + e.alpha * a.z,
                         r.w + e.alpha * a.w);
    } else {
      float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e.bias) b = *reinterpret_cast<const float4*>(e.bias + n);
      float v[4] = {e.alpha * a.x + b.x, e.alpha * a.y + b.y, e.alpha * a.z + b.z,
                    e.alpha * a.w + b.w};
      store_vec<OutT, 4>(reinterpret_cast<OutT*>(e.out) + o, v);
    }
  }
}

// ------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Number of CTA pairs that can be resident at once (1 CTA per SM; not every
// SM need have a partner in its cluster domain).
int pair_slots();

// Split-K count for 256 x 256 pair tiles: the estimated time is the rounds of
// persistent tiles over the resident pairs times the MMA time of one tile,
// plus, with split-K, the traffic of the partial sums and one more launch.
// Only plain stores and gradient accumulation may split.
int choose_splits_tc(int M, int N, int K, bool splittable, size_t ws_bytes) {
  const int pairs = pair_slots();
  const int kb = cdiv(K, BK);
  const int tiles = cdiv(M, BM2) * cdiv(N, 256);
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= (splittable ? 16 : 1); ++s) {
    if (s > 1 && kb / s < 4) break;
    const int kbs = cdiv(kb, s), se = cdiv(kb, kbs);
    if (se > 1 && size_t(se) * M * N * sizeof(float) > ws_bytes) break;
    const double tile_s = 2.0 * BM2 * 256 * kbs * BK / (2 * 15.5e12) + 0.5e-6;
    double cost = cdiv(tiles * se, pairs) * tile_s;
    if (se > 1) cost += double(M) * N * 4.0 * (se + 1) / 4.0e12 + 5e-6;
    if (cost < best_cost * 0.97) {
      best_cost = cost;
      best = se;
    }
  }
  return best;
}

int pair_slots() {
  static int slots = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    using Cfg = TcCfg<256, true, EPI_STORE>;
    auto kern = gemm_tc_kernel<256, EPI_STORE, bf16, true>;
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * gpt2_internal::sm_count());
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = Cfg::SMEM;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    (void)cudaGetLastError();  // no device (build hosts): fall back to SMs / 2
    slots = n > 0 ? n : std::max(1, gpt2_internal::sm_count() / 2);
  });
  return slots;
}

// The TMA epilogue needs 16-byte aligned arrays and rows (tensor-map rules);
// split-K partial tiles (but those of weight gradients over whole 256-row
// tiles) and the LSE-partial epilogue use the staged path.
bool te_eligible(const GemmArgs& g, int splits) {
  auto al16 = [](const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (splits != 1) {
    // fp32 weight-gradient partial sums by TMA into the workspace viewed as
    // [splits * M, N]: whole 256-row tiles only, so no tile reaches into the
    // next split's rows
    return g.ep.kind == EPI_ACC && g.M % BM2 == 0 && (g.N * 4) % 16 == 0 && al16(g.ws);
  }
  if (g.ep.kind == EPI_LSE_PARTIAL) return false;
  const int eb = (g.ep.kind == EPI_RESID || g.ep.kind == EPI_ACC || !g.ep.out_bf16) ? 4 : 2;
  if ((g.ep.ldo * eb) % 16 != 0) return false;
  switch (g.ep.kind) {
    case EPI_RESID: return al16(g.ep.rin) && al16(g.ep.rout);
    case EPI_GELU: return al16(g.ep.out) && al16(g.ep.out2);
    case EPI_GELU_BWD: return al16(g.ep.out) && al16(g.ep.aux);
    default: return al16(g.ep.out);
  }
}

template <int BN, int EPI, typename OutT, bool TE>
int launch_tc(const GemmArgs& g, int splits, cudaStream_t st) {
  using Cfg = TcCfg<BN, TE, EPI>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI, OutT, TE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) {
      gpt2_internal::set_error(std::string("tc gemm smem attribute: ") + cudaGetErrorString(e));
      return GPT2_ERR_CUDA;
    }
    attr_set = true;
  }
  CUtensorMap ma, mb, mo, mo2, mi;
  memset(&mo, 0, sizeof(mo));
  memset(&mo2, 0, sizeof(mo2));
  memset(&mi, 0, sizeof(mi));
  // boxes of one CTA's half: 128 rows of A, BN/2 rows of B
  bool ok = g.a_kmajor ? tc::make_map_bf16(&ma, g.A, g.K, g.M, g.lda, BM)
                       : tc::make_map_bf16(&ma, g.A, g.M, g.K, g.lda, BK);
  ok = ok && (g.b_kmajor ? tc::make_map_bf16(&mb, g.B, g.K, g.N, g.ldb, BN / 2)
                         : tc::make_map_bf16(&mb, g.B, g.N, g.K, g.ldb, BK));
  if (TE) {
    constexpr int eb = int(sizeof(OutT));
    const void* o = EPI == EPI_RESID ? static_cast<const void*>(g.ep.rout) : g.ep.out;
    if (EPI == EPI_ACC && splits > 1)
      ok = ok && tc::make_map_epi(&mo, g.ws, 4, g.N, int64_t(splits) * g.M, g.N);
    else
      ok = ok && tc::make_map_epi(&mo, o, eb, g.N, g.M, g.ep.ldo);
    if (EPI == EPI_GELU) ok = ok && tc::make_map_epi(&mo2, g.ep.out2, eb, g.N, g.M, g.ep.ldo);
    if (EPI == EPI_RESID) ok = ok && tc::make_map_epi(&mi, g.ep.rin, 4, g.N, g.M, g.ep.ldo);
    if (EPI == EPI_GELU_BWD) ok = ok && tc::make_map_epi(&mi, g.ep.aux, eb, g.N, g.M, g.ep.ldo);
  }
  if (!ok) {
    gpt2_internal::set_error("tc gemm: tensor map encoding failed");
    return GPT2_ERR_CUDA;
  }
  TcParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.a_mn = g.a_kmajor ? 0 : 1;
  p.b_mn = g.b_kmajor ? 0 : 1;
  p.tiles_m = cdiv(g.M, BM2);
  p.tiles_n = cdiv(g.N, BN);
  p.num_kb = cdiv(g.K, BK);
  p.kb_per_split = cdiv(p.num_kb, splits);
  p.splits = cdiv(p.num_kb, p.kb_per_split);
  p.total_tiles = p.tiles_m * p.tiles_n * p.splits;
  p.n_fast = g.M > g.N ? 1 : 0;  // A (M x K) is the larger operand: read its panels once
  p.ep = g.ep;
  p.ws = p.splits > 1 ? g.ws : nullptr;
  p.err = device_error_word();
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * std::min(p.total_tiles, pair_slots()));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, EPI, OutT, TE>, ma, mb, mo, mo2, mi, p);
  if (le != cudaSuccess) {
    gpt2_internal::set_error(std::string("tc gemm launch: ") + cudaGetErrorString(le));
    return GPT2_ERR_CUDA;
  }
  COUNT_LAUNCH(1);
  if (p.splits > 1) {
    const bool vec = (g.ep.kind == EPI_STORE || g.ep.kind == EPI_ACC) && (g.N % 4) == 0 &&
                     (g.ep.ldo % 4) == 0 &&
                     (!g.ep.bias || (reinterpret_cast<uintptr_t>(g.ep.bias) & 15) == 0);
    if (vec) {
      const dim3 grid(cdiv(g.N / 4, 128), std::min(g.M, 2048));
      tc_splitk_reduce4_kernel<OutT><<<grid, 128, 0, st>>>(g.ws, p.splits, g.M, g.N, g.ep);
    } else {
      const int64_t n = int64_t(g.M) * g.N;
      tc_splitk_reduce_kernel<OutT><<<int(cdiv64(n, 256)), 256, 0, st>>>(g.ws, p.splits, g.M, g.N,
                                                                         g.ep);
    }
    COUNT_LAUNCH(1);
  }
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template <int BN, int EPI, typename OutT>
int launch_te(const GemmArgs& g, int splits, cudaStream_t st) {
  return te_eligible(g, splits) ? launch_tc<BN, EPI, OutT, true>(g, splits, st)
                                : launch_tc<BN, EPI, OutT, false>(g, splits, st);
}

template <int BN>
int dispatch_epi(const GemmArgs& g, int splits, cudaStream_t st) {
  const bool ob = g.ep.out_bf16;
  switch (g.ep.kind) {
    case EPI_STORE:
      return ob ? launch_te<BN, EPI_STORE, bf16>(g, splits, st)
                : launch_te<BN, EPI_STORE, float>(g, splits, st);
    case EPI_GELU: return launch_te<BN, EPI_GELU, bf16>(g, splits, st);
    case EPI_RESID: return launch_te<BN, EPI_RESID, float>(g, splits, st);
    case EPI_ACC: return launch_te<BN, EPI_ACC, float>(g, splits, st);
    case EPI_GELU_BWD: return launch_te<BN, EPI_GELU_BWD, bf16>(g, splits, st);
    case EPI_CE_GRAD: return launch_te<BN, EPI_CE_GRAD, bf16>(g, splits, st);
    case EPI_LSE_PARTIAL: return launch_tc<BN, EPI_LSE_PARTIAL, float, false>(g, splits, st);
  }
  gpt2_internal::set_error("tc gemm: unknown epilogue");
  return GPT2_ERR_ARG;
}

}  // namespace

namespace tc {
bool make_map_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld,
                   int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(outer)};
  cuuint64_t strides[1] = {cuuint64_t(ld) * 2};
  cuuint32_t box[2] = {64, cuuint32_t(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
bool make_map_epi(CUtensorMap* map, const void* base, int elem_bytes, int64_t inner,
                  int64_t outer, int64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(outer)};
  cuuint64_t strides[1] = {cuuint64_t(ld) * cuuint64_t(elem_bytes)};
  cuuint32_t box[2] = {cuuint32_t(64 / elem_bytes), 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace tc

bool gemm_tc_supported(const GemmArgs& g) {
  if (!g.bf16_in || !encode_fn()) return false;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(g.A) || !al16(g.B) || (g.lda & 7) || (g.ldb & 7)) return false;
  if (g.ep.out && (!al16(g.ep.out) || (g.ep.ldo & 7))) return false;
  if (g.ep.kind == EPI_LSE_PARTIAL && (!g.ep.part_max || !g.ep.part_sum || !g.ep.tgt_logit))
    return false;
  if ((g.ep.kind == EPI_GELU || g.ep.kind == EPI_GELU_BWD || g.ep.kind == EPI_CE_GRAD) &&
      !g.ep.out_bf16)
    return false;
  if (g.ep.kind == EPI_RESID && (!al16(g.ep.rin) || !al16(g.ep.rout) || (g.ep.ldo & 7)))
    return false;
  if (g.ep.bias && !al16(g.ep.bias)) return false;
  return true;
}

size_t gemm_tc_workspace_bytes(int M, int N, int K) {
  const int sp = choose_splits_tc(M, N, K, true, SIZE_MAX);
  return sp > 1 ? size_t(sp) * M * N * sizeof(float) : 0;
}

int gemm_tc_launch(const GemmArgs& g, cudaStream_t st) {
  // split-K needs the workspace; its reduction applies any epilogue but the
  // LM-head ones (the cost model splits only when the output tiles leave most
  // CTA pairs idle, e.g. the one-row GEMMs of incremental decoding)
  const bool splittable = g.ep.kind != EPI_LSE_PARTIAL && g.ep.kind != EPI_CE_GRAD && g.ws;
  const int sp = choose_splits_tc(g.M, g.N, g.K, splittable, splittable ? g.ws_bytes : 0);
  return dispatch_epi<256>(g, sp, st);
}
