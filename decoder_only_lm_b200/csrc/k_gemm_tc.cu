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
//     warps 4-7 (one warpgroup) drain the accumulator with tcgen05.ld and run
//     the epilogue;
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
#include <mutex>

#include "epilogue.cuh"
#include "tc_common.cuh"

using namespace tc;

namespace {

constexpr int BM = 128, UMMA_K = 16;
constexpr int kThreads = 256;

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int STAGE_ROW = 36;  // fp32 per staged accumulator row (32 + 4 pad)
  static constexpr int EPI_BYTES = BM * STAGE_ROW * 4;
  static constexpr int SMEM = STAGES * STAGE + EPI_BYTES + BAR_BYTES + 1024;
};

struct TcParams {
  int M, N, K;
  int a_mn, b_mn;
  int tiles_m, tiles_n, splits, kb_per_split, num_kb, total_tiles;
  EpiParams ep;
  float* ws;
  int* err;
};

// Instruction descriptor: kind::f16, bf16 A and B, fp32 D, M = 128, N = BN.
template <int BN>
__device__ __forceinline__ uint32_t gemm_idesc(int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
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

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

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

template <int BN, int EPI, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tma_a,
                   const __grid_constant__ CUtensorMap tma_b, const TcParams p) {
  using Cfg = TcCfg<BN>;
  constexpr int S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * Cfg::STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);
  const uint32_t sbase = smem_u32(smem);
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + S + s); };
  auto tfull = [&](int a) { return smem_u32(bars + 2 * S + a); };
  auto tempty = [&](int a) { return smem_u32(bars + 2 * S + 2 + a); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 128);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 2) tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.total_tiles && ok; tile += gridDim.x) {
      const int tm = tile % p.tiles_m;
      const int rest = tile / p.tiles_m;
      const int tn = rest % p.tiles_n, sp = rest / p.tiles_n;
      const int kb0 = sp * p.kb_per_split, kb1 = min(p.num_kb, kb0 + p.kb_per_split);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1, p.err, 1)) {
          ok = false;
          break;
        }
        mbar_expect_tx(full(stage), Cfg::STAGE);
        const uint32_t sa = sbase + stage * Cfg::STAGE, sb = sa + Cfg::A_BYTES;
        const int k0 = kb * BK;
        if (!p.a_mn) {
          tma_load_2d(sa, &tma_a, full(stage), k0, tm * BM);
        } else {
          tma_load_2d(sa, &tma_a, full(stage), tm * BM, k0);
          tma_load_2d(sa + BK * 128, &tma_a, full(stage), tm * BM + 64, k0);
        }
        if (!p.b_mn) {
          tma_load_2d(sb, &tma_b, full(stage), k0, tn * BN);
        } else {
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sb + j * BK * 128, &tma_b, full(stage), tn * BN + 64 * j, k0);
        }
        ++issued;
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    // wait until the copies of the last (up to S) issued stages have landed
    for (int q = 1; q <= min(issued, S); ++q) {
      const int idx = issued - q;
      mbar_wait(full(idx % S), uint32_t((idx / S) & 1), p.err, 5);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    const uint32_t idesc = gemm_idesc<BN>(p.a_mn, p.b_mn);
    int stage = 0;
    uint32_t phase = 0;
    int t_local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.total_tiles && ok; tile += gridDim.x, ++t_local) {
      const int rest = tile / p.tiles_m;
      const int sp = rest / p.tiles_n;
      const int kb0 = sp * p.kb_per_split, kb1 = min(p.num_kb, kb0 + p.kb_per_split);
      const int acc = t_local & 1;
      if (!mbar_wait(tempty(acc), ((t_local >> 1) & 1) ^ 1, p.err, 2)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + uint32_t(acc * BN);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full(stage), phase, p.err, 3)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = sbase + stage * Cfg::STAGE, sb = sa + Cfg::A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k) {
          const uint64_t ad = p.a_mn ? desc_mnmajor(sa, k) : desc_kmajor(sa, k);
          const uint64_t bd = p.b_mn ? desc_mnmajor(sb, k) : desc_kmajor(sb, k);
          umma_bf16(d, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
        }
        umma_commit(empty(stage));
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      umma_commit(tfull(acc));
    }
    // all issued MMAs complete before TMEM is released
    if (t_local > 0) {
      const int last = t_local - 1;
      mbar_wait(tfull(last & 1), uint32_t((last >> 1) & 1), p.err, 6);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue warpgroup
    // TMEM phase: thread e (= tile row e, TMEM lane e) loads 32 accumulator
    // columns and stages them in shared memory; store phase: the 128 threads
    // apply the epilogue op to row segments and write them coalesced.
    const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
    const int e = threadIdx.x - 128;
    float* stg = reinterpret_cast<float*>(smem + S * Cfg::STAGE);
    constexpr int SR = Cfg::STAGE_ROW;
    int t_local = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++t_local) {
      const int tm = tile % p.tiles_m;
      const int rest = tile / p.tiles_m;
      const int tn = rest % p.tiles_n, sp = rest / p.tiles_n;
      const int acc = t_local & 1;
      bool ok = mbar_wait(tfull(acc), (t_local >> 1) & 1, p.err, 4);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int m_row = tm * BM + e;
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
          float cm = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (n0 + j < p.N) cm = fmaxf(cm, v[j]);
          const float nm = fmaxf(run_m, cm);
          float sacc = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (n0 + j < p.N) sacc += __expf(v[j] - nm);
          run_s = run_s * __expf(run_m - nm) + sacc;
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
        epi_bar();
        if (p.ws || sizeof(OutT) == 4)
          epi_store_chunk<EPI, OutT, 4>(p, stg, SR, e, tm * BM, n0, sp);
        else
          epi_store_chunk<EPI, OutT, 8>(p, stg, SR, e, tm * BM, n0, sp);
        epi_bar();
      }
      if (EPI == EPI_LSE_PARTIAL && m_row < p.M) {
        p.ep.part_max[int64_t(m_row) * p.ep.part_ld + tn] = run_m;
        p.ep.part_sum[int64_t(m_row) * p.ep.part_ld + tn] = run_s;
        if (has_t) p.ep.tgt_logit[m_row] = zt;
      }
      tc_fence_before();
      mbar_arrive(tempty(acc));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
}

// Split-K reduction, splits added in order:
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
  const int64_t o = int64_t(m) * e.ldo + n;
  if (e.kind == EPI_ACC) {
    float* out = reinterpret_cast<float*>(e.out);
    out[o] = (e.accumulate ? out[o] : 0.f) + e.alpha * acc;
  } else {
    reinterpret_cast<OutT*>(e.out)[o] = from_f32<OutT>(e.alpha * acc + (e.bias ? e.bias[n] : 0.f));
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

int choose_splits_tc(int tiles, int num_kb) {
  const int sms = gpt2_internal::sm_count();
  if (tiles * 2 > sms) return 1;
  int s = std::min(16, sms / tiles);
  while (s > 1 && num_kb / s < 4) --s;
  return s;
}

template <int BN, int EPI, typename OutT>
int launch_tc(const GemmArgs& g, int splits, cudaStream_t st) {
  using Cfg = TcCfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI, OutT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) {
      gpt2_internal::set_error(std::string("tc gemm smem attribute: ") + cudaGetErrorString(e));
      return GPT2_ERR_CUDA;
    }
    attr_set = true;
  }
  CUtensorMap ma, mb;
  const bool okA = g.a_kmajor ? tc::make_map_bf16(&ma, g.A, g.K, g.M, g.lda, BM)
                              : tc::make_map_bf16(&ma, g.A, g.M, g.K, g.lda, BK);
  const bool okB = g.b_kmajor ? tc::make_map_bf16(&mb, g.B, g.K, g.N, g.ldb, BN)
                              : tc::make_map_bf16(&mb, g.B, g.N, g.K, g.ldb, BK);
  if (!okA || !okB) {
    gpt2_internal::set_error("tc gemm: tensor map encoding failed");
    return GPT2_ERR_CUDA;
  }
  TcParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.a_mn = g.a_kmajor ? 0 : 1;
  p.b_mn = g.b_kmajor ? 0 : 1;
  p.tiles_m = cdiv(g.M, BM);
  p.tiles_n = cdiv(g.N, BN);
  p.num_kb = cdiv(g.K, BK);
  p.kb_per_split = cdiv(p.num_kb, splits);
  p.splits = cdiv(p.num_kb, p.kb_per_split);
  p.total_tiles = p.tiles_m * p.tiles_n * p.splits;
  p.ep = g.ep;
  p.ws = p.splits > 1 ? g.ws : nullptr;
  p.err = device_error_word();
  const int grid = std::min(p.total_tiles, gpt2_internal::sm_count());
  gemm_tc_kernel<BN, EPI, OutT><<<grid, kThreads, Cfg::SMEM, st>>>(ma, mb, p);
  COUNT_LAUNCH(1);
  if (p.splits > 1) {
    const int64_t n = int64_t(g.M) * g.N;
    tc_splitk_reduce_kernel<OutT><<<int(cdiv64(n, 256)), 256, 0, st>>>(g.ws, p.splits, g.M, g.N,
                                                                       g.ep);
    COUNT_LAUNCH(1);
  }
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

template <int BN>
int dispatch_epi(const GemmArgs& g, int splits, cudaStream_t st) {
  const bool ob = g.ep.out_bf16;
  switch (g.ep.kind) {
    case EPI_STORE:
      return ob ? launch_tc<BN, EPI_STORE, bf16>(g, splits, st)
                : launch_tc<BN, EPI_STORE, float>(g, splits, st);
    case EPI_GELU: return launch_tc<BN, EPI_GELU, bf16>(g, splits, st);
    case EPI_RESID: return launch_tc<BN, EPI_RESID, float>(g, splits, st);
    case EPI_ACC: return launch_tc<BN, EPI_ACC, float>(g, splits, st);
    case EPI_GELU_BWD: return launch_tc<BN, EPI_GELU_BWD, bf16>(g, splits, st);
    case EPI_CE_GRAD: return launch_tc<BN, EPI_CE_GRAD, bf16>(g, splits, st);
    case EPI_LSE_PARTIAL: return launch_tc<BN, EPI_LSE_PARTIAL, float>(g, splits, st);
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

int gemm_tc_tile_n() { return 256; }

size_t gemm_tc_workspace_bytes(int M, int N, int K) {
  const int tiles = cdiv(M, BM) * cdiv(N, 256);
  const int s = choose_splits_tc(tiles, cdiv(K, BK));
  return s > 1 ? size_t(s) * M * N * sizeof(float) : 0;
}

int gemm_tc_launch(const GemmArgs& g, cudaStream_t st) {
  constexpr int BN = 256;
  int splits = 1;
  if (g.ep.kind == EPI_ACC || g.ep.kind == EPI_STORE) {
    splits = choose_splits_tc(cdiv(g.M, BM) * cdiv(g.N, BN), cdiv(g.K, BK));
    if (!g.ws || size_t(splits) * g.M * g.N * sizeof(float) > g.ws_bytes) splits = 1;
  }
  return dispatch_epi<BN>(g, splits, st);
}
