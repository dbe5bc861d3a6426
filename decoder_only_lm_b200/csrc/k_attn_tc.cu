// Causal flash attention on the 5th-generation tensor cores (tcgen05 MMAs with
// TMEM accumulators, operands loaded by TMA), head size 64, bf16 in / fp32
// accumulate [ZERO: Attention, OpFlashAttention recomputes the scores in the
// backward; LECTURE: flash attention, causal mask].  The [T, T] scores and
// probabilities never leave TMEM, registers and shared memory.
//
// Every kernel: one CTA of 192 threads per block of 128 rows (queries, or keys
// in dK/dV) = the 128 TMEM lanes, streaming 64-row tiles of the other operand:
//   warp 0, one lane   TMA loads (128-row tile once, 64-row tiles in a ring);
//   warp 1             owns the TMEM allocation (256 columns); one lane issues
//                      the tcgen05.mma instructions and commits;
//   warps 2-5          elementwise warpgroup, thread = row (TMEM lane
//                      32 * (warp % 4) + lane): reads the score tile from TMEM,
//                      writes probabilities / score gradients as bf16 K-major
//                      operands (128-byte swizzle) to shared memory.
// 256 TMEM columns and < 100 KB of shared memory let two CTAs share an SM, so
// one CTA's elementwise work overlaps the other's MMAs.
//
// Forward (per 128 queries, 64-key tiles j <= diagonal):
//   S_j = Q K_j^T (TMEM, double buffered); m, l kept in the log2 domain; the
//   O accumulator (TMEM) is rescaled only when a row maximum grows by more than
//   2^8 (probabilities are taken relative to the kept maximum, so they stay
//   <= 256); P_j double buffered in shared memory; O += P_j V_j (V MN-major).
// Backward, with Delta_i = dO_i . O_i and P = exp(S / sqrt(D) - lse):
//   dK/dV kernel (per 128 keys, 64-query tiles i >= keys): S^T, dP^T = V dO^T,
//   dS^T = P^T (dP^T - Delta); dV += P^T dO, dK += dS^T Q / sqrt(D);
//   dQ kernel (per 128 queries, 64-key tiles): S, dP, dS; dQ += dS K / sqrt(D).
// Both recompute P, so no two CTAs add into one element (deterministic).
// Every wait is bounded (2 s of global time) and reports a timeout in the
// error word instead of hanging.

#include "tc_common.cuh"

using namespace tc;

namespace {

constexpr int D = 64;
constexpr int BR = 128;                 // rows per CTA = TMEM lanes
constexpr int BS = 64;                  // rows of a streamed tile
constexpr int kRowTile = BR * D * 2;    // 16 KB: 128 x 64 bf16
constexpr int kStrTile = BS * D * 2;    // 8 KB: 64 x 64 bf16
constexpr int kOpTile = BR * BS * 2;    // 16 KB: 128 x 64 bf16 operand from the warpgroup
constexpr int kTmemCols = 256;
constexpr int kThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;         // lazy-rescale threshold, log2 units

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
// three-input maximum (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// packed pair arithmetic of sm_100: (a0, a1) * (b0, b1) + (c0, c1) and (a0, a1) + (b0, b1)
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                     float c0, float c1) {
  uint64_t ra, rb, rc, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b0), "f"(b1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c0), "f"(c1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(rd));
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1) {
  uint64_t ra, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rd) : "f"(d0), "f"(d1));
  asm("add.rn.f32x2 %0, %0, %1;" : "+l"(rd) : "l"(ra));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(rd));
}
__device__ __forceinline__ void mul2(float& d0, float& d1, float a0, float a1) {
  uint64_t ra, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rd) : "f"(d0), "f"(d1));
  asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(rd) : "l"(ra));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(rd));
}
// maximum of 64 values as four independent chains of three-input maxima
__device__ __forceinline__ float max64(const float (&x)[64]) {
  float c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float* y = x + 16 * k;
    float a = max3f(y[0], y[1], y[2]);
#pragma unroll
    for (int i = 3; i < 15; i += 2) a = max3f(a, y[i], y[i + 1]);
    c[k] = fmaxf(a, y[15]);
  }
  return max3f(c[0], c[1], fmaxf(c[2], c[3]));
}
__device__ __forceinline__ void wg_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Row e of a 128 x 64 K-major bf16 operand tile (128-byte swizzle) from 32
// packed bf16 pairs.
__device__ __forceinline__ void put_row64(uint8_t* tile, int e, const uint32_t (&pk)[32]) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch)
    *reinterpret_cast<uint4*>(tile + e * 128 + ((ch ^ (e & 7)) << 4)) =
        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
}

// Writes a 64-element fp32 row (two 32-column chunks) as bf16, times scale.
__device__ __forceinline__ void store_row64(bf16* dst, const uint32_t (&a)[32],
                                            const uint32_t (&b)[32], float scale) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      const uint32_t* src = h ? b : a;
      uint4 u;
      u.x = pack2(__uint_as_float(src[8 * ch]) * scale, __uint_as_float(src[8 * ch + 1]) * scale);
      u.y = pack2(__uint_as_float(src[8 * ch + 2]) * scale, __uint_as_float(src[8 * ch + 3]) * scale);
      u.z = pack2(__uint_as_float(src[8 * ch + 4]) * scale, __uint_as_float(src[8 * ch + 5]) * scale);
      u.w = pack2(__uint_as_float(src[8 * ch + 6]) * scale, __uint_as_float(src[8 * ch + 7]) * scale);
      *reinterpret_cast<uint4*>(dst + 32 * h + 8 * ch) = u;
    }
}

__device__ __forceinline__ void init_bar_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ====================================================================== forward
constexpr int NSF = 3;  // K/V stages
constexpr int kFwdSmem = kRowTile + NSF * 2 * kStrTile + 2 * kOpTile + 256 + 1024;

struct FwdParams {
  int T, C, H;
  bf16* out;
  float* lse;
  int* err;
};

__global__ void __launch_bounds__(kThreads, 2)
    fa_tc_fwd_kernel(const __grid_constant__ CUtensorMap m128, const __grid_constant__ CUtensorMap m64,
                     const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + kRowTile;             // NSF x 8 KB
  const uint32_t sV = sK + NSF * kStrTile;       // NSF x 8 KB
  uint8_t* pP = smem + kRowTile + 2 * NSF * kStrTile;
  const uint32_t sP = smem_u32(pP);              // 2 x 16 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(pP + 2 * kOpTile);
  // q_full | kv_full[NSF] | kv_empty[NSF] | s_full[2] | s_free[2] | p_full[2] | o_done[2] | slot
  const uint32_t b_q = smem_u32(bars);
  auto b_kvf = [&](int s) { return smem_u32(bars + 1 + s); };
  auto b_kve = [&](int s) { return smem_u32(bars + 1 + NSF + s); };
  auto b_sf = [&](int i) { return smem_u32(bars + 1 + 2 * NSF + i); };
  auto b_sfr = [&](int i) { return smem_u32(bars + 3 + 2 * NSF + i); };
  auto b_pf = [&](int i) { return smem_u32(bars + 5 + 2 * NSF + i); };
  auto b_od = [&](int i) { return smem_u32(bars + 7 + 2 * NSF + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9 + 2 * NSF);

  const int qb = gridDim.x - 1 - blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T = p.T, C = p.C;
  const int last_key = min(T, (qb + 1) * BR) - 1;
  const int nkt = last_key / BS + 1;  // 64-key tiles 0 .. nkt-1
  const int row_base = b * T;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < NSF; ++s) {
      mbar_init(b_kvf(s), 1);
      mbar_init(b_kve(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_sf(i), 1);
      mbar_init(b_sfr(i), 128);
      mbar_init(b_pf(i), 128);
      mbar_init(b_od(i), 1);
    }
    init_bar_fence();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;  // S buffers at +0 and +64

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA
    mbar_expect_tx(b_q, kRowTile);
    tma_load_2d(sQ, &m128, b_q, h * D, row_base + qb * BR);
    int issued = 0;
    for (int j = 0; j < nkt; ++j) {
      const int s = j % NSF;
      if (!mbar_wait(b_kve(s), ((j / NSF) & 1) ^ 1, p.err, 11)) break;
      mbar_expect_tx(b_kvf(s), 2 * kStrTile);
      tma_load_2d(sK + s * kStrTile, &m64, b_kvf(s), C + h * D, row_base + j * BS);
      tma_load_2d(sV + s * kStrTile, &m64, b_kvf(s), 2 * C + h * D, row_base + j * BS);
      ++issued;
    }
    mbar_wait(b_q, 0, p.err, 15);
    for (int q = 1; q <= min(issued, NSF); ++q) {
      const int idx = issued - q;
      mbar_wait(b_kvf(idx % NSF), uint32_t((idx / NSF) & 1), p.err, 15);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA
    const uint32_t id_s = idesc_bf16(BR, BS, 0, 0);
    const uint32_t id_o = idesc_bf16(BR, D, 0, 1);
    bool ok = mbar_wait(b_q, 0, p.err, 12);
    int last_pv = -1;
    for (int j = 0; ok && j <= nkt; ++j) {
      if (j < nkt) {
        const int s = j % NSF;
        if (!mbar_wait(b_kvf(s), (j / NSF) & 1, p.err, 12) ||
            !mbar_wait(b_sfr(j & 1), ((j >> 1) & 1) ^ 1, p.err, 12)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          umma_bf16(tS + (j & 1) * BS, desc_kmajor(sQ, k), desc_kmajor(sK + s * kStrTile, k), id_s,
                    k > 0);
        umma_commit(b_sf(j & 1));
      }
      if (j >= 1) {
        const int jj = j - 1, s = jj % NSF;
        if (!mbar_wait(b_pf(jj & 1), (jj >> 1) & 1, p.err, 13)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BS / 16; ++k)
          umma_bf16(tO, desc_kmajor(sP + (jj & 1) * kOpTile, k),
                    desc_mnmajor(sV + s * kStrTile, k), id_o, (jj > 0 || k > 0) ? 1u : 0u);
        umma_commit(b_od(jj & 1));
        umma_commit(b_kve(s));
        last_pv = jj;
      }
    }
    if (last_pv >= 0) mbar_wait(b_od(last_pv & 1), uint32_t((last_pv >> 1) & 1), p.err, 16);
  } else if (warp >= 2) {
    // ------------------------------------------------ softmax warpgroup
    const int e = (warp & 3) * 32 + lane;  // query row in the block = TMEM lane
    const int q = qb * BR + e;
    const uint32_t lo = uint32_t((warp & 3) * 32) << 16;
    const float sl2 = rsqrtf(float(D)) * kLog2e;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkt; ++j) {
      bool w = mbar_wait(b_sf(j & 1), (j >> 1) & 1, p.err, 14);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32_async(tS + lo + (j & 1) * BS, r0);
      tmem_ld32_async(tS + lo + (j & 1) * BS + 32, r1);
      tmem_wait_ld(r0);
      reg_after_wait(r1);
      tc_fence_before();
      mbar_arrive(b_sfr(j & 1));
      const int key0 = j * BS;
      const bool need_mask = key0 + BS - 1 > qb * BR || key0 + BS > T;
      float x[64];  // raw scores; keys past the query or past T become -inf
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        x[i] = __uint_as_float(r0[i]);
        x[32 + i] = __uint_as_float(r1[i]);
      }
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (key0 + i > q || key0 + i >= T) x[i] = -INFINITY;
      }
      // running maximum in log2 units (scale > 0 commutes with max)
      const float mn = fmaxf(m, max64(x) * sl2);
      const bool resc = mn > m + kRescale;  // always on the first tile (m = -inf)
      const float mu = resc ? mn : m;
      const float corr = resc ? ex2(m - mn) : 1.f;
      // p = 2^(x sl2 - mu): one packed FMA per pair, ex2 per element, packed sums
      uint32_t pk[32];
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        float t0, t1;
        fma2(t0, t1, x[i], x[i + 1], sl2, sl2, -mu, -mu);
        const float p0 = ex2(t0), p1 = ex2(t1);
        add2(sa[(i >> 1) & 3], sb[(i >> 1) & 3], p0, p1);
        pk[i >> 1] = pack2(p0, p1);
      }
      const float rs = ((sa[0] + sb[0]) + (sa[1] + sb[1])) + ((sa[2] + sb[2]) + (sa[3] + sb[3]));
      l = l * corr + rs;
      m = mu;
      if (j >= 1 && __any_sync(0xffffffffu, resc)) {
        // O must hold P_{j-1} V_{j-1} before it is rescaled
        w = mbar_wait(b_od((j - 1) & 1), ((j - 1) >> 1) & 1, p.err, 17);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t o0[32], o1[32];
        tmem_ld32_async(tO + lo, o0);
        tmem_ld32_async(tO + lo + 32, o1);
        tmem_wait_ld(o0);
        reg_after_wait(o1);
        float f0[32], f1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          f0[i] = __uint_as_float(o0[i]) * corr;
          f1[i] = __uint_as_float(o1[i]) * corr;
        }
        tmem_st32(tO + lo, f0);
        tmem_st32(tO + lo + 32, f1);
      }
      // P buffer j%2 was last read by P_{j-2} V_{j-2}
      if (j >= 2) {
        w = mbar_wait(b_od(j & 1), ((j - 2) >> 1) & 1, p.err, 18);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
      }
      put_row64(pP + (j & 1) * kOpTile, e, pk);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(b_pf(j & 1));
    }
    if (ok) {
      const int jl = nkt - 1;
      bool w = mbar_wait(b_od(jl & 1), (jl >> 1) & 1, p.err, 19);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        uint32_t o0[32], o1[32];
        tmem_ld32_async(tO + lo, o0);
        tmem_ld32_async(tO + lo + 32, o1);
        tmem_wait_ld(o0);
        reg_after_wait(o1);
        if (q < T) {
          store_row64(p.out + (int64_t(row_base) + q) * C + h * D, o0, o1, 1.f / l);
          p.lse[(int64_t(b) * p.H + h) * T + q] = (m + log2f(l)) / kLog2e;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ====================================================================== backward
constexpr int NSB = 2;  // streamed-tile stages

struct BwdParams {
  int T, C, H;
  const float* lse;
  const float* delta;
  bf16* dqkv;
  int* err;
};

// ---------------------------------------------------------------- dK, dV
// CTA: 128 keys kb*128 ..; 64-query tiles i from the diagonal to the end.
// TMEM: S^T +0, dP^T +64, dV +128, dK +192.
constexpr int kDkdvSmem = 2 * kRowTile + NSB * 2 * kStrTile + 2 * kOpTile + 2 * BS * 4 + 256 + 1024;

__global__ void __launch_bounds__(kThreads, 2)
    fa_tc_dkdv_kernel(const __grid_constant__ CUtensorMap q128, const __grid_constant__ CUtensorMap q64,
                      const __grid_constant__ CUtensorMap o64, const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sK = smem_u32(smem), sV = sK + kRowTile;
  const uint32_t sQ = sV + kRowTile;            // NSB x 8 KB
  const uint32_t sO = sQ + NSB * kStrTile;      // dO, NSB x 8 KB
  uint8_t* pPt = smem + 2 * kRowTile + 2 * NSB * kStrTile;
  uint8_t* pDt = pPt + kOpTile;
  const uint32_t sPt = smem_u32(pPt), sDt = smem_u32(pDt);
  float* sLD = reinterpret_cast<float*>(pDt + kOpTile);  // [64] -lse*log2e, [64] -delta
  uint64_t* bars = reinterpret_cast<uint64_t*>(sLD + 2 * BS);
  // kv_full | qo_full[NSB] | qo_empty[NSB] | s_full | s_free | p_full | mm_done | slot
  const uint32_t b_kv = smem_u32(bars);
  auto b_qf = [&](int s) { return smem_u32(bars + 1 + s); };
  auto b_qe = [&](int s) { return smem_u32(bars + 1 + NSB + s); };
  const uint32_t b_sf = smem_u32(bars + 1 + 2 * NSB);
  const uint32_t b_sfr = smem_u32(bars + 2 + 2 * NSB);
  const uint32_t b_pf = smem_u32(bars + 3 + 2 * NSB);
  const uint32_t b_mm = smem_u32(bars + 4 + 2 * NSB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5 + 2 * NSB);

  const int kb = blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T = p.T, C = p.C;
  const int qt0 = (kb * BR) / BS;
  const int nqt = (T + BS - 1) / BS;
  const int n = nqt - qt0;
  const int row_base = b * T;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(b_kv, 1);
    for (int s = 0; s < NSB; ++s) {
      mbar_init(b_qf(s), 1);
      mbar_init(b_qe(s), 1);
    }
    mbar_init(b_sf, 1);
    mbar_init(b_sfr, 128);
    mbar_init(b_pf, 128);
    mbar_init(b_mm, 1);
    init_bar_fence();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 64, tV = tmem + 128, tKd = tmem + 192;

  if (warp == 0 && lane == 0) {
    mbar_expect_tx(b_kv, 2 * kRowTile);
    tma_load_2d(sK, &q128, b_kv, C + h * D, row_base + kb * BR);
    tma_load_2d(sV, &q128, b_kv, 2 * C + h * D, row_base + kb * BR);
    int issued = 0;
    for (int i = 0; i < n; ++i) {
      const int s = i % NSB;
      if (!mbar_wait(b_qe(s), ((i / NSB) & 1) ^ 1, p.err, 21)) break;
      mbar_expect_tx(b_qf(s), 2 * kStrTile);
      const int row = row_base + (qt0 + i) * BS;
      tma_load_2d(sQ + s * kStrTile, &q64, b_qf(s), h * D, row);
      tma_load_2d(sO + s * kStrTile, &o64, b_qf(s), h * D, row);
      ++issued;
    }
    mbar_wait(b_kv, 0, p.err, 25);
    for (int q = 1; q <= min(issued, NSB); ++q) {
      const int idx = issued - q;
      mbar_wait(b_qf(idx % NSB), uint32_t((idx / NSB) & 1), p.err, 25);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t id_s = idesc_bf16(BR, BS, 0, 0);
    const uint32_t id_o = idesc_bf16(BR, D, 0, 1);
    bool ok = mbar_wait(b_kv, 0, p.err, 22);
    int mm = 0;
    for (int i = 0; ok && i <= n; ++i) {
      if (i < n) {
        const int s = i % NSB;
        if (!mbar_wait(b_qf(s), (i / NSB) & 1, p.err, 22) ||
            !mbar_wait(b_sfr, (i & 1) ^ 1, p.err, 22)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          umma_bf16(tS, desc_kmajor(sK, k), desc_kmajor(sQ + s * kStrTile, k), id_s, k > 0);
          umma_bf16(tP, desc_kmajor(sV, k), desc_kmajor(sO + s * kStrTile, k), id_s, k > 0);
        }
        umma_commit(b_sf);
      }
      if (i >= 1) {
        const int ii = i - 1, s = ii % NSB;
        if (!mbar_wait(b_pf, ii & 1, p.err, 23)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BS / 16; ++k) {
          const uint32_t acc = (ii > 0 || k > 0) ? 1u : 0u;
          umma_bf16(tV, desc_kmajor(sPt, k), desc_mnmajor(sO + s * kStrTile, k), id_o, acc);
          umma_bf16(tKd, desc_kmajor(sDt, k), desc_mnmajor(sQ + s * kStrTile, k), id_o, acc);
        }
        umma_commit(b_mm);
        umma_commit(b_qe(s));
        ++mm;
      }
    }
    if (mm > 0) mbar_wait(b_mm, uint32_t((mm - 1) & 1), p.err, 26);
  } else if (warp >= 2) {
    const int e = (warp & 3) * 32 + lane;  // key row in the block = TMEM lane
    const int key = kb * BR + e;
    const uint32_t lo = uint32_t((warp & 3) * 32) << 16;
    const float scale = rsqrtf(float(D));
    const float sl2 = scale * kLog2e;
    bool ok = true;
    // lse and delta of the 64 queries of a tile, fetched one tile ahead so the
    // global loads overlap the current tile's work (threads e < 64); negated,
    // so that each pair of queries costs one packed FMA / add
    const int64_t bh = (int64_t(b) * p.H + h) * T;
    float nl_next = 0.f, nd_next = 0.f;
    auto fetch = [&](int i) {
      const int q = (qt0 + i) * BS + e;
      nl_next = q < T ? -p.lse[bh + q] * kLog2e : 0.f;
      nd_next = q < T ? -p.delta[bh + q] : 0.f;
    };
    if (e < BS && n > 0) fetch(0);
    for (int i = 0; i < n; ++i) {
      const int q0 = (qt0 + i) * BS;
      if (e < BS) {
        sLD[e] = nl_next;
        sLD[BS + e] = nd_next;
        if (i + 1 < n) fetch(i + 1);
      }
      // an expired wait (error word set) skips later waits but keeps the
      // warpgroup's named barriers in step, so no warp is left at one
      if (ok) {
        bool w = mbar_wait(b_sf, i & 1, p.err, 24);
        if (i >= 1) w = w && mbar_wait(b_mm, (i - 1) & 1, p.err, 24);  // P^T / dS^T free
        ok = w;
      }
      tc_fence_after();
      wg_bar();  // sLD of this tile visible
      const bool need_mask = q0 < kb * BR + BR || q0 + BS > T;
      // two halves of 32 queries, so that only one half of S^T and dP^T is
      // held in registers at a time; every 8 queries give one 16-byte chunk
      // of the P^T and dS^T rows, written at once
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t sx[32], dx[32];
        tmem_ld32_async(tS + lo + 32 * hh, sx);
        tmem_ld32_async(tP + lo + 32 * hh, dx);
        tmem_wait_ld(sx);
        reg_after_wait(dx);
        if (hh == 1) {  // S^T and dP^T read: the MMA may overwrite them
          tc_fence_before();
          mbar_arrive(b_sfr);
        }
#pragma unroll
        for (int c8 = 0; c8 < 32; c8 += 8) {
          uint32_t pp[4], pd[4];
#pragma unroll
          for (int c = c8; c < c8 + 8; c += 2) {
            const int qc = 32 * hh + c;  // query column within the tile
            const float2 nl = *reinterpret_cast<const float2*>(sLD + qc);       // -lse log2 e
            const float2 nd = *reinterpret_cast<const float2*>(sLD + BS + qc);  // -delta
            float t0, t1;
            fma2(t0, t1, __uint_as_float(sx[c]), __uint_as_float(sx[c + 1]), sl2, sl2, nl.x,
                 nl.y);
            float p0 = ex2(t0), p1 = ex2(t1);
            if (need_mask) {
              if (q0 + qc < key || q0 + qc >= T) p0 = 0.f;
              if (q0 + qc + 1 < key || q0 + qc + 1 >= T) p1 = 0.f;
            }
            float g0 = __uint_as_float(dx[c]), g1 = __uint_as_float(dx[c + 1]);
            add2(g0, g1, nd.x, nd.y);  // dP - delta
            mul2(g0, g1, p0, p1);      // dS = P (dP - delta)
            pp[(c - c8) >> 1] = pack2(p0, p1);
            pd[(c - c8) >> 1] = pack2(g0, g1);
          }
          const int ch = (32 * hh + c8) >> 3;  // 16-byte chunk of the 128-byte row
          const int off = e * 128 + ((ch ^ (e & 7)) << 4);
          *reinterpret_cast<uint4*>(pPt + off) = make_uint4(pp[0], pp[1], pp[2], pp[3]);
          *reinterpret_cast<uint4*>(pDt + off) = make_uint4(pd[0], pd[1], pd[2], pd[3]);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(b_pf);
      wg_bar();  // sLD may be rewritten for the next tile
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && n > 0) {
      bool w = mbar_wait(b_mm, (n - 1) & 1, p.err, 27);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        bf16* drow = p.dqkv + (int64_t(row_base) + key) * 3 * C + h * D;
        // dV then dK, one 64-column row each
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) {
          uint32_t a0[32], a1[32];
          tmem_ld32_async((w2 ? tKd : tV) + lo, a0);
          tmem_ld32_async((w2 ? tKd : tV) + lo + 32, a1);
          tmem_wait_ld(a0);
          reg_after_wait(a1);
          if (key < T) store_row64(drow + (w2 ? C : 2 * C), a0, a1, w2 ? scale : 1.f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- dQ
// CTA: 128 queries qb*128 ..; 64-key tiles j up to the diagonal.
// TMEM: S +0, dP +64, dQ +128.
constexpr int kDqSmem = 2 * kRowTile + NSB * 2 * kStrTile + kOpTile + 256 + 1024;

__global__ void __launch_bounds__(kThreads, 2)
    fa_tc_dq_kernel(const __grid_constant__ CUtensorMap q128, const __grid_constant__ CUtensorMap q64,
                    const __grid_constant__ CUtensorMap o128, const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sQ = smem_u32(smem), sO = sQ + kRowTile;
  const uint32_t sK = sO + kRowTile;            // NSB x 8 KB
  const uint32_t sV = sK + NSB * kStrTile;      // NSB x 8 KB
  uint8_t* pDs = smem + 2 * kRowTile + 2 * NSB * kStrTile;
  const uint32_t sDs = smem_u32(pDs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(pDs + kOpTile);
  const uint32_t b_q = smem_u32(bars);
  auto b_kf = [&](int s) { return smem_u32(bars + 1 + s); };
  auto b_ke = [&](int s) { return smem_u32(bars + 1 + NSB + s); };
  const uint32_t b_sf = smem_u32(bars + 1 + 2 * NSB);
  const uint32_t b_sfr = smem_u32(bars + 2 + 2 * NSB);
  const uint32_t b_df = smem_u32(bars + 3 + 2 * NSB);
  const uint32_t b_mm = smem_u32(bars + 4 + 2 * NSB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5 + 2 * NSB);

  const int qb = gridDim.x - 1 - blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T = p.T, C = p.C;
  const int last_key = min(T, (qb + 1) * BR) - 1;
  const int nkt = last_key / BS + 1;
  const int row_base = b * T;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < NSB; ++s) {
      mbar_init(b_kf(s), 1);
      mbar_init(b_ke(s), 1);
    }
    mbar_init(b_sf, 1);
    mbar_init(b_sfr, 128);
    mbar_init(b_df, 128);
    mbar_init(b_mm, 1);
    init_bar_fence();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 64, tQd = tmem + 128;

  if (warp == 0 && lane == 0) {
    mbar_expect_tx(b_q, 2 * kRowTile);
    tma_load_2d(sQ, &q128, b_q, h * D, row_base + qb * BR);
    tma_load_2d(sO, &o128, b_q, h * D, row_base + qb * BR);
    int issued = 0;
    for (int j = 0; j < nkt; ++j) {
      const int s = j % NSB;
      if (!mbar_wait(b_ke(s), ((j / NSB) & 1) ^ 1, p.err, 31)) break;
      mbar_expect_tx(b_kf(s), 2 * kStrTile);
      tma_load_2d(sK + s * kStrTile, &q64, b_kf(s), C + h * D, row_base + j * BS);
      tma_load_2d(sV + s * kStrTile, &q64, b_kf(s), 2 * C + h * D, row_base + j * BS);
      ++issued;
    }
    mbar_wait(b_q, 0, p.err, 35);
    for (int q = 1; q <= min(issued, NSB); ++q) {
      const int idx = issued - q;
      mbar_wait(b_kf(idx % NSB), uint32_t((idx / NSB) & 1), p.err, 35);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t id_s = idesc_bf16(BR, BS, 0, 0);
    const uint32_t id_o = idesc_bf16(BR, D, 0, 1);
    bool ok = mbar_wait(b_q, 0, p.err, 32);
    int mm = 0;
    for (int j = 0; ok && j <= nkt; ++j) {
      if (j < nkt) {
        const int s = j % NSB;
        if (!mbar_wait(b_kf(s), (j / NSB) & 1, p.err, 32) ||
            !mbar_wait(b_sfr, (j & 1) ^ 1, p.err, 32)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          umma_bf16(tS, desc_kmajor(sQ, k), desc_kmajor(sK + s * kStrTile, k), id_s, k > 0);
          umma_bf16(tP, desc_kmajor(sO, k), desc_kmajor(sV + s * kStrTile, k), id_s, k > 0);
        }
        umma_commit(b_sf);
      }
      if (j >= 1) {
        const int jj = j - 1, s = jj % NSB;
        if (!mbar_wait(b_df, jj & 1, p.err, 33)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BS / 16; ++k)
          umma_bf16(tQd, desc_kmajor(sDs, k), desc_mnmajor(sK + s * kStrTile, k), id_o,
                    (jj > 0 || k > 0) ? 1u : 0u);
        umma_commit(b_mm);
        umma_commit(b_ke(s));
        ++mm;
      }
    }
    if (mm > 0) mbar_wait(b_mm, uint32_t((mm - 1) & 1), p.err, 36);
  } else if (warp >= 2) {
    const int e = (warp & 3) * 32 + lane;  // query row in the block = TMEM lane
    const int q = qb * BR + e;
    const uint32_t lo = uint32_t((warp & 3) * 32) << 16;
    const float scale = rsqrtf(float(D));
    const float sl2 = scale * kLog2e;
    const float L2 = q < T ? p.lse[(int64_t(b) * p.H + h) * T + q] * kLog2e : 0.f;
    const float Dl = q < T ? p.delta[(int64_t(b) * p.H + h) * T + q] : 0.f;
    bool ok = true;
    for (int j = 0; j < nkt; ++j) {
      bool w = mbar_wait(b_sf, j & 1, p.err, 34);
      if (j >= 1) w = w && mbar_wait(b_mm, (j - 1) & 1, p.err, 34);  // dS buffer free
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s0[32], s1[32], d0[32], d1[32];
      tmem_ld32_async(tS + lo, s0);
      tmem_ld32_async(tS + lo + 32, s1);
      tmem_ld32_async(tP + lo, d0);
      tmem_ld32_async(tP + lo + 32, d1);
      tmem_wait_ld(s0);
      reg_after_wait(s1);
      reg_after_wait(d0);
      reg_after_wait(d1);
      tc_fence_before();
      mbar_arrive(b_sfr);
      const int key0 = j * BS;
      const bool need_mask = key0 + BS - 1 > qb * BR || key0 + BS > T || qb * BR + BR > T;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float sa = __uint_as_float(c < 32 ? s0[c] : s1[c - 32]);
        const float sb = __uint_as_float(c < 32 ? s0[c + 1] : s1[c - 31]);
        float g0 = __uint_as_float(c < 32 ? d0[c] : d1[c - 32]);
        float g1 = __uint_as_float(c < 32 ? d0[c + 1] : d1[c - 31]);
        float t0, t1;
        fma2(t0, t1, sa, sb, sl2, sl2, -L2, -L2);
        float p0 = ex2(t0), p1 = ex2(t1);
        if (need_mask) {
          if (key0 + c > q || key0 + c >= T || q >= T) p0 = 0.f;
          if (key0 + c + 1 > q || key0 + c + 1 >= T || q >= T) p1 = 0.f;
        }
        add2(g0, g1, -Dl, -Dl);  // dP - delta
        mul2(g0, g1, p0, p1);    // dS = P (dP - delta)
        pk[c >> 1] = pack2(g0, g1);
      }
      put_row64(pDs, e, pk);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      mbar_arrive(b_df);
    }
    if (ok) {
      bool w = mbar_wait(b_mm, (nkt - 1) & 1, p.err, 37);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        uint32_t a0[32], a1[32];
        tmem_ld32_async(tQd + lo, a0);
        tmem_ld32_async(tQd + lo + 32, a1);
        tmem_wait_ld(a0);
        reg_after_wait(a1);
        if (q < T) store_row64(p.dqkv + (int64_t(row_base) + q) * 3 * C + h * D, a0, a1, scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool attn_tc_supported(int B, int T, int C, int H) {
  return C / H == D && C % H == 0 && C % 8 == 0 && int64_t(B) * T < (int64_t(1) << 31);
}

int launch_attn_tc_fwd(const bf16* qkv, int B, int T, int C, int H, bf16* out, float* lse,
                       cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(fa_tc_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFwdSmem);
    attr = true;
  }
  CUtensorMap m128, m64;
  const int64_t rows = int64_t(B) * T;
  if (!make_map_bf16(&m128, qkv, 3 * int64_t(C), rows, 3 * int64_t(C), BR) ||
      !make_map_bf16(&m64, qkv, 3 * int64_t(C), rows, 3 * int64_t(C), BS)) {
    gpt2_internal::set_error("attention: tensor map encoding failed");
    return GPT2_ERR_CUDA;
  }
  FwdParams p{T, C, H, out, lse, device_error_word()};
  dim3 grid(cdiv(T, BR), H, B);
  fa_tc_fwd_kernel<<<grid, kThreads, kFwdSmem, st>>>(m128, m64, p);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_attn_tc_bwd(const bf16* dout, const bf16* qkv, const float* lse, const float* delta,
                       int B, int T, int C, int H, bf16* dqkv, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(fa_tc_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDkdvSmem);
    cudaFuncSetAttribute(fa_tc_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem);
    attr = true;
  }
  CUtensorMap q128, q64, o128, o64;
  const int64_t rows = int64_t(B) * T;
  if (!make_map_bf16(&q128, qkv, 3 * int64_t(C), rows, 3 * int64_t(C), BR) ||
      !make_map_bf16(&q64, qkv, 3 * int64_t(C), rows, 3 * int64_t(C), BS) ||
      !make_map_bf16(&o128, dout, int64_t(C), rows, int64_t(C), BR) ||
      !make_map_bf16(&o64, dout, int64_t(C), rows, int64_t(C), BS)) {
    gpt2_internal::set_error("attention: tensor map encoding failed");
    return GPT2_ERR_CUDA;
  }
  BwdParams p{T, C, H, lse, delta, dqkv, device_error_word()};
  dim3 grid(cdiv(T, BR), H, B);
  fa_tc_dkdv_kernel<<<grid, kThreads, kDkdvSmem, st>>>(q128, q64, o64, p);
  COUNT_LAUNCH(1);
  fa_tc_dq_kernel<<<grid, kThreads, kDqSmem, st>>>(q128, q64, o128, p);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
