// Causal flash attention on the 5th-generation tensor cores (tcgen05 MMAs with
// TMEM accumulators, operands loaded by TMA), head size 64, bf16 in / fp32
// accumulate [ZERO: Attention, OpFlashAttention recomputes the scores in the
// backward; LECTURE: flash attention, causal mask].  The [T, T] scores and
// probabilities never leave TMEM and registers; the backward may keep the
// causal half of the score gradients (bf16) for its dQ step.
//
// Every kernel: CTAs of 192 threads working on blocks of 128 rows (queries, or
// keys in dK/dV) = the 128 TMEM lanes, streaming 64-row tiles of the other
// operand (the forward's CTAs are persistent and take several blocks in turn,
// the backward's take one each):
//   warp 0, one lane   TMA loads (128-row tile once, 64-row tiles in a ring);
//   warp 1             owns the TMEM allocation (256 columns); one lane issues
//                      the tcgen05.mma instructions and commits;
//   warps 2-5          elementwise warpgroup, thread = row (TMEM lane
//                      32 * (warp % 4) + lane): reads a score tile from TMEM
//                      and writes the probabilities / score gradients back
//                      as bf16 over the first 32 columns of that tile, where
//                      the next MMA takes them as its A operand (kind::f16
//                      with A in TMEM), so they never pass through shared
//                      memory (except the kept score gradients, below).
// 256 TMEM columns and < 100 KB of shared memory let two CTAs share an SM, so
// one CTA's elementwise work overlaps the other's MMAs; the shared memory is
// a deep ring of streamed K/V (or Q/dO) tiles that hides load latency.
//
// Forward (per 128 queries, 64-key tiles j <= diagonal):
//   S_j = Q K_j^T (TMEM, double buffered); m, l kept in the log2 domain; the
//   O accumulator (TMEM) is rescaled only when a row maximum grows by more than
//   2^8 (probabilities are taken relative to the kept maximum, so they stay
//   <= 256); P_j (bf16) is written back over its own score buffer in TMEM
//   and O += P_j V_j reads it from there (A operand in TMEM, V MN-major).
//   Q and O are double-buffered across a CTA's blocks; the normalised output
//   tile goes through the block's Q buffer to one TMA store.
// Backward, with Delta_i = dO_i . O_i and P = exp(S / sqrt(D) - lse):
//   dK/dV kernel (per 128 keys, 64-query tiles i >= keys): S^T, dP^T = V dO^T,
//   dS^T = P^T (dP^T - Delta); dV += P^T dO, dK += dS^T Q / sqrt(D);
//   dQ kernel (per 128 queries, 64-key tiles): S, dP, dS; dQ += dS K / sqrt(D).
//   With a score-gradient buffer the dK/dV kernel also writes dS^T (bf16, the
//   values its dK MMA takes) and dQ is one contraction over it (no
//   exponentials, no second S or dP); without one (the no-allocation entry
//   point) the dQ kernel recomputes P and dS as above.  Both backward kernels
//   may also leave per-block column sums of dq, dk, dv (the qkv bias gradient).
// CTAs take the longest causal row blocks first (work_item; the persistent
// forward: one block per round of grid-size blocks, alternate rounds reversed).
// Every output element is written by one CTA, no atomics (deterministic).
// Every wait is bounded (2 s of global time) and reports a timeout in the
// error word instead of hanging.

#include "attn_internal.h"
#include "tc_common.cuh"

using namespace tc;

namespace {

constexpr int D = 64;
constexpr int BR = 128;                 // rows per CTA = TMEM lanes
constexpr int BS = 64;                  // rows of a streamed tile
constexpr int kRowTile = BR * D * 2;    // 16 KB: 128 x 64 bf16
constexpr int kStrTile = BS * D * 2;    // 8 KB: 64 x 64 bf16
constexpr int kTmemCols = 256;
constexpr int kThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;         // lazy-rescale threshold, log2 units

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x for a pair on the FMA pipe: x = n + f with n the nearest integer (from
// the 1.5 * 2^23 shift) and f in [-1/2, 1/2]; 2^f from a cubic fitted here to
// 2^f on that interval (equal-ripple relative error, at most 7.5e-5, below the
// bf16 rounding of the probabilities); 2^n added to the exponent field (the
// shift's own bits drop out of bits(t) << 23).  Arguments below -126 give ~0.
__device__ __forceinline__ void ex2_poly2(float x0, float x1, float& y0, float& y1) {
  constexpr float kShift = 12582912.f;  // 1.5 * 2^23
  constexpr float c0 = 0.99992806f, c1 = 0.69326097f, c2 = 0.24261113f, c3 = 0.05517167f;
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  float t0 = x0, t1 = x1;
  add2(t0, t1, kShift, kShift);  // n in the low mantissa bits of t
  float n0 = t0, n1 = t1;
  add2(n0, n1, -kShift, -kShift);
  float f0, f1, p0, p1;
  fma2(f0, f1, n0, n1, -1.f, -1.f, x0, x1);  // f = x - n (exact)
  fma2(p0, p1, f0, f1, c3, c3, c2, c2);
  fma2(p0, p1, p0, p1, f0, f1, c1, c1);
  fma2(p0, p1, p0, p1, f0, f1, c0, c0);
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
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
// This CTA's (row block step, head, batch), longest work first.  CTAs start in
// linear block order (x fastest); block step s of every (batch, head) pair is
// issued before step s + 1 of any, so the longest blocks start first and the
// shortest fill the tail of the last wave (greedy list scheduling, longest
// first).  Grid (n_blocks, H, B).  With G < B * H the order is longest first
// within consecutive groups of G (batch, head) pairs.
struct WorkItem {
  int step, h, b;
};
__device__ __forceinline__ WorkItem work_item(int G = 1 << 30) {
  const int BH = gridDim.y * gridDim.z, nblk = gridDim.x;
  const int i = blockIdx.x + nblk * (blockIdx.y + gridDim.y * blockIdx.z);
  G = min(G, BH);
  const int chunk = i / (G * nblk), j = i % (G * nblk);
  const int Gc = min(G, BH - chunk * G);
  const int bh = chunk * G + j % Gc;
  return WorkItem{j / Gc, bh % int(gridDim.y), bh / int(gridDim.y)};
}

// L2 policies for the kept score gradients: written to stay (evict_last),
// read once (evict_first)
__device__ __forceinline__ uint64_t l2_keep() {
  uint64_t q;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(q));
  return q;
}
__device__ __forceinline__ uint64_t l2_once() {
  uint64_t q;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(q));
  return q;
}
__device__ __forceinline__ void tma_store_2d_l2(const CUtensorMap* map, uint32_t src, int c0,
                                                int c1, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_l2(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                               int c0, int c1, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(pol)
      : "memory");
}

// One 64-deep contraction as four K = 16 MMAs, the accumulate flag an
// immediate: the first MMA overwrites D unless acc; descriptors advance by
// a_k / b_k per slice (+2 K-major, +128 MN-major).  A from shared memory (ss)
// or from TMEM (ts: 8 columns of packed bf16 per slice).
__device__ __forceinline__ void mma_ss4(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                        uint64_t a_k, uint64_t b_k, bool acc) {
  if (acc)
    umma_i<1>(d, a, b, id);
  else
    umma_i<0>(d, a, b, id);
#pragma unroll
  for (int k = 1; k < 4; ++k) umma_i<1>(d, a + k * a_k, b + k * b_k, id);
}
__device__ __forceinline__ void mma_ts4(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id,
                                        uint64_t b_k, bool acc) {
  if (acc)
    umma_ts_i<1>(d, a_tmem, b, id);
  else
    umma_ts_i<0>(d, a_tmem, b, id);
#pragma unroll
  for (int k = 1; k < 4; ++k) umma_ts_i<1>(d, a_tmem + 8 * k, b + k * b_k, id);
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
// Persistent: two CTAs per SM walk the (query block, head, batch) items,
// listed longest first, one per round of grid-size items, every other round
// in reverse CTA order (long and short items pair up).  Q and the O
// accumulator are double-buffered per item (shared memory, TMEM) and every
// barrier's phase follows a tile counter that runs across items, so the next
// item's Q / K / V loads and first S MMAs overlap the current item's last
// tiles and its output store.
constexpr int NSF = 4;  // K/V stages (5 measured 0.7% slower)
constexpr int kFwdSmem = 2 * kRowTile + NSF * 2 * kStrTile + 256 + 1024;

struct FwdParams {
  int T, C, H;
  int nblk, n_items;  // query blocks per (batch, head); items = nblk * H * B
  bf16* out;
  float* lse;
  int* err;
};
// item i: query block nblk - 1 - i / (B H) (longest first), then (batch, head)
struct FwdItem {
  int qb, h, b;
};
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int i, int BH) {
  const int bh = i % BH;
  return FwdItem{p.nblk - 1 - i / BH, bh % p.H, bh / p.H};
}

__global__ void __launch_bounds__(kThreads, 2)
    fa_tc_fwd_kernel(const __grid_constant__ CUtensorMap m128, const __grid_constant__ CUtensorMap m64,
                     const __grid_constant__ CUtensorMap mo, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sQ0 = smem_u32(smem);            // 2 x 16 KB
  const uint32_t sK = sQ0 + 2 * kRowTile;         // NSF x 8 KB
  const uint32_t sV = sK + NSF * kStrTile;        // NSF x 8 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kRowTile + 2 * NSF * kStrTile);
  // q_full[2] | q_empty[2] | kv_full[NSF] | kv_empty[NSF] | s_full[2] | s_free[2] | p_full[2] |
  // o_done[2] | o_empty[2] | o_staged[2] | slot
  auto b_q = [&](int i) { return smem_u32(bars + i); };
  auto b_qe = [&](int i) { return smem_u32(bars + 2 + i); };
  auto b_kvf = [&](int s) { return smem_u32(bars + 4 + s); };
  auto b_kve = [&](int s) { return smem_u32(bars + 4 + NSF + s); };
  auto b_sf = [&](int i) { return smem_u32(bars + 4 + 2 * NSF + i); };
  auto b_sfr = [&](int i) { return smem_u32(bars + 6 + 2 * NSF + i); };
  auto b_pf = [&](int i) { return smem_u32(bars + 8 + 2 * NSF + i); };
  auto b_od = [&](int i) { return smem_u32(bars + 10 + 2 * NSF + i); };
  auto b_oe = [&](int i) { return smem_u32(bars + 12 + 2 * NSF + i); };
  auto b_ost = [&](int i) { return smem_u32(bars + 14 + 2 * NSF + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16 + 2 * NSF);

  const int T = p.T, C = p.C, BH = p.H * (p.n_items / (p.nblk * p.H));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // 64-key tiles of an item: keys 0 .. min(T, (qb + 1) BR) - 1
  auto n_tiles = [&](int qb) { return (min(T, (qb + 1) * BR) - 1) / BS + 1; };
  // whole query blocks leave their output tile in their Q buffer for one TMA
  // store (a block that runs past T is stored row by row: a 2-D box would
  // reach into the next sequence)
  auto whole = [&](int qb) { return (qb + 1) * BR <= T; };
  // this CTA's k-th item: one per round of gridDim.x items, the rounds taken
  // in alternating directions so that long and short items pair up
  auto item_of = [&](int k) {
    const int G = int(gridDim.x), c = int(blockIdx.x);
    return k * G + ((k & 1) ? G - 1 - c : c);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_q(i), 1);
      mbar_init(b_qe(i), 1);
      mbar_init(b_sf(i), 1);
      mbar_init(b_sfr(i), 128);
      mbar_init(b_pf(i), 128);
      mbar_init(b_od(i), 1);
      mbar_init(b_oe(i), 128);
      mbar_init(b_ost(i), 128);
    }
    for (int s = 0; s < NSF; ++s) {
      mbar_init(b_kvf(s), 1);
      mbar_init(b_kve(s), 1);
    }
    init_bar_fence();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;  // S buffers at +0 and +64; O buffers at +128 and +192

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA
    // item kk's output tile, staged by the softmax warpgroup in its Q buffer
    auto store_out = [&](int kk) -> bool {
      if (!mbar_wait(b_ost(kk & 1), uint32_t((kk >> 1) & 1), p.err, 18)) return false;
      const FwdItem w = fwd_item(p, item_of(kk), BH);
      if (whole(w.qb)) {
        tma_store_2d(&mo, sQ0 + (kk & 1) * kRowTile, w.h * D, w.b * T + w.qb * BR);
        bulk_commit();
      }
      return true;
    };
    int g = 0, issued_q = 0, k = 0;
    bool ok = true;
    for (; ok && item_of(k) < p.n_items; ++k) {
      const FwdItem w = fwd_item(p, item_of(k), BH);
      const int row_base = w.b * T, nkt = n_tiles(w.qb), qbuf = k & 1;
      // Q_k goes into the buffer item k - 2 used, once its last S MMA is done
      // and the output tile staged there has been read by its store
      if (!mbar_wait(b_qe(qbuf), ((k >> 1) & 1) ^ 1, p.err, 11)) break;
      if (k >= 2) {
        if (!store_out(k - 2)) break;
        bulk_wait_read<0>();
      }
      mbar_expect_tx(b_q(qbuf), kRowTile);
      tma_load_2d(sQ0 + qbuf * kRowTile, &m128, b_q(qbuf), w.h * D, row_base + w.qb * BR);
      ++issued_q;
      for (int j = 0; j < nkt; ++j, ++g) {
        const int s = g % NSF;
        if (!mbar_wait(b_kve(s), ((g / NSF) & 1) ^ 1, p.err, 11)) {
          ok = false;
          break;
        }
        mbar_expect_tx(b_kvf(s), 2 * kStrTile);
        tma_load_2d(sK + s * kStrTile, &m64, b_kvf(s), C + w.h * D, row_base + j * BS);
        tma_load_2d(sV + s * kStrTile, &m64, b_kvf(s), 2 * C + w.h * D, row_base + j * BS);
      }
    }
    // the last two items' outputs; every issued copy has landed (loads) or
    // completed (stores) before the CTA may exit
    if (ok)
      for (int kk = max(0, k - 2); kk < k; ++kk)
        if (!store_out(kk)) break;
    bulk_wait_all();
    for (int q = max(0, issued_q - 2); q < issued_q; ++q)
      mbar_wait(b_q(q & 1), uint32_t((q >> 1) & 1), p.err, 15);
    for (int q = max(0, g - NSF); q < g; ++q)
      mbar_wait(b_kvf(q % NSF), uint32_t((q / NSF) & 1), p.err, 15);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA
    // per tile: S_g = Q K_g^T; then O += P_{g-1} V_{g-1} of the previous tile
    // (possibly of the previous item), so the next S is queued before it
    const uint32_t id_s = idesc_bf16(BR, BS, 0, 0);
    const uint32_t id_o = idesc_bf16(BR, D, 0, 1);
    const uint64_t dK = desc_kmajor(sK, 0), dVm = desc_mnmajor(sV, 0);
    struct Pending {
      int g, k, j;  // tile counter, item number, tile within the item
    } pv{-1, 0, 0};
    bool ok = true;
    auto issue_pv = [&](const Pending& t) -> bool {
      if (!mbar_wait(b_pf(t.g & 1), (t.g >> 1) & 1, p.err, 13)) return false;
      // the first P V of item k overwrites O buffer k & 1: item k - 2's output read
      if (t.j == 0 && !mbar_wait(b_oe(t.k & 1), ((t.k >> 1) & 1) ^ 1, p.err, 13)) return false;
      tc_fence_after();
      // P sits in the first 32 columns of its score buffer (two bf16 per
      // column); S_{g+2} reuses that buffer only after this MMA (issue order)
      mma_ts4(tmem + 128 + 64 * (t.k & 1), tS + (t.g & 1) * BS,
              desc_offset(dVm, (t.g % NSF) * kStrTile), id_o, 128, t.j > 0);
      umma_commit(b_od(t.g & 1));
      umma_commit(b_kve(t.g % NSF));
      return true;
    };
    int g = 0;
    for (int k = 0; ok && item_of(k) < p.n_items; ++k) {
      const FwdItem w = fwd_item(p, item_of(k), BH);
      const int nkt = n_tiles(w.qb), qbuf = k & 1;
      if (!mbar_wait(b_q(qbuf), (k >> 1) & 1, p.err, 12)) break;
      const uint64_t dQ = desc_kmajor(sQ0 + qbuf * kRowTile, 0);
      for (int j = 0; j < nkt; ++j, ++g) {
        const int s = g % NSF;
        if (!mbar_wait(b_kvf(s), (g / NSF) & 1, p.err, 12) ||
            !mbar_wait(b_sfr(g & 1), ((g >> 1) & 1) ^ 1, p.err, 12)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_ss4(tS + (g & 1) * BS, dQ, desc_offset(dK, s * kStrTile), id_s, 2, 2, false);
        umma_commit(b_sf(g & 1));
        if (j == nkt - 1) umma_commit(b_qe(qbuf));  // Q_k read by its last S MMA
        if (pv.g >= 0 && !issue_pv(pv)) {
          ok = false;
          break;
        }
        pv = Pending{g, k, j};
      }
    }
    if (ok && pv.g >= 0) ok = issue_pv(pv);
    // all issued MMAs complete before TMEM is released
    if (pv.g >= 0) mbar_wait(b_od(pv.g & 1), uint32_t((pv.g >> 1) & 1), p.err, 16);
  } else if (warp >= 2) {
    // ------------------------------------------------ softmax warpgroup
    const int e = (warp & 3) * 32 + lane;  // query row in the block = TMEM lane
    const uint32_t lo = uint32_t((warp & 3) * 32) << 16;
    const float sl2 = rsqrtf(float(D)) * kLog2e;
    bool ok = true;
    int g = 0;
    for (int k = 0; ok && item_of(k) < p.n_items; ++k) {
      const FwdItem w = fwd_item(p, item_of(k), BH);
      const int nkt = n_tiles(w.qb), row_base = w.b * T;
      const int q = w.qb * BR + e;
      const uint32_t tO = tmem + 128 + 64 * (k & 1);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nkt; ++j, ++g) {
        bool wt = mbar_wait(b_sf(g & 1), (g >> 1) & 1, p.err, 14);
        if (!__all_sync(0xffffffffu, wt)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32_async(tS + lo + (g & 1) * BS, r0);
        tmem_ld32_async(tS + lo + (g & 1) * BS + 32, r1);
        tmem_wait_ld(r0);
        reg_after_wait(r1);
        tc_fence_before();
        mbar_arrive(b_sfr(g & 1));
        const int key0 = j * BS;
        const bool need_mask = key0 + BS - 1 > w.qb * BR || key0 + BS > T;
        float x[64];  // raw scores; keys past the query or past T become -inf
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = __uint_as_float(r0[i]);
          x[32 + i] = __uint_as_float(r1[i]);
        }
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 64; ++i) x[i] = (key0 + i > q || key0 + i >= T) ? -INFINITY : x[i];
        }
        // running maximum in log2 units (scale > 0 commutes with max)
        const float mn = fmaxf(m, max64(x) * sl2);
        const bool resc = mn > m + kRescale;  // always on the first tile (m = -inf)
        const float mu = resc ? mn : m;
        const float corr = resc ? ex2(m - mn) : 1.f;
        // p = 2^(x sl2 - mu): one packed FMA per pair, ex2 per element, packed sums
        uint32_t pk[32];
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        // branch-free (so the pairs interleave); masked scores are -inf and
        // ex2.approx(-inf) is exactly 0
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
          // O must hold P_{g-1} V_{g-1} before it is rescaled
          wt = mbar_wait(b_od((g - 1) & 1), ((g - 1) >> 1) & 1, p.err, 17);
          if (!__all_sync(0xffffffffu, wt)) {
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
        // P_g (bf16) over the first 32 columns of S_g's buffer, the A operand of P_g V_g
        tmem_st32_async(tS + lo + (g & 1) * BS, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_pf(g & 1));
      }
      if (!ok) break;
      const int jl = g - 1;  // the item's last tile
      bool wt = mbar_wait(b_od(jl & 1), (jl >> 1) & 1, p.err, 19);
      if (!__all_sync(0xffffffffu, wt)) break;
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld32_async(tO + lo, o0);
      tmem_ld32_async(tO + lo + 32, o1);
      tmem_wait_ld(o0);
      reg_after_wait(o1);
      tc_fence_before();
      mbar_arrive(b_oe(k & 1));  // the O buffer may take item k + 2
      const float il = 1.f / l;
      if (whole(w.qb)) {
        // row e of the output tile into Q_k's buffer (every MMA that read Q_k
        // is complete: they precede the P V whose completion was awaited), in
        // the 128-byte swizzle of the tensor map: unit u of row e at
        // e * 128 + 16 * (u ^ (e & 7))
        uint8_t* row = smem + (k & 1) * kRowTile + e * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t* src = u < 4 ? o0 + 8 * u : o1 + 8 * (u - 4);
          uint4 v;
          v.x = pack2(__uint_as_float(src[0]) * il, __uint_as_float(src[1]) * il);
          v.y = pack2(__uint_as_float(src[2]) * il, __uint_as_float(src[3]) * il);
          v.z = pack2(__uint_as_float(src[4]) * il, __uint_as_float(src[5]) * il);
          v.w = pack2(__uint_as_float(src[6]) * il, __uint_as_float(src[7]) * il);
          *reinterpret_cast<uint4*>(row + ((u ^ (e & 7)) << 4)) = v;
        }
        fence_proxy_async();  // visible to the TMA store the producer issues
      } else if (q < T) {
        store_row64(p.out + (int64_t(row_base) + q) * C + w.h * D, o0, o1, il);
      }
      mbar_arrive(b_ost(k & 1));
      if (q < T) p.lse[(int64_t(w.b) * p.H + w.h) * T + q] = (m + log2f(l)) / kLog2e;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ====================================================================== backward

struct BwdParams {
  int T, C, H;
  const float* lse;
  const float* delta;
  bf16* dqkv;
  // score gradients kept for the dQ contraction (null: the dQ kernel
  // recomputes them): dS^T in 128 x 128 bf16 tiles [key][query], one per
  // (key block kb, query block qb >= kb), tile kb + qb (qb + 1) / 2 of
  // (batch, head) b * H + h, ntri = nqb (nqb + 1) / 2 tiles per (batch, head)
  bf16* dst;
  int ntri;
  int* err;
  // column sums of this CTA's 128 rows of dq, dk, dv (rows past T excluded)
  // -> bias_part[(b * gridDim.x + block) * 3C + column] (null: not computed)
  float* bias_part = nullptr;
};

// Sum over the 128 rows of the warpgroup of a 64-column row per thread into
// out[0..63], in a fixed order: thread e adds column e % 64 over rows
// 64 (e / 64) .. + 63 in eight interleaved chains (rows r = 8 i + k into chain
// k), the chains in order, then the two halves.  All 128 threads call it
// (named barriers); stg holds 128 x 65 floats of shared memory that nothing
// else uses at this point.
__device__ __forceinline__ void wg_colsum64(float* stg, int e, const float (&v)[64], float* out) {
#pragma unroll
  for (int c = 0; c < 64; ++c) stg[e * 65 + c] = v[c];
  wg_bar();
  const float* col = stg + (e >> 6) * 64 * 65 + (e & 63);
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = col[k * 65];
#pragma unroll
  for (int i = 1; i < 8; ++i)
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] += col[(8 * i + k) * 65];
  const float half = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  wg_bar();  // every read of stg done
  stg[e] = half;
  wg_bar();
  if (e < 64) out[e] = stg[e] + stg[64 + e];
  wg_bar();  // stg may be rewritten
}

// ---------------------------------------------------------------- dK, dV
// CTA: 128 keys kb*128 ..; 64-query tiles i from the diagonal to the end.
// TMEM: S^T +0, dP^T +64, dV +128, dK +192.  The warpgroup writes P^T (bf16)
// over the first 32 columns of S^T and dS^T over those of dP^T, where
// dV += P^T dO and dK += dS^T Q read them (A operands in TMEM).  MMA order per
// step i: dV(i-1) (after P^T_{i-1} is written); S^T_i; dK(i-1) (after dS^T_{i-1});
// dP^T_i: each MMA that overwrites a TMEM region is issued after the one
// that last reads it.
// KEEP: the warpgroup writes dS^T_i (bf16) into a 128-byte-swizzled 16 KB
// shared-memory tile instead of TMEM; dK += dS^T_i Q_i reads it from there
// (A K-major) and the MMA thread stores it into the score-gradient buffer with
// one TMA store, then waits for that store to have read the tile and tells the
// warpgroup (ds_free) that tile i+1 may be written.  The tile takes one Q/dO
// stage, so that two CTAs still share an SM.
template <bool KEEP>
struct DkdvCfg {
  static constexpr int NSK = KEEP ? 3 : 4;  // Q/dO stages
  static constexpr int kStage = KEEP ? kRowTile : 0;
  static constexpr int kSmem = 2 * kRowTile + NSK * 2 * kStrTile + kStage + 2 * BS * 4 + 256 + 1024;
};

template <bool KEEP>
__global__ void __launch_bounds__(kThreads, 2)
    fa_tc_dkdv_kernel(const __grid_constant__ CUtensorMap q128, const __grid_constant__ CUtensorMap q64,
                      const __grid_constant__ CUtensorMap o64, const __grid_constant__ CUtensorMap ds_map,
                      const __grid_constant__ CUtensorMap dqkv_map, const BwdParams p) {
  constexpr int NSK = DkdvCfg<KEEP>::NSK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sK = smem_u32(smem), sV = sK + kRowTile;
  const uint32_t sQ = sV + kRowTile;            // NSK x 8 KB
  const uint32_t sO = sQ + NSK * kStrTile;      // dO, NSK x 8 KB
  uint8_t* sDs = smem + 2 * kRowTile + 2 * NSK * kStrTile;  // KEEP: dS^T, 128 x 64 bf16
  float* sLD = reinterpret_cast<float*>(sDs + DkdvCfg<KEEP>::kStage);  // [64] -lse*log2e, [64] -delta
  uint64_t* bars = reinterpret_cast<uint64_t*>(sLD + 2 * BS);
  // kv_full | qo_full[NSK] | qo_empty[NSK] | s_full | p_full | dp_full | ds_full | mm_done |
  // ds_free | slot
  const uint32_t b_kv = smem_u32(bars);
  auto b_qf = [&](int s) { return smem_u32(bars + 1 + s); };
  auto b_qe = [&](int s) { return smem_u32(bars + 1 + NSK + s); };
  const uint32_t b_sf = smem_u32(bars + 1 + 2 * NSK);
  const uint32_t b_pf = smem_u32(bars + 2 + 2 * NSK);
  const uint32_t b_dpf = smem_u32(bars + 3 + 2 * NSK);
  const uint32_t b_df = smem_u32(bars + 4 + 2 * NSK);
  const uint32_t b_mm = smem_u32(bars + 5 + 2 * NSK);
  const uint32_t b_dsf = smem_u32(bars + 6 + 2 * NSK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7 + 2 * NSK);

  // longest first within groups of 24 (batch, head) pairs: the key blocks
  // of a pair run close together and share its Q / dO tiles in L2 (fully
  // longest-first measured 4 us slower at B=16, T=1024, H=12)
  const WorkItem wi = work_item(24);
  const int kb = wi.step;
  const int h = wi.h, b = wi.b;
  const int T = p.T, C = p.C;
  const int qt0 = (kb * BR) / BS;
  const int nqt = (T + BS - 1) / BS;
  const int n = nqt - qt0;
  const int row_base = b * T;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(b_kv, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(b_qf(s), 1);
      mbar_init(b_qe(s), 1);
    }
    mbar_init(b_sf, 1);
    mbar_init(b_pf, 128);
    mbar_init(b_dpf, 1);
    mbar_init(b_df, 128);
    mbar_init(b_mm, 1);
    mbar_init(b_dsf, 1);
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
      const int s = i % NSK;
      if (!mbar_wait(b_qe(s), ((i / NSK) & 1) ^ 1, p.err, 21)) break;
      mbar_expect_tx(b_qf(s), 2 * kStrTile);
      const int row = row_base + (qt0 + i) * BS;
      tma_load_2d(sQ + s * kStrTile, &q64, b_qf(s), h * D, row);
      tma_load_2d(sO + s * kStrTile, &o64, b_qf(s), h * D, row);
      ++issued;
    }
    mbar_wait(b_kv, 0, p.err, 25);
    for (int q = 1; q <= min(issued, NSK); ++q) {
      const int idx = issued - q;
      mbar_wait(b_qf(idx % NSK), uint32_t((idx / NSK) & 1), p.err, 25);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t id_s = idesc_bf16(BR, BS, 0, 0);
    const uint32_t id_o = idesc_bf16(BR, D, 0, 1);
    // slice-0 descriptors, stage s adds s * kStrTile bytes
    const uint64_t dK = desc_kmajor(sK, 0), dV = desc_kmajor(sV, 0);
    const uint64_t dQ = desc_kmajor(sQ, 0), dO = desc_kmajor(sO, 0);
    const uint64_t dQm = desc_mnmajor(sQ, 0), dOm = desc_mnmajor(sO, 0);
    bool ok = mbar_wait(b_kv, 0, p.err, 22);
    int mm = 0;
    for (int i = 0; ok && i <= n; ++i) {
      const int s = i % NSK, si = (i + NSK - 1) % NSK;  // stages of tiles i and i-1
      if (i >= 1) {  // dV += P^T_{i-1} dO_{i-1}
        if (!mbar_wait(b_pf, (i - 1) & 1, p.err, 23)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_ts4(tV, tS, desc_offset(dOm, si * kStrTile), id_o, 128, i > 1);
      }
      if (i < n) {  // S^T_i = K Q_i^T
        if (!mbar_wait(b_qf(s), (i / NSK) & 1, p.err, 22)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_ss4(tS, dK, desc_offset(dQ, s * kStrTile), id_s, 2, 2, false);
        umma_commit(b_sf);
      }
      if (i >= 1) {  // dK += dS^T_{i-1} Q_{i-1}
        if (!mbar_wait(b_df, (i - 1) & 1, p.err, 24)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (KEEP) {
          mma_ss4(tKd, desc_kmajor(smem_u32(sDs), 0), desc_offset(dQm, si * kStrTile), id_o, 2,
                  128, i > 1);
        } else {
          mma_ts4(tKd, tP, desc_offset(dQm, si * kStrTile), id_o, 128, i > 1);
        }
        umma_commit(b_mm);
        umma_commit(b_qe(si));
        ++mm;
        if (KEEP) {  // dS^T_{i-1} into its tile of the score-gradient buffer
          const int qt = qt0 + i - 1, qbt = qt >> 1;
          const int y = int((int64_t(b * p.H + h) * p.ntri + qbt * (qbt + 1) / 2 + kb) * BR);
          tma_store_2d_l2(&ds_map, smem_u32(sDs), (qt & 1) * BS, y, l2_keep());
          bulk_commit();
        }
      }
      if (i < n) {  // dP^T_i = V dO_i^T
        mma_ss4(tP, dV, desc_offset(dO, s * kStrTile), id_s, 2, 2, false);
        umma_commit(b_dpf);
        if (KEEP && i >= 1) {  // the store of dS^T_{i-1} has read the tile
          bulk_wait_read<0>();
          mbar_arrive(b_dsf);
        }
      }
    }
    if (KEEP) bulk_wait_all();
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
      if (ok) ok = mbar_wait(b_sf, i & 1, p.err, 27);
      tc_fence_after();
      wg_bar();  // sLD of this tile visible
      const bool need_mask = q0 < kb * BR + BR || q0 + BS > T;
      // P^T = 2^(S^T sl2 - lse log2 e), masked; kept in fp32 for dS^T
      float pv[64];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t sx[32];
        tmem_ld32_async(tS + lo + 32 * hh, sx);
        tmem_wait_ld(sx);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {  // branch-free, so the pairs interleave
          const int qc = 32 * hh + c;  // query column within the tile
          const float2 nl = *reinterpret_cast<const float2*>(sLD + qc);
          float t0, t1;
          fma2(t0, t1, __uint_as_float(sx[c]), __uint_as_float(sx[c + 1]), sl2, sl2, nl.x, nl.y);
          if (((qc >> 1) % 2 == 1)) {
            ex2_poly2(t0, t1, pv[qc], pv[qc + 1]);
          } else {
            pv[qc] = ex2(t0);
            pv[qc + 1] = ex2(t1);
          }
        }
      }
      if (need_mask) {
#pragma unroll
        for (int qc = 0; qc < 64; ++qc)
          pv[qc] = (q0 + qc < key || q0 + qc >= T) ? 0.f : pv[qc];
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) pk[c >> 1] = pack2(pv[c], pv[c + 1]);
        tmem_st32_async(tS + lo, pk);  // P^T over the first 32 columns of S^T
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(b_pf);
      if (ok) ok = mbar_wait(b_dpf, i & 1, p.err, 28);
      tc_fence_after();
      uint32_t pd[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t dx[32];
        tmem_ld32_async(tP + lo + 32 * hh, dx);
        tmem_wait_ld(dx);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const int qc = 32 * hh + c;
          const float2 nd = *reinterpret_cast<const float2*>(sLD + BS + qc);  // -delta
          float g0 = __uint_as_float(dx[c]), g1 = __uint_as_float(dx[c + 1]);
          add2(g0, g1, nd.x, nd.y);        // dP - delta
          mul2(g0, g1, pv[qc], pv[qc + 1]);  // dS = P (dP - delta)
          pd[qc >> 1] = pack2(g0, g1);
        }
      }
      if (KEEP) {
        // row e of the dS^T tile (K-major, 128-byte swizzle), once the dK MMA
        // (done before dP^T_i) and the store of dS^T_{i-1} have read it
        if (i > 0 && ok) ok = mbar_wait(b_dsf, (i - 1) & 1, p.err, 30);
        uint8_t* row = sDs + e * 128;
#pragma unroll
        for (int v = 0; v < 8; ++v)
          *reinterpret_cast<uint4*>(row + ((v ^ (e & 7)) << 4)) =
              make_uint4(pd[4 * v], pd[4 * v + 1], pd[4 * v + 2], pd[4 * v + 3]);
        fence_proxy_async();  // visible to the MMA and the bulk copy
      } else {
        tmem_st32_async(tP + lo, pd);  // dS^T over the first 32 columns of dP^T
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(b_df);
      wg_bar();  // sLD may be rewritten for the next tile
    }
    ok = __all_sync(0xffffffffu, ok);
    bool have = false;
    if (ok && n > 0) {
      const bool w = mbar_wait(b_mm, (n - 1) & 1, p.err, 29);
      have = __all_sync(0xffffffffu, w);
    }
    if (have) tc_fence_after();
    bf16* drow = p.dqkv + (int64_t(row_base) + key) * 3 * C + h * D;
    // a whole key block leaves its dV and dK tiles in two 16 KB buffers of
    // the Q/dO ring (idle now: every load has been consumed by an MMA that
    // has completed; the column sums below use the K/V tiles) for two TMA
    // stores; a block that runs past T is stored row by row (a 2-D box would
    // reach into the next sequence)
    const bool whole = (kb + 1) * BR <= T;
    uint8_t* stage = smem + 40 * 1024;
    // dV then dK, one 64-column row each (and their column sums: every
    // thread of the warpgroup takes part, whatever the waits gave)
#pragma unroll 1
    for (int w2 = 0; w2 < 2; ++w2) {
      uint32_t a0[32], a1[32];
      if (have) {
        tmem_ld32_async((w2 ? tKd : tV) + lo, a0);
        tmem_ld32_async((w2 ? tKd : tV) + lo + 32, a1);
        tmem_wait_ld(a0);
        reg_after_wait(a1);
        const float f = w2 ? scale : 1.f;
        if (whole) {
          // row e in the 128-byte swizzle of the tensor map: unit u at e * 128 + 16 * (u ^ (e & 7))
          uint8_t* row = stage + w2 * kRowTile + e * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t* src = u < 4 ? a0 + 8 * u : a1 + 8 * (u - 4);
            uint4 v;
            v.x = pack2(__uint_as_float(src[0]) * f, __uint_as_float(src[1]) * f);
            v.y = pack2(__uint_as_float(src[2]) * f, __uint_as_float(src[3]) * f);
            v.z = pack2(__uint_as_float(src[4]) * f, __uint_as_float(src[5]) * f);
            v.w = pack2(__uint_as_float(src[6]) * f, __uint_as_float(src[7]) * f);
            *reinterpret_cast<uint4*>(row + ((u ^ (e & 7)) << 4)) = v;
          }
          fence_proxy_async();  // visible to the TMA stores below
        } else if (key < T) {
          store_row64(drow + (w2 ? C : 2 * C), a0, a1, f);
        }
      }
      if (p.bias_part) {
        // the K / V rows of the keys past T are excluded by selection (a
        // product with 0 would keep a NaN of a row nothing defines)
        const bool use = have && key < T;
        const float f = w2 ? scale : 1.f;
        float v[64];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          v[c] = use ? __uint_as_float(a0[c]) * f : 0.f;
          v[32 + c] = use ? __uint_as_float(a1[c]) * f : 0.f;
        }
        // the K/V tiles' shared memory: every MMA that read it has completed
        wg_colsum64(reinterpret_cast<float*>(smem), e, v,
                    p.bias_part + (int64_t(b) * gridDim.x + kb) * 3 * C + (w2 ? C : 2 * C) +
                        h * D);
      }
    }
    wg_bar();  // every row of both tiles written
    if (whole && have && e == 0) {
      tma_store_2d(&dqkv_map, smem_u32(stage), 2 * C + h * D, row_base + kb * BR);             // dV
      tma_store_2d(&dqkv_map, smem_u32(stage + kRowTile), C + h * D, row_base + kb * BR);  // dK
      bulk_commit();
      bulk_wait_read<0>();  // the shared memory is released with the CTA
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- dQ
// CTA: 128 queries qb*128 ..; 64-key tiles j up to the diagonal.
// TMEM: S +0, dP +64, dQ +128, dS +192.  The warpgroup writes dS_j (bf16,
// 32 columns) to its own region, where dQ += dS_j K_j reads it (A operand in
// TMEM).  MMA order per step j: S_j (once the warpgroup has read S_{j-1});
// dP_j (once it has read dP_{j-1}); dQ += dS_{j-1} K_{j-1} (once dS_{j-1} is
// written).  S_j and dP_j are so issued while the warpgroup still works on
// tile j-1; it waits for dQ(j-1) only before it overwrites dS.
constexpr int NSQ = 4;  // K/V stages
constexpr int kDqSmem = 2 * kRowTile + NSQ * 2 * kStrTile + 256 + 1024;

__global__ void __launch_bounds__(kThreads, 2)
    fa_tc_dq_kernel(const __grid_constant__ CUtensorMap q128, const __grid_constant__ CUtensorMap q64,
                    const __grid_constant__ CUtensorMap o128, const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sQ = smem_u32(smem), sO = sQ + kRowTile;
  const uint32_t sK = sO + kRowTile;            // NSQ x 8 KB
  const uint32_t sV = sK + NSQ * kStrTile;      // NSQ x 8 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kRowTile + 2 * NSQ * kStrTile);
  // q_full | kv_full[NSQ] | kv_empty[NSQ] | s_full | s_read | dp_full | ds_full | dq_done | dp_read | slot
  const uint32_t b_q = smem_u32(bars);
  auto b_kf = [&](int s) { return smem_u32(bars + 1 + s); };
  auto b_ke = [&](int s) { return smem_u32(bars + 1 + NSQ + s); };
  const uint32_t b_sf = smem_u32(bars + 1 + 2 * NSQ);
  const uint32_t b_sfr = smem_u32(bars + 2 + 2 * NSQ);
  const uint32_t b_dpf = smem_u32(bars + 3 + 2 * NSQ);
  const uint32_t b_df = smem_u32(bars + 4 + 2 * NSQ);
  const uint32_t b_mm = smem_u32(bars + 5 + 2 * NSQ);
  const uint32_t b_dpr = smem_u32(bars + 6 + 2 * NSQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7 + 2 * NSQ);
  const WorkItem wi = work_item();
  const int qb = gridDim.x - 1 - wi.step;
  const int h = wi.h, b = wi.b;
  const int T = p.T, C = p.C;
  const int last_key = min(T, (qb + 1) * BR) - 1;
  const int nkt = last_key / BS + 1;
  const int row_base = b * T;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < NSQ; ++s) {
      mbar_init(b_kf(s), 1);
      mbar_init(b_ke(s), 1);
    }
    mbar_init(b_sf, 1);
    mbar_init(b_sfr, 128);
    mbar_init(b_dpf, 1);
    mbar_init(b_df, 128);
    mbar_init(b_mm, 1);
    mbar_init(b_dpr, 128);
    init_bar_fence();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 64, tQd = tmem + 128, tDs = tmem + 192;
  if (warp == 0 && lane == 0) {
    mbar_expect_tx(b_q, 2 * kRowTile);
    tma_load_2d(sQ, &q128, b_q, h * D, row_base + qb * BR);
    tma_load_2d(sO, &o128, b_q, h * D, row_base + qb * BR);
    int issued = 0;
    for (int j = 0; j < nkt; ++j) {
      const int s = j % NSQ;
      if (!mbar_wait(b_ke(s), ((j / NSQ) & 1) ^ 1, p.err, 31)) break;
      mbar_expect_tx(b_kf(s), 2 * kStrTile);
      tma_load_2d(sK + s * kStrTile, &q64, b_kf(s), C + h * D, row_base + j * BS);
      tma_load_2d(sV + s * kStrTile, &q64, b_kf(s), 2 * C + h * D, row_base + j * BS);
      ++issued;
    }
    mbar_wait(b_q, 0, p.err, 35);
    for (int q = 1; q <= min(issued, NSQ); ++q) {
      const int idx = issued - q;
      mbar_wait(b_kf(idx % NSQ), uint32_t((idx / NSQ) & 1), p.err, 35);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t id_s = idesc_bf16(BR, BS, 0, 0);
    const uint32_t id_o = idesc_bf16(BR, D, 0, 1);
    // slice-0 descriptors, stage s adds s * kStrTile bytes
    const uint64_t dQ = desc_kmajor(sQ, 0), dO = desc_kmajor(sO, 0);
    const uint64_t dK = desc_kmajor(sK, 0), dV = desc_kmajor(sV, 0), dKm = desc_mnmajor(sK, 0);
    bool ok = mbar_wait(b_q, 0, p.err, 32);
    int mm = 0;
    for (int j = 0; ok && j <= nkt; ++j) {
      const int s = j % NSQ;
      if (j < nkt) {
        if (!mbar_wait(b_kf(s), (j / NSQ) & 1, p.err, 32) ||
            !mbar_wait(b_sfr, (j & 1) ^ 1, p.err, 32)) {  // S_{j-1} read
          ok = false;
          break;
        }
        tc_fence_after();
        mma_ss4(tS, dQ, desc_offset(dK, s * kStrTile), id_s, 2, 2, false);
        umma_commit(b_sf);
        if (!mbar_wait(b_dpr, (j & 1) ^ 1, p.err, 32)) {  // dP_{j-1} read
          ok = false;
          break;
        }
        tc_fence_after();
        mma_ss4(tP, dO, desc_offset(dV, s * kStrTile), id_s, 2, 2, false);
        umma_commit(b_dpf);
      }
      if (j >= 1) {
        const int jj = j - 1, sj = jj % NSQ;
        if (!mbar_wait(b_df, jj & 1, p.err, 33)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_ts4(tQd, tDs, desc_offset(dKm, sj * kStrTile), id_o, 128, jj > 0);
        umma_commit(b_mm);
        umma_commit(b_ke(sj));
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
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s0[32], s1[32];
      tmem_ld32_async(tS + lo, s0);
      tmem_ld32_async(tS + lo + 32, s1);
      tmem_wait_ld(s0);
      reg_after_wait(s1);
      tc_fence_before();
      mbar_arrive(b_sfr);
      const int key0 = j * BS;
      const bool need_mask = key0 + BS - 1 > qb * BR || key0 + BS > T || qb * BR + BR > T;
      float pv[64];  // P = 2^(S sl2 - lse log2 e), masked
#pragma unroll
      for (int c = 0; c < 64; c += 2) {  // branch-free, so the pairs interleave
        const float sa = __uint_as_float(c < 32 ? s0[c] : s1[c - 32]);
        const float sb = __uint_as_float(c < 32 ? s0[c + 1] : s1[c - 31]);
        float t0, t1;
        fma2(t0, t1, sa, sb, sl2, sl2, -L2, -L2);
        pv[c] = ex2(t0);
        pv[c + 1] = ex2(t1);
      }
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          pv[c] = (key0 + c > q || key0 + c >= T || q >= T) ? 0.f : pv[c];
      }
      w = mbar_wait(b_dpf, j & 1, p.err, 38);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t d0[32], d1[32];
      tmem_ld32_async(tP + lo, d0);
      tmem_ld32_async(tP + lo + 32, d1);
      tmem_wait_ld(d0);
      reg_after_wait(d1);
      tc_fence_before();
      mbar_arrive(b_dpr);  // dP_j read: the MMA may write dP_{j+1}
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float g0 = __uint_as_float(c < 32 ? d0[c] : d1[c - 32]);
        float g1 = __uint_as_float(c < 32 ? d0[c + 1] : d1[c - 31]);
        add2(g0, g1, -Dl, -Dl);            // dP - delta
        mul2(g0, g1, pv[c], pv[c + 1]);    // dS = P (dP - delta)
        pk[c >> 1] = pack2(g0, g1);
      }
      // dS_{j-1} consumed by its dQ MMA before dS_j overwrites it
      if (j >= 1) {
        w = mbar_wait(b_mm, (j - 1) & 1, p.err, 39);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      tmem_st32_async(tDs + lo, pk);
      tmem_wait_st();
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

// ---------------------------------------------------------------- dQ from kept dS
// With the score gradients kept by the dK/dV kernel, dQ is a plain contraction,
// dQ_i = sum_j dS_ij K_j / sqrt(D), with no exponentials and no recomputed S
// or dP.  CTA: 128 queries, 64-key steps up to the diagonal; one TMA stage =
// dS^T of the 64 keys x 128 queries (two 64-query chunks: A MN-major) and K_j
// (64 keys x 64 channels: B MN-major); TMEM: one 128 x 64 fp32 accumulator.
constexpr int NSG = 3;                            // stages (three CTAs per SM)
constexpr int kGStage = kRowTile + kStrTile;      // 16 KB dS^T + 8 KB K
constexpr int kDqgSmem = NSG * kGStage + 256 + 1024;
constexpr int kDqgTmemCols = 64;

__global__ void __launch_bounds__(kThreads, 3)
    fa_tc_dq_ds_kernel(const __grid_constant__ CUtensorMap ds_map,
                       const __grid_constant__ CUtensorMap q64, const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NSG * kGStage);
  // full[NSG] | empty[NSG] | acc_done | slot
  auto b_full = [&](int s) { return smem_u32(bars + s); };
  auto b_empty = [&](int s) { return smem_u32(bars + NSG + s); };
  const uint32_t b_acc = smem_u32(bars + 2 * NSG);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NSG + 1);
  const WorkItem wi = work_item();
  const int qb = gridDim.x - 1 - wi.step;
  const int h = wi.h, b = wi.b;
  const int T = p.T, C = p.C;
  const int last_key = min(T, (qb + 1) * BR) - 1;
  const int nkt = last_key / BS + 1;
  const int row_base = b * T;
  const int64_t tile0 = (int64_t(b) * p.H + h) * p.ntri + qb * (qb + 1) / 2;  // (kb 0, qb)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSG; ++s) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    mbar_init(b_acc, 1);
    init_bar_fence();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kDqgTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0 && lane == 0) {
    int issued = 0;
    for (int j = 0; j < nkt; ++j) {
      const int s = j % NSG;
      if (!mbar_wait(b_empty(s), ((j / NSG) & 1) ^ 1, p.err, 41)) break;
      const uint32_t sa = sbase + s * kGStage;
      const int y = int((tile0 + (j >> 1)) * BR + (j & 1) * BS);  // first key row of step j
      mbar_expect_tx(b_full(s), kGStage);
      tma_load_2d_l2(sa, &ds_map, b_full(s), 0, y, l2_once());
      tma_load_2d_l2(sa + BK * 128, &ds_map, b_full(s), BS, y, l2_once());
      tma_load_2d(sa + kRowTile, &q64, b_full(s), C + h * D, row_base + j * BS);
      ++issued;
    }
    for (int q = 1; q <= min(issued, NSG); ++q) {
      const int idx = issued - q;
      mbar_wait(b_full(idx % NSG), uint32_t((idx / NSG) & 1), p.err, 45);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t id = idesc_bf16(BR, D, 1, 1);
    const uint64_t dA = desc_mnmajor(sbase, 0), dB = desc_mnmajor(sbase + kRowTile, 0);
    for (int j = 0; j < nkt; ++j) {
      const int s = j % NSG;
      if (!mbar_wait(b_full(s), (j / NSG) & 1, p.err, 42)) break;
      tc_fence_after();
      mma_ss4(tmem, desc_offset(dA, s * kGStage), desc_offset(dB, s * kGStage), id, 128, 128,
              j > 0);
      umma_commit(b_empty(s));
    }
    // tracks every MMA issued, so the accumulator is released only after them
    umma_commit(b_acc);
    mbar_wait(b_acc, 0, p.err, 43);
  } else if (warp >= 2) {
    const int e = (warp & 3) * 32 + lane;  // query row in the block = TMEM lane
    const int q = qb * BR + e;
    const uint32_t lo = uint32_t((warp & 3) * 32) << 16;
    const bool w = mbar_wait(b_acc, 0, p.err, 44);
    const bool have = __all_sync(0xffffffffu, w);
    const float scale = rsqrtf(float(D));
    uint32_t a0[32], a1[32];
    if (have) {
      tc_fence_after();
      tmem_ld32_async(tmem + lo, a0);
      tmem_ld32_async(tmem + lo + 32, a1);
      tmem_wait_ld(a0);
      reg_after_wait(a1);
      if (q < T) store_row64(p.dqkv + (int64_t(row_base) + q) * 3 * C + h * D, a0, a1, scale);
    }
    if (p.bias_part) {
      // the rows of the queries past T are excluded by selection: their score
      // gradients may be memory nothing has written (a product with 0 would
      // keep a NaN)
      const bool use = have && q < T;
      float v[64];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        v[c] = use ? __uint_as_float(a0[c]) * scale : 0.f;
        v[32 + c] = use ? __uint_as_float(a1[c]) * scale : 0.f;
      }
      // the stage ring: every copy into it has been consumed by the MMAs
      wg_colsum64(reinterpret_cast<float*>(smem), e, v,
                  p.bias_part + (int64_t(b) * gridDim.x + qb) * 3 * C + h * D);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kDqgTmemCols);
}

}  // namespace

size_t attn_tc_ds_bytes(int B, int T, int H) {
  const int64_t nqb = cdiv(T, BR);
  return size_t(B) * H * (nqb * (nqb + 1) / 2) * BR * BR * sizeof(bf16);
}

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
  CUtensorMap mo;
  if (!make_map_bf16(&m128, qkv, 3 * int64_t(C), rows, 3 * int64_t(C), BR) ||
      !make_map_bf16(&m64, qkv, 3 * int64_t(C), rows, 3 * int64_t(C), BS) ||
      !make_map_bf16(&mo, out, int64_t(C), rows, int64_t(C), BR)) {
    gpt2_internal::set_error("attention: tensor map encoding failed");
    return GPT2_ERR_CUDA;
  }
  const int nblk = cdiv(T, BR);
  const int64_t items = int64_t(nblk) * H * B;
  if (items <= 0) return GPT2_OK;
  FwdParams p{T, C, H, nblk, int(items), out, lse, device_error_word()};
  const int grid = int(std::min<int64_t>(items, 2 * int64_t(gpt2_internal::sm_count())));
  fa_tc_fwd_kernel<<<grid, kThreads, kFwdSmem, st>>>(m128, m64, mo, p);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_attn_tc_bwd(const bf16* dout, const bf16* qkv, const float* lse, const float* delta,
                       int B, int T, int C, int H, bf16* dqkv, bf16* ds, float* bias_part,
                       cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(fa_tc_dkdv_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         DkdvCfg<false>::kSmem);
    cudaFuncSetAttribute(fa_tc_dkdv_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         DkdvCfg<true>::kSmem);
    cudaFuncSetAttribute(fa_tc_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem);
    cudaFuncSetAttribute(fa_tc_dq_ds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqgSmem);
    attr = true;
  }
  const int nqb = cdiv(T, BR), ntri = nqb * (nqb + 1) / 2;
  const int64_t ds_rows = int64_t(B) * H * ntri * BR;
  if (ds && (reinterpret_cast<uintptr_t>(ds) % 16 || ds_rows >= (int64_t(1) << 31))) {
    gpt2_internal::set_error("attention: score-gradient buffer misaligned or too large");
    return GPT2_ERR_ARG;
  }
  CUtensorMap q128, q64, o128, o64, dmap;
  const int64_t rows = int64_t(B) * T;
  if (!make_map_bf16(&q128, qkv, 3 * int64_t(C), rows, 3 * int64_t(C), BR) ||
      !make_map_bf16(&q64, qkv, 3 * int64_t(C), rows, 3 * int64_t(C), BS) ||
      !make_map_bf16(&o128, dout, int64_t(C), rows, int64_t(C), BR) ||
      !make_map_bf16(&o64, dout, int64_t(C), rows, int64_t(C), BS) ||
      !make_map_bf16(&dmap, dqkv, 3 * int64_t(C), rows, 3 * int64_t(C), BR)) {
    gpt2_internal::set_error("attention: tensor map encoding failed");
    return GPT2_ERR_CUDA;
  }
  // score-gradient buffer: stored as 128-key x 64-query boxes, read as 64 x 64
  CUtensorMap ds_st, ds_ld;
  if (ds && (!make_map_bf16(&ds_st, ds, BR, ds_rows, BR, BR) ||
             !make_map_bf16(&ds_ld, ds, BR, ds_rows, BR, BS))) {
    gpt2_internal::set_error("attention: tensor map encoding failed");
    return GPT2_ERR_CUDA;
  }
  BwdParams p{T, C, H, lse, delta, dqkv, ds, ntri, device_error_word(), ds ? bias_part : nullptr};
  dim3 grid(nqb, H, B);
  if (ds) {
    fa_tc_dkdv_kernel<true><<<grid, kThreads, DkdvCfg<true>::kSmem, st>>>(q128, q64, o64, ds_st, dmap,
                                                                          p);
    COUNT_LAUNCH(1);
    fa_tc_dq_ds_kernel<<<grid, kThreads, kDqgSmem, st>>>(ds_ld, q64, p);
  } else {
    fa_tc_dkdv_kernel<false><<<grid, kThreads, DkdvCfg<false>::kSmem, st>>>(q128, q64, o64, q64,
                                                                            dmap, p);
    COUNT_LAUNCH(1);
    fa_tc_dq_kernel<<<grid, kThreads, kDqSmem, st>>>(q128, q64, o128, p);
  }
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
