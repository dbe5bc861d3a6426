// Causal flash attention on tensor cores (bf16 in, fp32 accumulate), head
// size 64, for the bf16 training path [ZERO: Attention, OpFlashAttention;
// LECTURE: flash attention with the causal mask].
//
// The [T, T] scores never leave registers.  Forward: one CTA per (64-query
// block, head, sequence), 4 warps x 16 query rows; K/V tiles of 64 keys
// double-buffered in shared memory by cp.async; S = Q K^T and O += P V with
// mma.sync m16n8k16; online softmax in the log2 domain; saves the row
// log-normaliser (natural log) for the backward.  Blocks above the diagonal
// are skipped; the heaviest query blocks are scheduled first.
//
// Backward (deterministic, no atomics), with Delta_i = dO_i . O_i:
//   kernel dKdV: one CTA per 64-key block, loops over query blocks i >= j:
//     S^T = K Q^T, P^T = exp(S^T/sqrt(D) - lse), dP^T = V dO^T,
//     dS^T = P^T (dP^T - Delta), dV += P^T dO, dK += dS^T Q / sqrt(D);
//   kernel dQ: one CTA per 64-query block, loops over key blocks j <= i:
//     recomputes P and dP, dQ += dS K / sqrt(D).

#include "kernels.h"

namespace {

constexpr int D = 64;
constexpr int BQ = 64;    // query rows per CTA (16 per warp)
constexpr int BKV = 64;   // keys per tile
constexpr int LDS = 72;   // padded smem row (elements): conflict-free ldmatrix
constexpr int TILE = BQ * LDS;  // elements per smem tile
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t s_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Copies rows [r0, r0+64) x 64 columns of a row-major bf16 matrix (row stride
// `ld` elements) into a padded smem tile; rows >= nrows are zero-filled.
__device__ __forceinline__ void load_tile(bf16* s, const bf16* g, int64_t ld, int r0, int nrows) {
  for (int c = threadIdx.x; c < BQ * (D / 8); c += blockDim.x) {
    const int r = c >> 3, col = (c & 7) * 8;
    const int gr = r0 + r;
    const bool ok = gr < nrows;
    cp_async16(s_addr(s + r * LDS + col), g + int64_t(ok ? gr : 0) * ld + col, ok);
  }
}

// A fragments (16 rows x 64) of rows row0.. of an smem tile: a[kc] covers
// columns 16kc .. 16kc+15.
__device__ __forceinline__ void load_a_frags(const bf16* s, int row0, uint32_t (&a)[4][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kc = 0; kc < 4; ++kc)
    ldsm_x4(s_addr(s + (row0 + (lane & 15)) * LDS + kc * 16 + (lane >> 4) * 8), a[kc]);
}

// acc[nt] (16 x 8 each, nt = 0..7) += A (16 x 64, fragments a) * M^T where M is
// an smem tile [64 rows = n][64 cols = k]: B(k, n) = M[n][k].
__device__ __forceinline__ void mma_abt(const uint32_t (&a)[4][4], const bf16* s,
                                        float (&acc)[8][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kc = 0; kc < 4; ++kc)
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b[4];
      ldsm_x4(s_addr(s + (np * 16 + (lane & 7) + ((lane >> 4) << 3)) * LDS + kc * 16 +
                     ((lane >> 3) & 1) * 8),
              b);
      mma16816(acc[2 * np], a[kc], b[0], b[1]);
      mma16816(acc[2 * np + 1], a[kc], b[2], b[3]);
    }
}

// acc[nt] (16 x 8, nt over 64 columns n) += P (16 x 64 over k, given as fp32
// accumulator fragments p[8][4]) * M where M is an smem tile [64 rows = k][64
// cols = n]: B(k, n) = M[k][n].
__device__ __forceinline__ void mma_pm(const float (&p)[8][4], const bf16* s, float (&acc)[8][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kc = 0; kc < 4; ++kc) {
    uint32_t a[4];
    a[0] = pack_bf16(p[2 * kc][0], p[2 * kc][1]);
    a[1] = pack_bf16(p[2 * kc][2], p[2 * kc][3]);
    a[2] = pack_bf16(p[2 * kc + 1][0], p[2 * kc + 1][1]);
    a[3] = pack_bf16(p[2 * kc + 1][2], p[2 * kc + 1][3]);
#pragma unroll
    for (int dp = 0; dp < 4; ++dp) {
      uint32_t b[4];
      ldsm_x4_t(s_addr(s + (kc * 16 + (lane & 15)) * LDS + dp * 16 + (lane >> 4) * 8), b);
      mma16816(acc[2 * dp], a, b[0], b[1]);
      mma16816(acc[2 * dp + 1], a, b[2], b[3]);
    }
  }
}

__device__ __forceinline__ void zero(float (&x)[8][4]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) x[i][j] = 0.f;
}

// ------------------------------------------------------------------ forward
__global__ void __launch_bounds__(128) fa_fwd_kernel(const bf16* __restrict__ qkv, int T, int C,
                                                     int H, bf16* __restrict__ out,
                                                     float* __restrict__ lse) {
  extern __shared__ __align__(16) uint8_t smraw[];
  bf16* sQ = reinterpret_cast<bf16*>(smraw);
  bf16* sK = sQ + TILE;       // 2 buffers
  bf16* sV = sK + 2 * TILE;   // 2 buffers
  const int qb = gridDim.x - 1 - blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int64_t rs = 3 * int64_t(C);
  const bf16* Qg = qkv + int64_t(b) * T * rs + h * D;
  const bf16* Kg = Qg + C;
  const bf16* Vg = Qg + 2 * C;
  const float sl2 = rsqrtf(float(D)) * kLog2e;

  load_tile(sQ, Qg, rs, qb * BQ, T);
  load_tile(sK, Kg, rs, 0, T);
  load_tile(sV, Vg, rs, 0, T);
  cp_commit();

  float o[8][4];
  zero(o);
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  uint32_t qf[4][4];
  const int q0 = qb * BQ + warp * 16 + g;  // this thread's rows q0 and q0 + 8

  for (int kb = 0; kb <= qb; ++kb) {
    const int buf = kb & 1;
    if (kb < qb) {
      load_tile(sK + (buf ^ 1) * TILE, Kg, rs, (kb + 1) * BKV, T);
      load_tile(sV + (buf ^ 1) * TILE, Vg, rs, (kb + 1) * BKV, T);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (kb == 0) load_a_frags(sQ, warp * 16, qf);
    float s[8][4];
    zero(s);
    mma_abt(qf, sK + buf * TILE, s);
    // scale, mask (key > query, or beyond T), online softmax (log2 domain)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kb * BKV + nt * 8 + 2 * t4 + (e & 1);
        const int q = q0 + (e >> 1) * 8;
        float v = s[nt][e] * sl2;
        if (key > q || key >= T) v = -INFINITY;
        s[nt][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    float corr[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float mn = fmaxf(mrow[r], mx[r]);
      corr[r] = exp2f(mrow[r] - mn);
      mrow[r] = mn;
      lrow[r] *= corr[r];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[nt][e] - mrow[e >> 1]);
        s[nt][e] = p;
        lrow[e >> 1] += p;
        o[nt][e] *= corr[e >> 1];
      }
    mma_pm(s, sV + buf * TILE, o);
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int q = q0 + r * 8;
    if (q >= T) continue;
    const float inv = 1.f / lrow[r];
    bf16* orow = out + (int64_t(b) * T + q) * C + h * D;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<uint32_t*>(orow + nt * 8 + 2 * t4) =
          pack_bf16(o[nt][2 * r] * inv, o[nt][2 * r + 1] * inv);
    if (t4 == 0) lse[(int64_t(b) * H + h) * T + q] = (mrow[r] + log2f(lrow[r])) / kLog2e;
  }
}

// ------------------------------------------------------------------ backward: dK, dV
__global__ void __launch_bounds__(128) fa_bwd_dkdv_kernel(const bf16* __restrict__ dout,
                                                          const bf16* __restrict__ qkv,
                                                          const float* __restrict__ lse,
                                                          const float* __restrict__ delta, int T,
                                                          int C, int H, bf16* __restrict__ dqkv) {
  extern __shared__ __align__(16) uint8_t smraw[];
  bf16* sK = reinterpret_cast<bf16*>(smraw);
  bf16* sV = sK + TILE;
  bf16* sQ = sV + TILE;        // 2 buffers
  bf16* sO = sQ + 2 * TILE;    // dO, 2 buffers
  float* sL = reinterpret_cast<float*>(sO + 2 * TILE);  // 2 x 64 (lse * log2e)
  float* sD = sL + 2 * BQ;                              // 2 x 64
  const int nqb = (T + BQ - 1) / BQ;
  const int kb = blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int64_t rs = 3 * int64_t(C);
  const bf16* Qg = qkv + int64_t(b) * T * rs + h * D;
  const bf16* Kg = Qg + C;
  const bf16* Vg = Qg + 2 * C;
  const bf16* Og = dout + int64_t(b) * T * C + h * D;
  const float* Lg = lse + (int64_t(b) * H + h) * T;
  const float* Dg = delta + (int64_t(b) * H + h) * T;
  const float scale = rsqrtf(float(D));
  const float sl2 = scale * kLog2e;

  load_tile(sK, Kg, rs, kb * BKV, T);
  load_tile(sV, Vg, rs, kb * BKV, T);
  auto stage_q = [&](int qb, int buf) {
    load_tile(sQ + buf * TILE, Qg, rs, qb * BQ, T);
    load_tile(sO + buf * TILE, Og, C, qb * BQ, T);
    if (threadIdx.x < BQ) {
      const int q = qb * BQ + threadIdx.x;
      sL[buf * BQ + threadIdx.x] = q < T ? Lg[q] * kLog2e : 0.f;
      sD[buf * BQ + threadIdx.x] = q < T ? Dg[q] : 0.f;
    }
  };
  stage_q(kb, 0);
  cp_commit();

  float dk[8][4], dv[8][4];
  zero(dk);
  zero(dv);
  uint32_t kf[4][4], vf[4][4];
  const int key0 = kb * BKV + warp * 16 + g;  // this thread's keys key0, key0 + 8

  for (int qb = kb; qb < nqb; ++qb) {
    const int buf = (qb - kb) & 1;
    if (qb + 1 < nqb) {
      stage_q(qb + 1, buf ^ 1);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (qb == kb) {
      load_a_frags(sK, warp * 16, kf);
      load_a_frags(sV, warp * 16, vf);
    }
    const bf16* q_t = sQ + buf * TILE;
    const bf16* o_t = sO + buf * TILE;
    const float* L = sL + buf * BQ;
    const float* Dl = sD + buf * BQ;
    float st[8][4], dpt[8][4];  // rows = keys, columns = queries
    zero(st);
    zero(dpt);
    mma_abt(kf, q_t, st);
    mma_abt(vf, o_t, dpt);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qc = nt * 8 + 2 * t4 + (e & 1);
        const int q = qb * BQ + qc;
        const int key = key0 + (e >> 1) * 8;
        float p = exp2f(st[nt][e] * sl2 - L[qc]);
        if (q < key || q >= T || key >= T) p = 0.f;
        st[nt][e] = p;
        dpt[nt][e] = p * (dpt[nt][e] - Dl[qc]);
      }
    mma_pm(st, o_t, dv);   // dV += P^T dO
    mma_pm(dpt, q_t, dk);  // dK += dS^T Q
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int key = key0 + r * 8;
    if (key >= T) continue;
    bf16* drow = dqkv + (int64_t(b) * T + key) * rs + h * D;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      *reinterpret_cast<uint32_t*>(drow + C + nt * 8 + 2 * t4) =
          pack_bf16(dk[nt][2 * r] * scale, dk[nt][2 * r + 1] * scale);
      *reinterpret_cast<uint32_t*>(drow + 2 * C + nt * 8 + 2 * t4) =
          pack_bf16(dv[nt][2 * r], dv[nt][2 * r + 1]);
    }
  }
}

// ------------------------------------------------------------------ backward: dQ
__global__ void __launch_bounds__(128) fa_bwd_dq_kernel(const bf16* __restrict__ dout,
                                                        const bf16* __restrict__ qkv,
                                                        const float* __restrict__ lse,
                                                        const float* __restrict__ delta, int T,
                                                        int C, int H, bf16* __restrict__ dqkv) {
  extern __shared__ __align__(16) uint8_t smraw[];
  bf16* sQ = reinterpret_cast<bf16*>(smraw);
  bf16* sO = sQ + TILE;
  bf16* sK = sO + TILE;      // 2 buffers
  bf16* sV = sK + 2 * TILE;  // 2 buffers
  const int qb = gridDim.x - 1 - blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
  const int64_t rs = 3 * int64_t(C);
  const bf16* Qg = qkv + int64_t(b) * T * rs + h * D;
  const bf16* Kg = Qg + C;
  const bf16* Vg = Qg + 2 * C;
  const bf16* Og = dout + int64_t(b) * T * C + h * D;
  const float scale = rsqrtf(float(D));
  const float sl2 = scale * kLog2e;
  const int q0 = qb * BQ + warp * 16 + g;
  float Lr[2], Dr[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int q = q0 + 8 * r;
    Lr[r] = q < T ? lse[(int64_t(b) * H + h) * T + q] * kLog2e : 0.f;
    Dr[r] = q < T ? delta[(int64_t(b) * H + h) * T + q] : 0.f;
  }

  load_tile(sQ, Qg, rs, qb * BQ, T);
  load_tile(sO, Og, C, qb * BQ, T);
  load_tile(sK, Kg, rs, 0, T);
  load_tile(sV, Vg, rs, 0, T);
  cp_commit();

  float dq[8][4];
  zero(dq);
  uint32_t qf[4][4], of[4][4];
  for (int kb = 0; kb <= qb; ++kb) {
    const int buf = kb & 1;
    if (kb < qb) {
      load_tile(sK + (buf ^ 1) * TILE, Kg, rs, (kb + 1) * BKV, T);
      load_tile(sV + (buf ^ 1) * TILE, Vg, rs, (kb + 1) * BKV, T);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (kb == 0) {
      load_a_frags(sQ, warp * 16, qf);
      load_a_frags(sO, warp * 16, of);
    }
    float s[8][4], dp[8][4];
    zero(s);
    zero(dp);
    mma_abt(qf, sK + buf * TILE, s);
    mma_abt(of, sV + buf * TILE, dp);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kb * BKV + nt * 8 + 2 * t4 + (e & 1);
        const int r = e >> 1;
        const int q = q0 + 8 * r;
        float p = exp2f(s[nt][e] * sl2 - Lr[r]);
        if (key > q || key >= T || q >= T) p = 0.f;
        s[nt][e] = p * (dp[nt][e] - Dr[r]);  // dS
      }
    mma_pm(s, sK + buf * TILE, dq);  // dQ += dS K
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int q = q0 + r * 8;
    if (q >= T) continue;
    bf16* drow = dqkv + (int64_t(b) * T + q) * rs + h * D;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<uint32_t*>(drow + nt * 8 + 2 * t4) =
          pack_bf16(dq[nt][2 * r] * scale, dq[nt][2 * r + 1] * scale);
  }
}

constexpr int kFwdSmem = 5 * TILE * 2;
constexpr int kDkdvSmem = 6 * TILE * 2 + 4 * BQ * 4;
constexpr int kDqSmem = 6 * TILE * 2;

}  // namespace

bool attn_mma_supported(int C, int H) { return C / H == D && C % H == 0 && C % 8 == 0; }

int launch_attn_mma_fwd(const bf16* qkv, int B, int T, int C, int H, bf16* out, float* lse,
                        cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(fa_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFwdSmem);
    attr = true;
  }
  dim3 grid(cdiv(T, BQ), H, B);
  fa_fwd_kernel<<<grid, 128, kFwdSmem, st>>>(qkv, T, C, H, out, lse);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}

int launch_attn_mma_bwd(const bf16* dout, const bf16* qkv, const float* lse, const float* delta,
                        int B, int T, int C, int H, bf16* dqkv, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(fa_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kDkdvSmem);
    cudaFuncSetAttribute(fa_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem);
    attr = true;
  }
  dim3 grid(cdiv(T, BQ), H, B);
  fa_bwd_dkdv_kernel<<<grid, 128, kDkdvSmem, st>>>(dout, qkv, lse, delta, T, C, H, dqkv);
  COUNT_LAUNCH(1);
  fa_bwd_dq_kernel<<<grid, 128, kDqSmem, st>>>(dout, qkv, lse, delta, T, C, H, dqkv);
  COUNT_LAUNCH(1);
  GPT2_LAUNCH_CHECK();
  return GPT2_OK;
}
