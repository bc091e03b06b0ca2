// Causal multi-query attention, bf16 on tensor cores (warp-level
// mma.m16n8k16, fp32 accumulation), tiled so no T x T matrix is ever stored:
// the forward keeps a running max and sum per query row (online softmax) and
// writes the row log-sum-exp; the backward recomputes the probabilities from
// it.  One key/value head serves all H query heads (energyai.berlin page,
// "Multi-Query Attention (MQA)"), so:
//   - forward and dQ: one CTA per (row b, head h, 128-query tile);
//   - dK/dV: one CTA per (row b, 128-key tile) that loops over every head and
//     every later query tile, so the shared head's gradient sums over heads in
//     registers, with no atomics.
// Heaviest tiles (late queries / early keys) are launched first.
//
// Shared-memory tiles are rows of 128 bf16 (256 bytes, 16 chunks of 16 B);
// chunk c of row r is stored at chunk c ^ (r & 7) so ldmatrix reads of 8 rows
// hit 8 distinct bank groups.
#pragma once

#include "common.cuh"

namespace nc {
namespace fa {

constexpr int kD = 128;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// byte offset of (row, 16-byte chunk) in a swizzled tile
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool pred) {
  const int n = pred ? 16 : 0;  // 0 source bytes: the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D += A B, A 16x16 (row), B 16x8 (col), bf16 in, fp32 accumulate
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Copy `rows` rows of 128 bf16 (global row stride ld elements) starting at
// global row g0 into a swizzled tile; rows at or past `limit` are zero-filled.
template <int ROWS, int NT>
__device__ __forceinline__ void load_tile(uint32_t tile, const bf16 *src, int64_t ld, int g0, int limit) {
  constexpr int chunks = ROWS * 16;
  for (int c = threadIdx.x; c < chunks; c += NT) {
    const int r = c >> 4, k = c & 15;
    const int g = g0 + r;
    const bool ok = g < limit;
    cp_async16(tile + swz(r, k), src + (int64_t)(ok ? g : 0) * ld + k * 8, ok);
  }
}

// A fragment (16 rows x 16 k) of a swizzled row tile: rows r0..r0+15, k chunk kc (16 elems)
__device__ __forceinline__ void frag_a(uint32_t tile, int r0, int kc, uint32_t (&a)[4]) {
  const int lane = threadIdx.x & 31;
  const int j = lane >> 3;
  const int row = r0 + (j & 1) * 8 + (lane & 7);
  const int chunk = kc * 2 + (j >> 1);
  ldsm_x4(tile + swz(row, chunk), a[0], a[1], a[2], a[3]);
}
// B fragments for two n-tiles (rows n0..n0+15 of the stored tile are n), k chunk kc:
// b[0],b[1] -> n-tile n0..n0+7; b[2],b[3] -> n0+8..n0+15  (stored [n][k], "col" B)
__device__ __forceinline__ void frag_b_nk(uint32_t tile, int n0, int kc, uint32_t (&b)[4]) {
  const int lane = threadIdx.x & 31;
  const int j = lane >> 3;
  const int row = n0 + (j >> 1) * 8 + (lane & 7);
  const int chunk = kc * 2 + (j & 1);
  ldsm_x4(tile + swz(row, chunk), b[0], b[1], b[2], b[3]);
}
// B fragments for two n-tiles where the stored tile is [k][n] (rows = k):
// k rows k0..k0+15, n columns n0..n0+15 -> b[0],b[1] n-tile n0, b[2],b[3] n-tile n0+8
__device__ __forceinline__ void frag_b_kn(uint32_t tile, int k0, int n0, uint32_t (&b)[4]) {
  const int lane = threadIdx.x & 31;
  const int j = lane >> 3;
  const int row = k0 + (j & 1) * 8 + (lane & 7);
  const int chunk = (n0 >> 3) + (j >> 1);
  ldsm_x4_t(tile + swz(row, chunk), b[0], b[1], b[2], b[3]);
}

// ---------------------------------------------------------------------------
// forward: CTA = 128 queries of one head, 8 warps x 16 rows, keys in tiles of 64
constexpr int kFwdM = 128, kFwdN = 64, kFwdThreads = 256;
constexpr int kFwdSmem = (kFwdM + 4 * kFwdN) * 256;  // Q + 2 stages of K and V

__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const bf16 *__restrict__ qkv, int ld, bf16 *__restrict__ O, float *__restrict__ lse,
                    int T, int H, int n_qt) {
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sQ = smem_addr(sm);
  const uint32_t sK0 = sQ + kFwdM * 256, sV0 = sK0 + 2 * kFwdN * 256;
  const int bid = blockIdx.x;
  const int BH = gridDim.x / n_qt;
  const int qt = n_qt - 1 - bid / BH;  // latest query tiles (most keys) first
  const int h = (bid % BH) % H, b = (bid % BH) / H;
  const int q0 = qt * kFwdM;
  const int C = H * kD;
  const bf16 *base = qkv + (int64_t)b * T * ld;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_kv = (min(q0 + kFwdM, T) + kFwdN - 1) / kFwdN;

  load_tile<kFwdM, kFwdThreads>(sQ, base + h * kD, ld, q0, T);
  load_tile<kFwdN, kFwdThreads>(sK0, base + C, ld, 0, T);
  load_tile<kFwdN, kFwdThreads>(sV0, base + C + kD, ld, 0, T);
  cp_async_commit();

  const float sc = rsqrtf((float)kD) * kLog2e;  // scores in the log2 domain
  float acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int r_lo = q0 + warp * 16 + (lane >> 2);  // this thread's rows r_lo, r_lo + 8
  uint32_t qf[8][4];

  for (int j = 0; j < n_kv; ++j) {
    const int st = j & 1;
    if (j + 1 < n_kv) {
      load_tile<kFwdN, kFwdThreads>(sK0 + (st ^ 1) * kFwdN * 256, base + C, ld, (j + 1) * kFwdN, T);
      load_tile<kFwdN, kFwdThreads>(sV0 + (st ^ 1) * kFwdN * 256, base + C + kD, ld, (j + 1) * kFwdN, T);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) frag_a(sQ, warp * 16, kc, qf[kc]);
    }
    const uint32_t sK = sK0 + st * kFwdN * 256, sV = sV0 + st * kFwdN * 256;
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int t = 0; t < 4; ++t) s[i][t] = 0.f;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bf[4];
        frag_b_nk(sK, np * 16, kc, bf);
        mma16816(s[2 * np], qf[kc], bf[0], bf[1]);
        mma16816(s[2 * np + 1], qf[kc], bf[2], bf[3]);
      }
    }
    const int kv0 = j * kFwdN;
    const bool need_mask = kv0 + kFwdN > q0 || kv0 + kFwdN > T;
    float mx[2] = {m_r[0], m_r[1]};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float v = s[nt][t] * sc;
        if (need_mask) {
          const int col = kv0 + nt * 8 + (lane & 3) * 2 + (t & 1);
          const int row = r_lo + (t >> 1) * 8;
          if (col > row || col >= T) v = -INFINITY;
        }
        s[nt][t] = v;
        mx[t >> 1] = fmaxf(mx[t >> 1], v);
      }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float corr[2], rs[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float base_m = mx[r] == -INFINITY ? 0.f : mx[r];
      corr[r] = fast_exp2(m_r[r] - base_m);
      m_r[r] = mx[r];
      mx[r] = base_m;
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float p = fast_exp2(s[nt][t] - mx[t >> 1]);
        s[nt][t] = p;
        rs[t >> 1] += p;
      }
#pragma unroll
    for (int r = 0; r < 2; ++r) l_r[r] = l_r[r] * corr[r] + rs[r];
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      acc[dt][0] *= corr[0];
      acc[dt][1] *= corr[0];
      acc[dt][2] *= corr[1];
      acc[dt][3] *= corr[1];
    }
    // O += P V : P as A fragments (k = keys), V stored [key][d]
#pragma unroll
    for (int kc = 0; kc < kFwdN / 16; ++kc) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kc][0], s[2 * kc][1]);
      pa[1] = pack_bf16(s[2 * kc][2], s[2 * kc][3]);
      pa[2] = pack_bf16(s[2 * kc + 1][0], s[2 * kc + 1][1]);
      pa[3] = pack_bf16(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        uint32_t bf[4];
        frag_b_kn(sV, kc * 16, dp * 16, bf);
        mma16816(acc[2 * dp], pa, bf[0], bf[1]);
        mma16816(acc[2 * dp + 1], pa, bf[2], bf[3]);
      }
    }
    __syncthreads();  // the stage is refilled by the next iteration's prefetch
  }
  cp_async_wait<0>();
  // finalize: rows r_lo and r_lo + 8
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
  }
  const float inv0 = 1.f / l_r[0], inv1 = 1.f / l_r[1];
  // stage O through shared memory (the Q tile is free) for 16-byte stores
  uint8_t *sO = sm;
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    const int col = dt * 8 + (lane & 3) * 2;
    const int row0 = warp * 16 + (lane >> 2);
    *reinterpret_cast<uint32_t *>(sO + swz(row0, col >> 3) + (col & 7) * 2) = pack_bf16(acc[dt][0] * inv0, acc[dt][1] * inv0);
    *reinterpret_cast<uint32_t *>(sO + swz(row0 + 8, col >> 3) + (col & 7) * 2) = pack_bf16(acc[dt][2] * inv1, acc[dt][3] * inv1);
  }
  if ((lane & 3) == 0) {
    float *L = lse + ((int64_t)b * H + h) * T;
    if (r_lo < T) L[r_lo] = (m_r[0] + __log2f(l_r[0])) * (1.f / kLog2e);
    if (r_lo + 8 < T) L[r_lo + 8] = (m_r[1] + __log2f(l_r[1])) * (1.f / kLog2e);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < kFwdM * 16; c += kFwdThreads) {
    const int r = c >> 4, k = c & 15;
    const int g = q0 + r;
    if (g < T)
      *reinterpret_cast<uint4 *>(O + ((int64_t)b * T + g) * C + h * kD + k * 8) =
          *reinterpret_cast<const uint4 *>(sO + swz(r, k));
  }
}

// ---------------------------------------------------------------------------
// dQ: CTA = 128 queries of one head; recompute P from the saved lse, then
//   dS = P (dO V^T - D),  dQ = dS K / sqrt(d)
constexpr int kDqM = 128, kDqN = 64, kDqThreads = 256;
constexpr int kDqSmem = (2 * kDqM + 4 * kDqN) * 256;  // Q, dO, 2 stages of K and V

__global__ void __launch_bounds__(kDqThreads, 1)
    attn_bwd_dq_kernel(const bf16 *__restrict__ qkv, int ld, const bf16 *__restrict__ dO,
                       const float *__restrict__ lse, const float *__restrict__ Drow,
                       bf16 *__restrict__ dqkv, int T, int H, int n_qt) {
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sQ = smem_addr(sm), sG = sQ + kDqM * 256;
  const uint32_t sK0 = sG + kDqM * 256, sV0 = sK0 + 2 * kDqN * 256;
  const int bid = blockIdx.x;
  const int BH = gridDim.x / n_qt;
  const int qt = n_qt - 1 - bid / BH;
  const int h = (bid % BH) % H, b = (bid % BH) / H;
  const int q0 = qt * kDqM;
  const int C = H * kD;
  const bf16 *base = qkv + (int64_t)b * T * ld;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_kv = (min(q0 + kDqM, T) + kDqN - 1) / kDqN;

  load_tile<kDqM, kDqThreads>(sQ, base + h * kD, ld, q0, T);
  load_tile<kDqM, kDqThreads>(sG, dO + (int64_t)b * T * C + h * kD, C, q0, T);
  load_tile<kDqN, kDqThreads>(sK0, base + C, ld, 0, T);
  load_tile<kDqN, kDqThreads>(sV0, base + C + kD, ld, 0, T);
  cp_async_commit();

  const float sc = rsqrtf((float)kD) * kLog2e;
  const int r_lo = q0 + warp * 16 + (lane >> 2);
  float Lr[2], Dr[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = min(r_lo + 8 * r, T - 1);
    Lr[r] = lse[((int64_t)b * H + h) * T + row] * kLog2e;
    Dr[r] = Drow[((int64_t)b * H + h) * T + row];
  }
  float dq[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int t = 0; t < 4; ++t) dq[i][t] = 0.f;

  for (int j = 0; j < n_kv; ++j) {
    const int st = j & 1;
    if (j + 1 < n_kv) {
      load_tile<kDqN, kDqThreads>(sK0 + (st ^ 1) * kDqN * 256, base + C, ld, (j + 1) * kDqN, T);
      load_tile<kDqN, kDqThreads>(sV0 + (st ^ 1) * kDqN * 256, base + C + kD, ld, (j + 1) * kDqN, T);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sK = sK0 + st * kDqN * 256, sV = sV0 + st * kDqN * 256;
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int t = 0; t < 4; ++t) { s[i][t] = 0.f; dp[i][t] = 0.f; }
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      uint32_t qa[4], ga[4];
      frag_a(sQ, warp * 16, kc, qa);
      frag_a(sG, warp * 16, kc, ga);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t kb[4], vb[4];
        frag_b_nk(sK, np * 16, kc, kb);
        frag_b_nk(sV, np * 16, kc, vb);
        mma16816(s[2 * np], qa, kb[0], kb[1]);
        mma16816(s[2 * np + 1], qa, kb[2], kb[3]);
        mma16816(dp[2 * np], ga, vb[0], vb[1]);
        mma16816(dp[2 * np + 1], ga, vb[2], vb[3]);
      }
    }
    const int kv0 = j * kDqN;
    const bool need_mask = kv0 + kDqN > q0 || kv0 + kDqN > T;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float p = fast_exp2(s[nt][t] * sc - Lr[t >> 1]);
        if (need_mask) {
          const int col = kv0 + nt * 8 + (lane & 3) * 2 + (t & 1);
          const int row = r_lo + (t >> 1) * 8;
          if (col > row || col >= T) p = 0.f;
        }
        s[nt][t] = p * (dp[nt][t] - Dr[t >> 1]);  // dS
      }
    // dQ += dS K : dS as A fragments (k = keys), K stored [key][d]
#pragma unroll
    for (int kc = 0; kc < kDqN / 16; ++kc) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kc][0], s[2 * kc][1]);
      pa[1] = pack_bf16(s[2 * kc][2], s[2 * kc][3]);
      pa[2] = pack_bf16(s[2 * kc + 1][0], s[2 * kc + 1][1]);
      pa[3] = pack_bf16(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
      for (int dpp = 0; dpp < 8; ++dpp) {
        uint32_t bf[4];
        frag_b_kn(sK, kc * 16, dpp * 16, bf);
        mma16816(dq[2 * dpp], pa, bf[0], bf[1]);
        mma16816(dq[2 * dpp + 1], pa, bf[2], bf[3]);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  const float scale = rsqrtf((float)kD);
  uint8_t *sO = sm;  // reuse the Q tile
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    const int col = dt * 8 + (lane & 3) * 2;
    const int row0 = warp * 16 + (lane >> 2);
    *reinterpret_cast<uint32_t *>(sO + swz(row0, col >> 3) + (col & 7) * 2) = pack_bf16(dq[dt][0] * scale, dq[dt][1] * scale);
    *reinterpret_cast<uint32_t *>(sO + swz(row0 + 8, col >> 3) + (col & 7) * 2) = pack_bf16(dq[dt][2] * scale, dq[dt][3] * scale);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < kDqM * 16; c += kDqThreads) {
    const int r = c >> 4, k = c & 15;
    const int g = q0 + r;
    if (g < T)
      *reinterpret_cast<uint4 *>(dqkv + ((int64_t)b * T + g) * ld + h * kD + k * 8) =
          *reinterpret_cast<const uint4 *>(sO + swz(r, k));
  }
}

// ---------------------------------------------------------------------------
// dK, dV: CTA = 128 keys (8 warps x 16 keys), loop over heads and query tiles
// of 32 at or after the keys; transposed products keep keys as the row index:
//   S^T = K Q^T, P^T = exp(S^T - lse_q), dV += P^T dO,
//   dP^T = V dO^T, dS^T = P^T (dP^T - D_q), dK += dS^T Q / sqrt(d)
constexpr int kKvN = 128, kKvM = 32, kKvThreads = 256;
constexpr int kKvSmem = (2 * kKvN + 4 * kKvM) * 256 + 2 * 2 * kKvM * 4;

__global__ void __launch_bounds__(kKvThreads, 1)
    attn_bwd_dkdv_kernel(const bf16 *__restrict__ qkv, int ld, const bf16 *__restrict__ dO,
                         const float *__restrict__ lse, const float *__restrict__ Drow,
                         bf16 *__restrict__ dqkv, int T, int H, int n_kt) {
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sK = smem_addr(sm), sV = sK + kKvN * 256;
  const uint32_t sQ0 = sV + kKvN * 256, sG0 = sQ0 + 2 * kKvM * 256;
  float *sL = reinterpret_cast<float *>(sm + (2 * kKvN + 4 * kKvM) * 256);  // [2][kKvM]
  float *sD = sL + 2 * kKvM;                                                // [2][kKvM]
  const int bid = blockIdx.x;
  const int Bn = gridDim.x / n_kt;
  const int kt = bid / Bn;  // key tile 0 has the most work: launched first
  const int b = bid % Bn;
  const int k0 = kt * kKvN;
  const int C = H * kD;
  const bf16 *base = qkv + (int64_t)b * T * ld;
  const bf16 *gbase = dO + (int64_t)b * T * C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int first_qt = k0 / kKvM;
  const int n_q = (T + kKvM - 1) / kKvM - first_qt;  // query tiles per head
  const int n_it = n_q * H;

  load_tile<kKvN, kKvThreads>(sK, base + C, ld, k0, T);
  load_tile<kKvN, kKvThreads>(sV, base + C + kD, ld, k0, T);
  auto prefetch = [&](int it, int st) {
    const int h = it / n_q, q0 = (first_qt + it % n_q) * kKvM;
    load_tile<kKvM, kKvThreads>(sQ0 + st * kKvM * 256, base + h * kD, ld, q0, T);
    load_tile<kKvM, kKvThreads>(sG0 + st * kKvM * 256, gbase + h * kD, C, q0, T);
    if (threadIdx.x < kKvM) {
      const int q = min(q0 + (int)threadIdx.x, T - 1);
      sL[st * kKvM + threadIdx.x] = lse[((int64_t)b * H + h) * T + q] * kLog2e;
      sD[st * kKvM + threadIdx.x] = Drow[((int64_t)b * H + h) * T + q];
    }
  };
  prefetch(0, 0);
  cp_async_commit();

  const float sc = rsqrtf((float)kD) * kLog2e;
  const int key_lo = k0 + warp * 16 + (lane >> 2);  // this thread's keys key_lo, key_lo + 8
  float dk[16][4], dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int t = 0; t < 4; ++t) { dk[i][t] = 0.f; dv[i][t] = 0.f; }

  for (int it = 0; it < n_it; ++it) {
    const int st = it & 1;
    if (it + 1 < n_it) prefetch(it + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int q0 = (first_qt + it % n_q) * kKvM;
    const uint32_t sQ = sQ0 + st * kKvM * 256, sG = sG0 + st * kKvM * 256;
    const float *Ls = sL + st * kKvM, *Ds = sD + st * kKvM;
    float s[4][4], dp[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < 4; ++t) { s[i][t] = 0.f; dp[i][t] = 0.f; }
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      uint32_t ka[4], va[4];
      frag_a(sK, warp * 16, kc, ka);
      frag_a(sV, warp * 16, kc, va);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t qb[4], gb[4];
        frag_b_nk(sQ, np * 16, kc, qb);
        frag_b_nk(sG, np * 16, kc, gb);
        mma16816(s[2 * np], ka, qb[0], qb[1]);
        mma16816(s[2 * np + 1], ka, qb[2], qb[3]);
        mma16816(dp[2 * np], va, gb[0], gb[1]);
        mma16816(dp[2 * np + 1], va, gb[2], gb[3]);
      }
    }
    const bool need_mask = q0 < k0 + kKvN || q0 + kKvM > T;
    float ps[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int qi = nt * 8 + (lane & 3) * 2 + (t & 1);  // query within the tile
        float p = fast_exp2(s[nt][t] * sc - Ls[qi]);
        if (need_mask) {
          const int key = key_lo + (t >> 1) * 8;
          if (q0 + qi < key || q0 + qi >= T) p = 0.f;
        }
        ps[nt][t] = p;
        s[nt][t] = p * (dp[nt][t] - Ds[qi]);  // dS^T
      }
    // dV += P^T dO, dK += dS^T Q : A from registers (k = queries), B stored [query][d]
#pragma unroll
    for (int kc = 0; kc < kKvM / 16; ++kc) {
      uint32_t pa[4], sa[4];
      pa[0] = pack_bf16(ps[2 * kc][0], ps[2 * kc][1]);
      pa[1] = pack_bf16(ps[2 * kc][2], ps[2 * kc][3]);
      pa[2] = pack_bf16(ps[2 * kc + 1][0], ps[2 * kc + 1][1]);
      pa[3] = pack_bf16(ps[2 * kc + 1][2], ps[2 * kc + 1][3]);
      sa[0] = pack_bf16(s[2 * kc][0], s[2 * kc][1]);
      sa[1] = pack_bf16(s[2 * kc][2], s[2 * kc][3]);
      sa[2] = pack_bf16(s[2 * kc + 1][0], s[2 * kc + 1][1]);
      sa[3] = pack_bf16(s[2 * kc + 1][2], s[2 * kc + 1][3]);
#pragma unroll
      for (int dpp = 0; dpp < 8; ++dpp) {
        uint32_t gb[4], qb[4];
        frag_b_kn(sG, kc * 16, dpp * 16, gb);
        frag_b_kn(sQ, kc * 16, dpp * 16, qb);
        mma16816(dv[2 * dpp], pa, gb[0], gb[1]);
        mma16816(dv[2 * dpp + 1], pa, gb[2], gb[3]);
        mma16816(dk[2 * dpp], sa, qb[0], qb[1]);
        mma16816(dk[2 * dpp + 1], sa, qb[2], qb[3]);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  const float scale = rsqrtf((float)kD);
  uint8_t *sO = sm;  // K then V tiles are free: dk into the first, dv into the second
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    const int col = dt * 8 + (lane & 3) * 2;
    const int row0 = warp * 16 + (lane >> 2);
    *reinterpret_cast<uint32_t *>(sO + swz(row0, col >> 3) + (col & 7) * 2) = pack_bf16(dk[dt][0] * scale, dk[dt][1] * scale);
    *reinterpret_cast<uint32_t *>(sO + swz(row0 + 8, col >> 3) + (col & 7) * 2) = pack_bf16(dk[dt][2] * scale, dk[dt][3] * scale);
    *reinterpret_cast<uint32_t *>(sO + kKvN * 256 + swz(row0, col >> 3) + (col & 7) * 2) = pack_bf16(dv[dt][0], dv[dt][1]);
    *reinterpret_cast<uint32_t *>(sO + kKvN * 256 + swz(row0 + 8, col >> 3) + (col & 7) * 2) = pack_bf16(dv[dt][2], dv[dt][3]);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < kKvN * 16; c += kKvThreads) {
    const int r = c >> 4, k = c & 15;
    const int g = k0 + r;
    if (g < T) {
      bf16 *row = dqkv + ((int64_t)b * T + g) * ld + C;
      *reinterpret_cast<uint4 *>(row + k * 8) = *reinterpret_cast<const uint4 *>(sO + swz(r, k));
      *reinterpret_cast<uint4 *>(row + kD + k * 8) = *reinterpret_cast<const uint4 *>(sO + kKvN * 256 + swz(r, k));
    }
  }
}

inline cudaError_t attn_mma_init() {
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFwdSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem);
  return e;
}

// rows must be 16-byte aligned: ld a multiple of 8 and 16-byte aligned bases
inline bool supported(const void *qkv, int ld, const void *O) {
  return (ld % 8) == 0 && ((uintptr_t)qkv & 15) == 0 && ((uintptr_t)O & 15) == 0;
}

inline cudaError_t launch_fwd(const bf16 *qkv, int ld, bf16 *O, float *lse, int B, int T, int H,
                              cudaStream_t st) {
  const int n_qt = (T + kFwdM - 1) / kFwdM;
  attn_fwd_kernel<<<B * H * n_qt, kFwdThreads, kFwdSmem, st>>>(qkv, ld, O, lse, T, H, n_qt);
  return cudaGetLastError();
}

inline cudaError_t launch_bwd(const bf16 *qkv, int ld, const bf16 *dO, const float *lse,
                              const float *Drow, bf16 *dqkv, int B, int T, int H, cudaStream_t st) {
  const int n_qt = (T + kDqM - 1) / kDqM;
  attn_bwd_dq_kernel<<<B * H * n_qt, kDqThreads, kDqSmem, st>>>(qkv, ld, dO, lse, Drow, dqkv, T, H, n_qt);
  const int n_kt = (T + kKvN - 1) / kKvN;
  attn_bwd_dkdv_kernel<<<B * n_kt, kKvThreads, kKvSmem, st>>>(qkv, ld, dO, lse, Drow, dqkv, T, H, n_kt);
  return cudaGetLastError();
}

}  // namespace fa
}  // namespace nc
