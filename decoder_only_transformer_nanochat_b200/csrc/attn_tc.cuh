// Causal multi-query attention on the 5th-generation tensor cores, forward
// and backward (energyai.berlin page, "Multi-Query Attention (MQA)": one
// key/value head shared by the H query heads; scores q.k / sqrt(128), keys
// j <= i).
//
// Forward: CTA = 128 queries of one (row b, head h); keys in tiles of 128.
//   warp 0      TMA: Q once, then K (3-stage ring) and V (2-stage ring) tiles
//   warp 1      MMA: S_j = Q K_j^T into one of two TMEM score tiles,
//               O += P_j V_j into a TMEM accumulator with P_j read from TMEM
//   warps 2..9  softmax, two warps per query row (64 keys each): S row out of
//               TMEM, running max / sum, P_j as bf16 pairs back into one of two
//               TMEM P buffers, O rescaled in TMEM only when the row max grows
//               by more than 2^8 (the exponent base may lag the true max by up
//               to 8 in the log2 domain, which changes no result: P and the sum
//               carry the same factor)
// S_{j+1} is issued before P_j is ready, so the tensor core works on the next
// scores while the softmax warps finish the current tile.
//
// Operands, all bf16 with 128-byte swizzle: Q, K as K-major (d contiguous)
// tiles of 2 boxes [64 d x 128 rows]; V as an MN-major B operand (d
// contiguous) of 4 boxes [64 d x 64 keys].  The backward kernels further down
// are described where they start.
#pragma once

#include <stdio.h>

#include <atomic>

#include "tc_common.cuh"

namespace nc {
namespace fatc {

using namespace tc;

constexpr int kQ = 128, kKV = 128, kD = 128;
constexpr int kFwdThreads = 320;  // TMA warp, MMA warp, 8 softmax warps
constexpr int kTileBytes = kQ * kD * 2;      // 32 KB: Q, K, V or P tile
constexpr int kKStages = 3, kVStages = 2;
constexpr int kSmem = 1024 + kTileBytes /*Q*/ + (kKStages + kVStages) * kTileBytes + 256 + 3072;
constexpr int kTmemCols = 512;               // S0 [0,128), S1 [128,256), O [256,384), P0 [384,448), P1 [448,512)
constexpr int kPCol = 384;                   // P_j as bf16 pairs: key k of row m at lane m, column kPCol + 64 (j&1) + k/2
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for x in [-126, 0] on the FMA pipe: x = n + f with n = round(x) (the
// 1.5 * 2^23 shifter), f in [-1/2, 1/2], 2^f by a cubic whose coefficients
// were fitted here to the relative error (max 1.0e-4, far below the bf16
// rounding of a probability); n goes straight into the exponent bits.
// Used for half of the softmax exponentials so the MUFU unit does not
// bound the tile.
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  const int n = __float_as_int(t) - 0x4B400000;
  const float p = fmaf(f, fmaf(f, fmaf(f, 0.05500858f, 0.24221037f), 0.69328290f), 1.f);
  return __int_as_float(__float_as_int(p) + (n << 23));
}

// The same for a pair of exponents in f32x2 form (bit-identical to two
// ex2_poly calls): with t = x + 1.5 * 2^23, (t's bits << 23) is n << 23
// modulo 2^32, since 0x4B400000 << 23 vanishes there.
__device__ __forceinline__ void ex2_poly2(uint64_t x, float &e0, float &e1) {
  float x0, x1;
  f2split(x, x0, x1);
  const uint64_t xc = f2(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = add2(xc, f2(12582912.f, 12582912.f));
  const uint64_t u = add2(t, f2(-12582912.f, -12582912.f));
  const uint64_t f = fma2(u, f2(-1.f, -1.f), xc);
  uint64_t q = fma2(f, f2(0.05500858f, 0.05500858f), f2(0.24221037f, 0.24221037f));
  q = fma2(f, q, f2(0.69328290f, 0.69328290f));
  q = fma2(f, q, f2(1.f, 1.f));
  float p0, p1, t0, t1;
  f2split(q, p0, p1);
  f2split(t, t0, t1);
  e0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  e1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// MMA with the A operand read from TMEM (K-major, bf16 pairs per column)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// AND over the 256 element-wise threads (named barrier 1), so that all of
// them take the same branch and keep meeting at the same barriers
__device__ __forceinline__ bool epi_vote_all256(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 256, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v)
      : "memory");
  return out != 0;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// bf16 row r of a K-major 128-byte-swizzled [rows x 128] tile made of two
// 64-column blocks: 16-byte unit u (columns 8u..8u+7) of row r.
__device__ __forceinline__ uint32_t tile_unit(int r, int u) {
  return (uint32_t)((u >> 3) * (kQ * 128) + r * 128 + (((u & 7) ^ (r & 7)) << 4));
}

struct FwdParams {
  int T, H, n_qt, B;
  int window;   // windowed kernels: query i sees keys j with 0 <= i - j < window
  float *lse;   // [B, H, T]
  int *status;
};

// kWin: sliding-window variant (compiled separately, so the plain causal
// kernel is unchanged by it): key tiles start at the window's first tile and
// keys more than window - 1 before the query are masked.
template <bool kWin>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_qk,   // qkv [B][T][ld], box 64 x 128
                       const __grid_constant__ CUtensorMap map_v,    // qkv, box 64 x 64
                       const __grid_constant__ CUtensorMap map_o,    // O [B][T][C], box 64 x 128
                       const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sK = sQ + kTileBytes;                  // K ring: kKStages tiles
  uint8_t *sV = sK + kKStages * kTileBytes;       // V ring: kVStages tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(sV + kVStages * kTileBytes);
  // bars: q_full, k_full[3], k_empty[3], s_full[2], s_empty[2], p_full[2], drain,
  //       v_full[2], v_empty[2], o_done[2].  K and V have rings of their own: K_j is
  //       free as soon as S_j is computed, so the loads of K_{j+2}, K_{j+3} overlap
  //       softmax j.  P has two TMEM buffers: P_{j+1} is written while P_j V_j runs.
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 20);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t q_full = smem_u32(bars + 0);
  auto k_full = [&](int s) { return smem_u32(bars + 1 + s); };
  auto k_empty = [&](int s) { return smem_u32(bars + 4 + s); };
  auto s_full = [&](int s) { return smem_u32(bars + 7 + s); };
  auto s_empty = [&](int s) { return smem_u32(bars + 9 + s); };
  auto p_full = [&](int s) { return smem_u32(bars + 11 + s); };
  const uint32_t drain = smem_u32(bars + 13);
  auto v_full = [&](int s) { return smem_u32(bars + 14 + s); };
  auto v_empty = [&](int s) { return smem_u32(bars + 16 + s); };
  auto o_done = [&](int s) { return smem_u32(bars + 18 + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = gridDim.x / p.n_qt;
  const int qt = p.n_qt - 1 - (int)blockIdx.x / BH;  // latest query tiles (most keys) first
  const int h = ((int)blockIdx.x % BH) % p.H, b = ((int)blockIdx.x % BH) / p.H;
  const int q0 = qt * kQ;
  const int kt_lo = kWin ? max(0, q0 - p.window + 1) / kKV : 0;   // first key tile any query here sees
  const int n_kv = (min(q0 + kQ, p.T) + kKV - 1) / kKV - kt_lo;   // key tiles visited (qt + 1 when causal)
  const int kbase = kt_lo * kKV;                                  // first key of tile j = kbase + j * kKV
  const int C = p.H * kD;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(s_empty(s), 256);
      mbar_init(p_full(s), 256);
      mbar_init(o_done(s), 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      mbar_expect_tx(q_full, kTileBytes);
      for (int i = 0; i < 2; ++i) tma_load_3d(smem_u32(sQ) + i * 16384, &map_qk, h * kD + 64 * i, q0, b, q_full);
      int issued_k = 0, issued_v = 0;
      auto load_k = [&](int j) -> bool {
        const int st = j % kKStages;
        if (!mbar_wait(k_empty(st), ((j / kKStages) & 1) ^ 1, abort_flag, p.status)) return false;
        const uint32_t k_dst = smem_u32(sK) + st * kTileBytes;
        mbar_expect_tx(k_full(st), kTileBytes);
        for (int i = 0; i < 2; ++i) tma_load_3d(k_dst + i * 16384, &map_qk, C + 64 * i, kbase + j * kKV, b, k_full(st));
        ++issued_k;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(v_empty(st), ((j >> 1) & 1) ^ 1, abort_flag, p.status)) return false;
        const uint32_t v_dst = smem_u32(sV) + st * kTileBytes;
        mbar_expect_tx(v_full(st), kTileBytes);
        for (int hh = 0; hh < 2; ++hh)
          for (int a = 0; a < 2; ++a)
            tma_load_3d(v_dst + hh * 16384 + a * 8192, &map_v, C + kD + 64 * a, kbase + j * kKV + 64 * hh, b,
                        v_full(st));
        ++issued_v;
        return true;
      };
      // K runs two tiles ahead of V: K_{j+2} is requested before V_j
      bool okp = load_k(0) && (n_kv < 2 || load_k(1));
      for (int j = 0; j < n_kv && okp; ++j) {
        if (j + 2 < n_kv && !load_k(j + 2)) break;
        if (!load_v(j)) break;
      }
      // no copy of ours may still be landing when the CTA exits
      const uint64_t t0 = globaltimer();
      while (!mbar_try(q_full, 0) && globaltimer() - t0 < kWaitNs) {}
      for (int j = max(0, issued_k - kKStages); j < issued_k; ++j) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(k_full(j % kKStages), (j / kKStages) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
      for (int j = max(0, issued_v - 2); j < issued_v; ++j) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(v_full(j & 1), (j >> 1) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc_s = make_idesc(0, 0, kQ, kKV);   // Q K^T: both K-major
      const uint32_t idesc_o = make_idesc(0, 1, kQ, kD);    // P V: V is MN-major
      // Descriptors built once; (byte offset >> 4) added moves the start
      // address (no carry: shared addresses are below 2^18).
      const uint64_t dQd = smem_desc(smem_u32(sQ), 16, 1024), dKd = smem_desc(smem_u32(sK), 16, 1024);
      const uint64_t dVd = smem_desc(smem_u32(sV), 8192, 1024);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1, ks = j % kKStages;
        if (!mbar_wait(k_full(ks), (j / kKStages) & 1, abort_flag, p.status)) return false;
        if (!mbar_wait(s_empty(st), ((j >> 1) & 1) ^ 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint64_t bK = dKd + (uint64_t)((ks * kTileBytes) >> 4);
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
          const uint32_t off = ((s >> 2) * 16384 + (s & 3) * 32) >> 4;
          tc_mma(tmem + st * kKV, dQd + off, bK + off, idesc_s, s > 0 ? 1u : 0u);
        }
        tc_commit(s_full(st));
        tc_commit(k_empty(ks));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv && !issue_s(j + 1)) break;
        if (!mbar_wait(p_full(j & 1), (j >> 1) & 1, abort_flag, p.status)) break;
        if (!mbar_wait(v_full(j & 1), (j >> 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint64_t bV = dVd + (uint64_t)(((j & 1) * kTileBytes) >> 4);
        const uint32_t a_p = tmem + kPCol + 64 * (j & 1);
#pragma unroll
        for (int s = 0; s < kKV / 16; ++s) {
          const uint32_t b_off = ((s >> 2) * 16384 + (s & 3) * 2048) >> 4;  // V: MN-major, k rows
          // P from TMEM: 16 keys = 8 columns of bf16 pairs
          tc_mma_ts(tmem + 2 * kKV, a_p + 8 * s, bV + b_off, idesc_o, (j > 0 || s > 0) ? 1u : 0u);
        }
        tc_commit(o_done(j & 1));
        tc_commit(v_empty(j & 1));
      }
      tc_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try(drain, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ---------------- softmax warps 2..9: thread = query row, key half g ----------------
    // warps w and w + 4 share TMEM lane quarter (w & 3); warpgroup g = (w - 2) / 4
    // takes keys [64g, 64g + 64) of each tile and the same half of O's columns
    const int quarter = warp & 3, g = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int row = q0 + r;
    const int c0 = 64 * g;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    float *sMax = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + 256);  // [2 tiles][2 halves][128]
    float *sSum = sMax + 2 * 2 * kQ;                                                   // [2 halves][128]
    const float sc = rsqrtf((float)kD) * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j & 1;
      ok = mbar_wait(s_full(st), (j >> 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; }
      float s[64];
      if (ok) {
        tc_fence_after();
        uint32_t rr[2][32];
        tmem_ld32_nw(lane_base + st * kKV + c0, rr[0]);
        tmem_ld32_nw(lane_base + st * kKV + c0 + 32, rr[1]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(rr[c][i]) * sc;
        tc_fence_before();
        mbar_arrive(s_empty(st));
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = 0.f;
      }
      const int kv0 = kbase + j * kKV + c0;
      if (kv0 + 64 > q0 || kv0 + 64 > p.T || (kWin && kv0 <= q0 + kQ - 1 - p.window)) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (kv0 + i > row || kv0 + i >= p.T || (kWin && row - (kv0 + i) >= p.window)) s[i] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) mx = fmaxf(mx, s[i]);
      // the row max over both halves: exchange through shared memory (buffer j & 1)
      sMax[(st * 2 + g) * kQ + r] = mx;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      mx = fmaxf(sMax[(st * 2) * kQ + r], sMax[(st * 2 + 1) * kQ + r]);
      // every softmax warp learns whether any of them gave up; all take the same branch
      ok = epi_vote_all256(ok);
      if (!ok) break;
      // the exponent base for this tile; it only moves when the max grows by > 2^8
      const bool grow = j == 0 || mx > m_used + kRescaleLog2;
      const float corr = (j > 0 && grow) ? ex2(m_used - mx) : 1.f;
      if (grow) {
        l *= corr;
        m_used = mx;
      }
      // with a window a row may see no key of its first tile: its base stays
      // -inf there and its exponentials are taken against 0 (all of them 0)
      const float mb = (kWin && m_used == -INFINITY) ? 0.f : m_used;
      // P_j in registers first: the exponentials overlap the previous P V
      float sum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        // one exponential in four on the FMA pipe: measured fastest (half makes
        // the loop issue-bound, none leaves it MUFU-bound)
        const float e0 = ex2(s[i] - mb);
        const float e1 = (i & 2) ? ex2_poly(s[i + 1] - mb) : ex2(s[i + 1] - mb);
        sum += e0 + e1;
        pk[i / 2] = pack2(e0, e1);
      }
      // P_j goes to buffer j & 1 once P_{j-2} V_{j-2} has read it; a rescale of
      // O (rare: the base moves only when the max grows by more than 2^8) needs
      // P_{j-1} V_{j-1} done as well
      if (j > 0) {
        const bool rescale = __any_sync(0xffffffffu, grow);
        if (rescale) ok = mbar_wait(o_done((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, p.status);
        else if (j >= 2) ok = mbar_wait(o_done(j & 1), ((j >> 1) & 1) ^ 1, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, ok)) ok = false;
        ok = epi_vote_all256(ok);
        if (!ok) break;
        tc_fence_after();
        if (rescale) {
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t rr[32];
            tmem_ld32(lane_base + 2 * kKV + c0 + c * 32, rr);
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * corr);
            tmem_st32(lane_base + 2 * kKV + c0 + c * 32, rr);
          }
        }
      }
      tmem_st32(lane_base + kPCol + 64 * (j & 1) + 32 * g, pk);  // keys [64g, 64g + 64) of this row
      l += sum;
      tc_fence_before();
      mbar_arrive(p_full(j & 1));
    }
    // ---------------- epilogue: O / l, lse ----------------
    if (ok) ok = mbar_wait(o_done((n_kv - 1) & 1), ((n_kv - 1) >> 1) & 1, abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    sSum[g * kQ + r] = l;
    ok = epi_vote_all256(ok);
    const float lt = sSum[r] + sSum[kQ + r];
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / lt;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + 2 * kKV + c0 + c * 32, rr);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack2(__uint_as_float(rr[8 * u + 0]) * inv, __uint_as_float(rr[8 * u + 1]) * inv);
          w.y = pack2(__uint_as_float(rr[8 * u + 2]) * inv, __uint_as_float(rr[8 * u + 3]) * inv);
          w.z = pack2(__uint_as_float(rr[8 * u + 4]) * inv, __uint_as_float(rr[8 * u + 5]) * inv);
          w.w = pack2(__uint_as_float(rr[8 * u + 6]) * inv, __uint_as_float(rr[8 * u + 7]) * inv);
          *reinterpret_cast<uint4 *>(sQ + tile_unit(r, 8 * g + c * 4 + u)) = w;  // Q is no longer read
        }
      }
      if (g == 0 && row < p.T) p.lse[((int64_t)b * p.H + h) * p.T + row] = (m_used + __log2f(lt)) * (1.f / kLog2e);
    }
    fence_proxy_async();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ok && warp == 2 && lane == 0) {
      for (int i = 0; i < 2; ++i) tma_store_3d(&map_o, smem_u32(sQ) + i * 16384, h * kD + 64 * i, q0, b);
      bulk_commit();
      bulk_wait0();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------- forward, ping-pong: two softmax warpgroups on alternating key tiles ----------------
// Work item = 128 queries of one (row b, head h); operand layouts as above.
//   warp 0      TMA: Q of each item (two buffers: the next item's Q lands
//               while the current one runs), K and V rings of two tiles
//   warp 1      MMA: S_j = Q K_j^T into TMEM buffer j & 1, P_j written back
//               over S_j as bf16 pairs, O_{j&1} += P_j V_j; tensor-core order
//               S_0, S_1, PV_0, S_2, PV_1, S_3 ... (MMAs issued by one thread
//               run in order, so S_{j+2} overwrites P_j only after PV_j read it)
//   warps 4..7  softmax of the even key tiles, warps 8..11 of the odd ones;
//               thread = query row, the whole 128-key tile of its row in
//               registers, its own running max and sum (no exchange between
//               threads, no block-wide barrier inside the key loop)
// TMEM: S/P_0 [0,128), S/P_1 [128,256), O_0 [256,384), O_1 [384,512).
// The two partial outputs are merged once at the end:
//   m = max(m_0, m_1),  a_g = 2^(m_g - m),
//   O = (a_0 O_0 + a_1 O_1) / (a_0 l_0 + a_1 l_1),  lse = m + log2(a_0 l_0 + a_1 l_1)
// (log2 domain), the online-softmax merge of two disjoint key sets.  The
// commit that signals S_j covers every earlier MMA, so a group that rescales
// its O on a grown max finds its previous P V already complete.
// Persistent: CTA c takes items c, c + grid, c + 2 grid, ... (items ordered
// latest query tiles first, the most keys), so the next item's Q load and
// first score MMAs overlap the current item's merge and store; with grid =
// the item count every CTA takes one item.  Barrier phases count uses across
// items: a group's tiles for s_full, p_full and o_done, the K and V loads for
// their rings, the items for the Q buffers and o_free (the merge has read O).
constexpr int kPpOCol = 256;  // O_g at kPpOCol + 128 g
constexpr int kPpStages = 2;  // K and V ring depth (with two Q buffers: six tiles of 32 KB)
// Three warpgroups: warp 0 TMA, warp 1 MMA (warps 2, 3 idle), warps 4..7 and
// 8..11 the two softmax groups.  The first warpgroup gives registers to the
// other two (setmaxnreg): 128 x 56 + 256 x 224 = 64,512, all of the 384 x 168
// the CTA is launched with, so every increase can be met.
constexpr int kPpThreads = 384;
constexpr int kPpRegsLow = 56, kPpRegsHigh = 224;
static_assert(128 * kPpRegsLow + 256 * kPpRegsHigh <= kPpThreads * 168, "register split within the launch");
// engine 0 runs this kernel when true, the one above when false (engine 2 the other)
constexpr bool kFwdPingPongDefault = true;

template <bool kWin>
__global__ void __launch_bounds__(kPpThreads, 1)
    attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap map_qk,   // qkv [B][T][ld], box 64 x 128
                       const __grid_constant__ CUtensorMap map_v,    // qkv, box 64 x 64
                       const __grid_constant__ CUtensorMap map_o,    // O [B][T][C], box 64 x 128
                       const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;                              // two Q buffers; an item's output is staged in its own
  uint8_t *sK = sQ + 2 * kTileBytes;
  uint8_t *sV = sK + kPpStages * kTileBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sV + kPpStages * kTileBytes);
  // bars: q_full[2], q_empty[2], k_full[2], k_empty[2], v_full[2], v_empty[2],
  //       s_full[2], p_full[2], o_done[2], o_free, drain
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 24);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *sML = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + 256);  // [group][m, l][128]
  auto q_full = [&](int s) { return smem_u32(bars + 0 + s); };
  auto q_empty = [&](int s) { return smem_u32(bars + 2 + s); };
  auto k_full = [&](int s) { return smem_u32(bars + 4 + s); };
  auto k_empty = [&](int s) { return smem_u32(bars + 6 + s); };
  auto v_full = [&](int s) { return smem_u32(bars + 8 + s); };
  auto v_empty = [&](int s) { return smem_u32(bars + 10 + s); };
  auto s_full = [&](int s) { return smem_u32(bars + 12 + s); };
  auto p_full = [&](int s) { return smem_u32(bars + 14 + s); };
  auto o_done = [&](int s) { return smem_u32(bars + 16 + s); };
  const uint32_t o_free = smem_u32(bars + 18);
  const uint32_t drain = smem_u32(bars + 19);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  const int n_items = BH * p.n_qt;
  const int C = p.H * kD;
  // item -> (q0, b, h, first key tile, key tiles)
  auto item_of = [&](int it, int &q0, int &b, int &h, int &kbase, int &n_kv) {
    const int qt = p.n_qt - 1 - it / BH;  // latest query tiles (most keys) first
    h = (it % BH) % p.H;
    b = (it % BH) / p.H;
    q0 = qt * kQ;
    const int kt_lo = kWin ? max(0, q0 - p.window + 1) / kKV : 0;
    n_kv = (min(q0 + kQ, p.T) + kKV - 1) / kKV - kt_lo;
    kbase = kt_lo * kKV;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(p_full(s), 128);  // one warpgroup
      mbar_init(o_done(s), 1);
    }
    mbar_init(o_free, 256);  // both warpgroups, after the merge has read O
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPpRegsLow));
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int kc = 0, vc = 0, li = 0;  // K and V tiles and items requested so far
      bool okp = true;
      for (int it = blockIdx.x; it < n_items && okp; it += gridDim.x, ++li) {
        int q0, b, h, kbase, n_kv;
        item_of(it, q0, b, h, kbase, n_kv);
        const int qb = li & 1;
        if (!(okp = mbar_wait(q_empty(qb), ((li >> 1) & 1) ^ 1, abort_flag, p.status))) break;
        mbar_expect_tx(q_full(qb), kTileBytes);
        for (int i = 0; i < 2; ++i)
          tma_load_3d(smem_u32(sQ) + qb * kTileBytes + i * 16384, &map_qk, h * kD + 64 * i, q0, b, q_full(qb));
        auto load_k = [&](int j) -> bool {
          const int st = kc % kPpStages;
          if (!mbar_wait(k_empty(st), ((kc / kPpStages) & 1) ^ 1, abort_flag, p.status)) return false;
          const uint32_t k_dst = smem_u32(sK) + st * kTileBytes;
          mbar_expect_tx(k_full(st), kTileBytes);
          for (int i = 0; i < 2; ++i)
            tma_load_3d(k_dst + i * 16384, &map_qk, C + 64 * i, kbase + j * kKV, b, k_full(st));
          ++kc;
          return true;
        };
        auto load_v = [&](int j) -> bool {
          const int st = vc % kPpStages;
          if (!mbar_wait(v_empty(st), ((vc / kPpStages) & 1) ^ 1, abort_flag, p.status)) return false;
          const uint32_t v_dst = smem_u32(sV) + st * kTileBytes;
          mbar_expect_tx(v_full(st), kTileBytes);
          for (int hh = 0; hh < 2; ++hh)
            for (int a = 0; a < 2; ++a)
              tma_load_3d(v_dst + hh * 16384 + a * 8192, &map_v, C + kD + 64 * a, kbase + j * kKV + 64 * hh, b,
                          v_full(st));
          ++vc;
          return true;
        };
        // V_j is requested before K_{j+2}, whose slot frees only when S_j is done
        okp = load_k(0) && (n_kv < 2 || load_k(1));
        for (int j = 0; j < n_kv && okp; ++j) okp = load_v(j) && (j + 2 >= n_kv || load_k(j + 2));
      }
      // no copy of ours may still be landing when the CTA exits
      for (int i = max(0, li - 2); i < li; ++i) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(q_full(i & 1), (i >> 1) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
      for (int c = max(0, kc - kPpStages); c < kc; ++c) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(k_full(c % kPpStages), (c / kPpStages) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
      for (int c = max(0, vc - kPpStages); c < vc; ++c) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(v_full(c % kPpStages), (c / kPpStages) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc_s = make_idesc(0, 0, kQ, kKV);
      const uint32_t idesc_o = make_idesc(0, 1, kQ, kD);
      const uint64_t dQ0 = smem_desc(smem_u32(sQ), 16, 1024), dKd = smem_desc(smem_u32(sK), 16, 1024);
      const uint64_t dVd = smem_desc(smem_u32(sV), 8192, 1024);
      int kc = 0, vc = 0, li = 0;
      int pc[2] = {0, 0};  // P tiles taken per score buffer
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++li) {
        int q0, b, h, kbase, n_kv;
        item_of(it, q0, b, h, kbase, n_kv);
        const int qb = li & 1;
        if (!(ok = mbar_wait(q_full(qb), (li >> 1) & 1, abort_flag, p.status))) break;
        const uint64_t dQd = dQ0 + (uint64_t)((qb * kTileBytes) >> 4);
        auto issue_s = [&](int j) -> bool {
          const int ks = kc % kPpStages;
          if (!mbar_wait(k_full(ks), (kc / kPpStages) & 1, abort_flag, p.status)) return false;
          tc_fence_after();
          const uint64_t bK = dKd + (uint64_t)((ks * kTileBytes) >> 4);
#pragma unroll
          for (int s = 0; s < kD / 16; ++s) {
            const uint32_t off = ((s >> 2) * 16384 + (s & 3) * 32) >> 4;
            tc_mma(tmem + (j & 1) * kKV, dQd + off, bK + off, idesc_s, s > 0 ? 1u : 0u);
          }
          tc_commit(s_full(j & 1));
          tc_commit(k_empty(ks));
          ++kc;
          return true;
        };
        ok = issue_s(0) && (n_kv < 2 || issue_s(1));
        // the previous item's merge must have read O before P_0 V_0 overwrites it
        if (ok && li > 0) ok = mbar_wait(o_free, (li - 1) & 1, abort_flag, p.status);
        for (int j = 0; j < n_kv && ok; ++j) {
          const int bb = j & 1;
          if (!(ok = mbar_wait(p_full(bb), pc[bb] & 1, abort_flag, p.status))) break;
          ++pc[bb];
          const int vs = vc % kPpStages;
          if (!(ok = mbar_wait(v_full(vs), (vc / kPpStages) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint64_t bV = dVd + (uint64_t)((vs * kTileBytes) >> 4);
          const uint32_t a_p = tmem + bb * kKV;  // P_j over the first 64 columns of S_j
#pragma unroll
          for (int s = 0; s < kKV / 16; ++s) {
            const uint32_t b_off = ((s >> 2) * 16384 + (s & 3) * 2048) >> 4;
            tc_mma_ts(tmem + kPpOCol + bb * kD, a_p + 8 * s, bV + b_off, idesc_o, (j >= 2 || s > 0) ? 1u : 0u);
          }
          tc_commit(o_done(bb));
          tc_commit(v_empty(vs));
          ++vc;
          if (j + 2 < n_kv) ok = issue_s(j + 2);
        }
      }
      tc_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try(drain, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPpRegsHigh));
    // ---------------- softmax warpgroups: group g takes key tiles j = g, g + 2, ... ----------------
    const int grp = (warp - 4) >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t t_s = lane_base + grp * kKV;           // S_j, then P_j
    const uint32_t t_o = lane_base + kPpOCol + grp * kD;  // this group's O
    const float sc = rsqrtf((float)kD) * kLog2e;
    int scnt = 0;  // this group's tiles so far, over all items (phase of s_full, p_full, o_done)
    int li = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++li) {
    int q0, b, h, kbase, n_kv;
    item_of(it, q0, b, h, kbase, n_kv);
    const int row = q0 + r;
    const int qb = li & 1;
    uint8_t *sQb = sQ + qb * kTileBytes;  // this item's Q, then its output tile
    float m_used = -INFINITY, l = 0.f;
    int mine = 0;
    for (int j = grp; j < n_kv && ok; j += 2) {
      ok = mbar_wait(s_full(grp), scnt & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float s[kKV];
      {
        uint32_t u[kKV];
#pragma unroll
        for (int c = 0; c < kKV / 32; ++c) tmem_ld32_nw(t_s + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(u + 32 * c));
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kKV; ++i) s[i] = __uint_as_float(u[i]);  // raw scores: the scale goes into the exponent
      }
      const int kv0 = kbase + j * kKV;
      if (kv0 + kKV - 1 > q0 || kv0 + kKV > p.T || (kWin && kv0 <= q0 + kQ - 1 - p.window)) {
#pragma unroll
        for (int i = 0; i < kKV; ++i)
          if (kv0 + i > row || kv0 + i >= p.T || (kWin && row - (kv0 + i) >= p.window)) s[i] = -INFINITY;
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < kKV; i += 2) mx4[(i >> 1) & 3] = max3(mx4[(i >> 1) & 3], s[i], s[i + 1]);
      const float mx = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sc;
      // the exponent base moves only when the max grows by more than 2^8
      const bool first = j == grp;
      const bool grow = first || mx > m_used + kRescaleLog2;
      const float corr = (!first && grow) ? ex2(m_used - mx) : 1.f;
      if (grow) {
        l *= corr;
        m_used = mx;
      }
      // a row that has seen no key yet (windows only) keeps its base at -inf
      // and takes its exponentials against 0 (all of them 0)
      const float nmb = m_used == -INFINITY ? 0.f : -m_used;
      // exponents s sc - m two at a time (f32x2), then one pair in four on the
      // FMA pipe and the rest on MUFU; the row sum in two f32x2 accumulators
      const uint64_t sc2 = f2(sc, sc), nmb2 = f2(nmb, nmb);
      uint64_t sum2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < kKV / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int k = 32 * c + i;
          const uint64_t x = fma2(f2(s[k], s[k + 1]), sc2, nmb2);
          float e0, e1;
          if ((i & 6) == 6) {
            ex2_poly2(x, e0, e1);
          } else {
            float x0, x1;
            f2split(x, x0, x1);
            e0 = ex2(x0);
            e1 = ex2(x1);
          }
          sum2[(i >> 1) & 1] = add2(sum2[(i >> 1) & 1], f2(e0, e1));
          pk[i / 2] = pack2(e0, e1);
        }
        tmem_st16_nw(t_s + 16 * c, pk);  // keys [32c, 32c + 32) as 16 columns of bf16 pairs
      }
      {
        float a0, a1, b0, b1;
        f2split(sum2[0], a0, a1);
        f2split(sum2[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
      if (!first && __any_sync(0xffffffffu, grow)) {
        // the max grew: bring this group's O to the new base before P_j V_j
        // adds to it (its previous P V is complete: see the kernel's header)
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(t_o + 32 * c, rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * corr);
          tmem_st32(t_o + 32 * c, rr);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(grp));
      ++scnt;
      ++mine;
    }
    // ---------------- merge of the two groups, O / l, lse ----------------
    if (ok && mine > 0) ok = mbar_wait(o_done(grp), (scnt - 1) & 1, abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    sML[(grp * 2 + 0) * kQ + r] = m_used;
    sML[(grp * 2 + 1) * kQ + r] = l;
    ok = epi_vote_all256(ok);  // also the barrier that publishes sML
    const int n1 = n_kv / 2;   // tiles of group 1 (group 0 has at least one)
    if (ok) {
      tc_fence_after();
      const float m0 = sML[r], l0 = sML[kQ + r];
      const float m1 = sML[2 * kQ + r], l1 = sML[3 * kQ + r];
      const float mm = fmaxf(m0, m1);
      const float a0 = m0 == -INFINITY ? 0.f : ex2(m0 - mm);
      const float a1 = (n1 == 0 || m1 == -INFINITY) ? 0.f : ex2(m1 - mm);
      const float lt = a0 * l0 + a1 * l1;
      const float inv = 1.f / lt;
      const float f0 = a0 * inv, f1 = a1 * inv;
      // group g writes O's columns [64g, 64g + 64)
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int col = 64 * grp + 32 * c;
        uint32_t r0[32], r1[32];
        tmem_ld32_nw(lane_base + kPpOCol + col, r0);
        if (n1 > 0) tmem_ld32_nw(lane_base + kPpOCol + kD + col, r1);
        tmem_wait_ld();
        float o[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          o[i] = n1 > 0 ? __uint_as_float(r0[i]) * f0 + __uint_as_float(r1[i]) * f1 : __uint_as_float(r0[i]) * f0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack2(o[8 * u + 0], o[8 * u + 1]);
          w.y = pack2(o[8 * u + 2], o[8 * u + 3]);
          w.z = pack2(o[8 * u + 4], o[8 * u + 5]);
          w.w = pack2(o[8 * u + 6], o[8 * u + 7]);
          *reinterpret_cast<uint4 *>(sQb + tile_unit(r, 8 * grp + 4 * c + u)) = w;  // Q is no longer read
        }
      }
      if (grp == 0 && row < p.T) p.lse[((int64_t)b * p.H + h) * p.T + row] = (mm + __log2f(lt)) * (1.f / kLog2e);
    }
    tc_fence_before();
    mbar_arrive(o_free);  // O_0, O_1 may take the next item's P V now
    fence_proxy_async();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ok && warp == 4 && lane == 0) {
      for (int i = 0; i < 2; ++i) tma_store_3d(&map_o, smem_u32(sQb) + i * 16384, h * kD + 64 * i, q0, b);
      bulk_commit();
      bulk_wait_read0();
      mbar_arrive(q_empty(qb));  // the buffer may take a later item's Q
    }
    if (!ok) break;
    }
    if (warp == 4 && lane == 0) bulk_wait0();  // every store complete before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}


// ===========================================================================
// Backward.  With P = exp(S - lse) recomputed from the saved log-sum-exp and
// D = rowsum(dO * O):  dS = P (dO V^T - D),  dQ = dS K / sqrt(d),
// dK = dS^T Q / sqrt(d) and dV = P^T dO, the last two summed over every query
// head that shares the key/value head.

// ---------------- dQ: CTA = 128 queries of one (b, h), keys in tiles of 128 ----------------
// 128-key tiles keep every MMA at N = 128 (an M = 128, N = 64 MMA takes as
// long as an N = 128 one), and halve the hand-offs per key.
constexpr int kBK = 128;
constexpr int kDqKStages = 3, kDqVStages = 2;  // K is read by S and dQ, V only by dP: separate rings
constexpr int kDsCol = 384;                    // dS[2] as bf16 pairs: key k of row m at column 384 + 64 b + k/2
constexpr int kDqSmem = 1024 + 2 * kTileBytes + (kDqKStages + kDqVStages) * kTileBytes + 256 + 1024;

// backward kernels: warp 0 TMA, warp 1 MMA, warps 2..9 element-wise; the
// element-wise warps w and w+4 share TMEM lane quarter (w & 3) and split the
// tile's columns between them (warpgroup g = (w - 2) / 4 takes half g)
constexpr int kBwdThreads = 320;
constexpr int kSoft = 256;

struct BwdParams {
  int T, H, n_tiles, ld;
  int window;         // windowed kernels: query i sees keys j with 0 <= i - j < window
  const float *lse;   // [B, H, T]
  float *Drow;        // [B, H, T]: rowsum(dO * O), written by the dQ kernel
  const bf16 *O;      // [B*T, H*128]
  int *status;
  // dK/dV schedule: key tile kt's (head, query tile) iterations are cut into
  // ceil(n_it / chunk) pieces, one CTA each (chunk = 0: one piece); a tile cut
  // into several pieces leaves fp32 partial sums in `part` that
  // attn_bwd_dkdv_reduce_kernel adds in piece order
  int B, chunk;
  float *part;        // [grid][128][256]: dK | dV rows of a piece, unscaled
};

// Iterations (head x 128-query tile) of key tile kt in the dK/dV kernel.
__host__ __device__ inline int dkdv_iters(int kt, int n_tiles, int H, int window, bool win) {
  const int last_q = win ? min(n_tiles - 1, (kt * 128 + 127 + window - 1) / 128) : n_tiles - 1;
  return (last_q - kt + 1) * H;
}
__host__ __device__ inline int dkdv_pieces(int n_it, int chunk) {
  return chunk > 0 ? (n_it + chunk - 1) / chunk : 1;
}

// Persistent: CTA c takes the work items c, c + grid, ... (item = 128 queries
// of one (b, h), latest query tiles first); grid = the item count gives one
// item per CTA.  Q and dO have one buffer each: the next item's tiles are
// requested as soon as the last score MMAs of the current one are done
// (qg_free) and its D has been read out of the dO tile (d_done: an item with
// one key tile can finish its MMAs before that), so they land while its last
// dS, dQ MMA and store finish.  The
// output tile is staged in the V ring slot of the item's last key tile, whose
// release (v_empty) then waits for the store to have read it; the next item's
// first dQ MMA waits until the store's TMEM read is done (dq_free).  Barrier
// phases count uses over all items of the CTA.
template <bool kWin>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap map_q,    // qkv, box 64 x 128 (Q, K, V tiles)
                          const __grid_constant__ CUtensorMap map_do,   // dO [B][T][C], box 64 x 128
                          const __grid_constant__ CUtensorMap map_dq,   // dqkv, box 64 x 128
                          const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem, *sG = sQ + kTileBytes;
  uint8_t *sK = sG + kTileBytes;                 // K ring
  uint8_t *sV = sK + kDqKStages * kTileBytes;    // V ring
  uint64_t *bars = reinterpret_cast<uint64_t *>(sV + kDqVStages * kTileBytes);
  // q_full, k_full[3], k_empty[3], v_full[2], v_empty[2], s_full, s_empty, ds_full[2], ds_empty[2], fin,
  // drain, qg_free, dq_free, d_done
  constexpr int kB = 1 + 2 * kDqKStages + 2 * kDqVStages;
  static_assert((kB + 11) * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit their 256 bytes");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kB + 11);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t q_full = smem_u32(bars);
  auto k_full = [&](int s) { return smem_u32(bars + 1 + s); };
  auto k_empty = [&](int s) { return smem_u32(bars + 1 + kDqKStages + s); };
  auto v_full = [&](int s) { return smem_u32(bars + 1 + 2 * kDqKStages + s); };
  auto v_empty = [&](int s) { return smem_u32(bars + 1 + 2 * kDqKStages + kDqVStages + s); };
  const uint32_t s_full = smem_u32(bars + kB), s_empty = smem_u32(bars + kB + 1);
  auto ds_full = [&](int s) { return smem_u32(bars + kB + 2 + s); };
  auto ds_empty = [&](int s) { return smem_u32(bars + kB + 4 + s); };
  const uint32_t fin = smem_u32(bars + kB + 6), drain = smem_u32(bars + kB + 7);
  const uint32_t qg_free = smem_u32(bars + kB + 8), dq_free = smem_u32(bars + kB + 9);
  const uint32_t d_done = smem_u32(bars + kB + 10);  // the item's D has been read out of the dO tile

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  const int n_items = BH * p.n_tiles;
  const int C = p.H * kD;
  auto item_of = [&](int it, int &q0, int &b, int &h, int &kbase, int &n_kv) {
    const int qt = p.n_tiles - 1 - it / BH;
    h = (it % BH) % p.H;
    b = (it % BH) / p.H;
    q0 = qt * kQ;
    const int kt_lo = kWin ? max(0, q0 - p.window + 1) / kBK : 0;
    n_kv = (min(q0 + kQ, p.T) + kBK - 1) / kBK - kt_lo;
    kbase = kt_lo * kBK;
  };
  // TMEM columns: S at 0, dP at 128 (one buffer, free again as soon as the
  // element-wise warps have loaded it); dQ at 256; dS[2] (bf16 pairs) at 384, 448
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kDqKStages; ++s) { mbar_init(k_full(s), 1); mbar_init(k_empty(s), 1); }
    for (int s = 0; s < kDqVStages; ++s) { mbar_init(v_full(s), 1); mbar_init(v_empty(s), 1); }
    mbar_init(s_full, 1);
    mbar_init(s_empty, kSoft);
    for (int s = 0; s < 2; ++s) { mbar_init(ds_full(s), kSoft); mbar_init(ds_empty(s), 1); }
    mbar_init(fin, 1);
    mbar_init(drain, 1);
    mbar_init(qg_free, 1);
    mbar_init(dq_free, kSoft);
    mbar_init(d_done, kSoft);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int kc = 0, vc = 0, li = 0, nq = 0;  // K, V tiles, items, Q/dO pairs requested so far
      bool okp = true;
      for (int it = blockIdx.x; it < n_items && okp; it += gridDim.x, ++li) {
        int q0, b, h, kbase, n_kv;
        item_of(it, q0, b, h, kbase, n_kv);
        // Q and dO take the next item once the previous item's last score MMAs
        // are done and its D has been formed from the dO tile (with one key
        // tile the MMAs can finish first)
        if (li > 0 && !(okp = mbar_wait(qg_free, (li - 1) & 1, abort_flag, p.status) &&
                              mbar_wait(d_done, (li - 1) & 1, abort_flag, p.status)))
          break;
        mbar_expect_tx(q_full, 2 * kTileBytes);
        for (int i = 0; i < 2; ++i) {
          tma_load_3d(smem_u32(sQ) + i * 16384, &map_q, h * kD + 64 * i, q0, b, q_full);
          tma_load_3d(smem_u32(sG) + i * 16384, &map_do, h * kD + 64 * i, q0, b, q_full);
        }
        ++nq;
        for (int j = 0; j < n_kv; ++j) {
          const int ks = kc % kDqKStages, vs = vc % kDqVStages;
          if (!(okp = mbar_wait(k_empty(ks), ((kc / kDqKStages) & 1) ^ 1, abort_flag, p.status))) break;
          mbar_expect_tx(k_full(ks), kTileBytes);
          for (int i = 0; i < 2; ++i)
            tma_load_3d(smem_u32(sK) + ks * kTileBytes + i * 16384, &map_q, C + 64 * i, kbase + j * kBK, b,
                        k_full(ks));
          ++kc;
          if (!(okp = mbar_wait(v_empty(vs), ((vc / kDqVStages) & 1) ^ 1, abort_flag, p.status))) break;
          mbar_expect_tx(v_full(vs), kTileBytes);
          for (int i = 0; i < 2; ++i)
            tma_load_3d(smem_u32(sV) + vs * kTileBytes + i * 16384, &map_q, C + kD + 64 * i, kbase + j * kBK, b,
                        v_full(vs));
          ++vc;
        }
      }
      // let the loads in flight land before the CTA can exit
      if (nq > 0) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try(q_full, (nq - 1) & 1) && globaltimer() - t0 < kWaitNs) {}
      }
      for (int c = max(0, kc - kDqKStages); c < kc; ++c) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(k_full(c % kDqKStages), (c / kDqKStages) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
      for (int c = max(0, vc - kDqVStages); c < vc; ++c) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(v_full(c % kDqVStages), (c / kDqVStages) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc(0, 0, kQ, kBK);   // Q K^T, dO V^T
      const uint32_t idesc_q = make_idesc(0, 1, kQ, kD);    // dS K: dS from TMEM, K as MN-major B
      // Descriptors are built once; (byte offset >> 4) added to one moves its
      // start address (shared addresses stay below 2^18, so the 14-bit field
      // cannot carry).  The issuing thread shares its scheduler with two
      // element-wise warps, so every instruction it saves shortens the
      // hand-offs that keep the tensor pipe fed.
      const uint64_t dQd = smem_desc(smem_u32(sQ), 16, 1024), dGd = smem_desc(smem_u32(sG), 16, 1024);
      const uint64_t dKs = smem_desc(smem_u32(sK), 16, 1024);      // K-major view of K stage 0
      const uint64_t dKm = smem_desc(smem_u32(sK), 16384, 1024);   // MN-major view of K stage 0
      const uint64_t dVs = smem_desc(smem_u32(sV), 16, 1024);
      int kc = 0, vc = 0, sc = 0, li = 0;  // K, V tiles, score tiles and items taken so far
      int dsc[2] = {0, 0};                // dS tiles per TMEM buffer
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++li) {
        int q0, b, h, kbase, n_kv;
        item_of(it, q0, b, h, kbase, n_kv);
        if (!(ok = mbar_wait(q_full, li & 1, abort_flag, p.status))) break;
        const int kc0 = kc;  // this item's first K tile
        auto issue_sdp = [&](int j) -> bool {
          const int ks = kc % kDqKStages, vs = vc % kDqVStages;
          if (!mbar_wait(k_full(ks), (kc / kDqKStages) & 1, abort_flag, p.status)) return false;
          if (!mbar_wait(v_full(vs), (vc / kDqVStages) & 1, abort_flag, p.status)) return false;
          if (!mbar_wait(s_empty, (sc & 1) ^ 1, abort_flag, p.status)) return false;
          tc_fence_after();
          const uint64_t k = dKs + (uint64_t)((ks * kTileBytes) >> 4), v = dVs + (uint64_t)((vs * kTileBytes) >> 4);
#pragma unroll
          for (int s = 0; s < kD / 16; ++s) {
            const uint32_t o = ((s >> 2) * 16384 + (s & 3) * 32) >> 4;
            tc_mma(tmem + 0, dQd + o, k + o, idesc_s, s > 0);
            tc_mma(tmem + 128, dGd + o, v + o, idesc_s, s > 0);
          }
          tc_commit(s_full);
          if (j + 1 < n_kv) tc_commit(v_empty(vs));  // V is read by dP only; the last slot stages the output
          else tc_commit(qg_free);                    // Q and dO are read by no later MMA of this item
          ++kc;
          ++vc;
          ++sc;
          return true;
        };
        // Fixed order S_{j+1}, then dQ += dS_j K_j: the scores of the next tile
        // are on the tensor core while the element-wise warps turn S_j into dS_j.
        ok = issue_sdp(0);
        // the previous item's dQ must have left TMEM before this item's first dQ MMA
        if (ok && li > 0) ok = mbar_wait(dq_free, (li - 1) & 1, abort_flag, p.status);
        for (int j = 0; j < n_kv && ok; ++j) {
          if (j + 1 < n_kv && !(ok = issue_sdp(j + 1))) break;
          const int bb = j & 1, ks = (kc0 + j) % kDqKStages;
          if (!(ok = mbar_wait(ds_full(bb), dsc[bb] & 1, abort_flag, p.status))) break;
          ++dsc[bb];
          tc_fence_after();
          const uint64_t k = dKm + (uint64_t)((ks * kTileBytes) >> 4);
#pragma unroll
          for (int s = 0; s < kBK / 16; ++s)
            tc_mma_ts(tmem + 256, tmem + kDsCol + bb * 64 + 8 * s, k + ((s * 2048) >> 4), idesc_q,
                      (j > 0 || s > 0) ? 1u : 0u);
          tc_commit(ds_empty(bb));
          tc_commit(k_empty(ks));
        }
        if (ok) tc_commit(fin);
      }
      tc_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try(drain, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ---------------- element-wise warps: thread = query row, half g of the keys ----------------
    const int quarter = warp & 3, g = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = rsqrtf((float)kD) * kLog2e;
    const int c0 = g * 64;  // this thread's 64 keys of the 128-key tile
    float *sDpart = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + 256);  // [2][128]
    int tc = 0, vcount = 0, li = 0;  // score tiles, V tiles and items so far
    int dsc[2] = {0, 0};
    bool ok = true;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++li) {
    int q0, b, h, kbase, n_kv;
    item_of(it, q0, b, h, kbase, n_kv);
    const int row = q0 + r;
    const int rr_ = min(row, p.T - 1);
    const float L = p.lse[((int64_t)b * p.H + h) * p.T + rr_] * kLog2e;
    // D = rowsum(dO * O) for this row: dO from the shared tile, O from global;
    // warpgroup g sums dims [64g, 64g + 64) and the halves meet in shared memory
    if (ok) ok = mbar_wait(q_full, li & 1, abort_flag, p.status);
    {
      float part = 0.f;
      if (row < p.T) {
        const bf16 *orow = p.O + ((int64_t)b * p.T + row) * C + h * kD + 64 * g;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float o8[8], g8[8];
          Vec8<bf16>::load(orow + 8 * u, o8);
          Vec8<bf16>::load(reinterpret_cast<const bf16 *>(sG + g * 16384 + r * 128 + ((u ^ (r & 7)) << 4)), g8);
#pragma unroll
          for (int i = 0; i < 8; ++i) part += o8[i] * g8[i];
        }
      }
      sDpart[g * kQ + r] = part;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    mbar_arrive(d_done);  // every thread has read its part of the dO tile
    const float Dv = sDpart[r] + sDpart[kQ + r];
    if (g == 0 && row < p.T) p.Drow[((int64_t)b * p.H + h) * p.T + row] = Dv;
    for (int j = 0; j < n_kv && ok; ++j) {
      const int bb = j & 1;
      ok = mbar_wait(s_full, tc & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      ++tc;
      tc_fence_after();
      // all 64 S and dP values of this row half at once, so the buffer is
      // free for the next tile's MMAs before any arithmetic here
      uint32_t sv[64], dv[64];
      tmem_ld32_nw(lane_base + c0, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32_nw(lane_base + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_ld32_nw(lane_base + 128 + c0, *reinterpret_cast<uint32_t(*)[32]>(dv));
      tmem_ld32_nw(lane_base + 128 + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(dv + 32));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_empty);
      const int kv0 = kbase + j * kBK + c0;
      const bool need_mask = kv0 + 64 > q0 || kv0 + 64 > p.T || (kWin && kv0 <= q0 + kQ - 1 - p.window);
      uint32_t packed[32];
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        float d2[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          float pr = ex2(fmaf(__uint_as_float(sv[i + t]), sc, -L));
          const int key = kv0 + i + t;
          if (need_mask && (key > row || key >= p.T || (kWin && row - key >= p.window))) pr = 0.f;
          d2[t] = pr * (__uint_as_float(dv[i + t]) - Dv);
        }
        packed[i / 2] = pack2(d2[0], d2[1]);
      }
      // dS_j into TMEM buffer bb once the dQ MMA two tiles back has read it
      ok = mbar_wait(ds_empty(bb), (dsc[bb] & 1) ^ 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      ++dsc[bb];
      tmem_st32(lane_base + kDsCol + bb * 64 + 32 * g, packed);
      tc_fence_before();
      mbar_arrive(ds_full(bb));
    }
    vcount += n_kv;
    const int vslot = (vcount - 1) % kDqVStages;  // the item's last V tile: its slot stages the output
    uint8_t *stg = sV + vslot * kTileBytes;
    if (ok) ok = mbar_wait(fin, li & 1, abort_flag, p.status);
    ok = epi_vote_all256(ok);
    if (ok) {
      tc_fence_after();
      const float scale = rsqrtf((float)kD);
#pragma unroll 1
      for (int c = 2 * g; c < 2 * g + 2; ++c) {  // 64 of the 128 dQ columns
        uint32_t rr[32];
        tmem_ld32(lane_base + 256 + c * 32, rr);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack2(__uint_as_float(rr[8 * u + 0]) * scale, __uint_as_float(rr[8 * u + 1]) * scale);
          w.y = pack2(__uint_as_float(rr[8 * u + 2]) * scale, __uint_as_float(rr[8 * u + 3]) * scale);
          w.z = pack2(__uint_as_float(rr[8 * u + 4]) * scale, __uint_as_float(rr[8 * u + 5]) * scale);
          w.w = pack2(__uint_as_float(rr[8 * u + 6]) * scale, __uint_as_float(rr[8 * u + 7]) * scale);
          *reinterpret_cast<uint4 *>(stg + tile_unit(r, c * 4 + u)) = w;  // V of this slot is no longer read
        }
      }
    }
    tc_fence_before();
    mbar_arrive(dq_free);  // the dQ accumulator may take the next item's MMAs
    fence_proxy_async();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ok && warp == 2 && lane == 0) {
      for (int i = 0; i < 2; ++i) tma_store_3d(&map_dq, smem_u32(stg) + i * 16384, h * kD + 64 * i, q0, b);
      bulk_commit();
      bulk_wait_read0();
      mbar_arrive(v_empty(vslot));  // the slot may take a later V tile
    }
    if (!ok) break;
    }
    if (warp == 2 && lane == 0) bulk_wait0();  // every store complete before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------- dK, dV: CTA = 128 keys of row b; loop over heads x 128-query tiles ----------------
// 128-query tiles keep every MMA at N = 128.  TMEM holds one 128-column
// score buffer X that takes S^T and then dP^T of a tile in turn, P^T and dS^T
// as bf16 A operands, and the dV, dK accumulators:
//   X [0,128)   P^T [128,192)   dS^T [192,256)   dV [256,384)   dK [384,512)
// Per tile the tensor core runs S^T = K Q^T, dP^T = V dO^T (once the
// element-wise warps have loaded S^T), dV += P^T dO (once P^T is stored),
// S^T of the next tile (once dP^T is loaded), dK += dS^T Q.
constexpr int kBQ2 = 128;
constexpr int kKvStages = 2;
constexpr int kQStage = 2 * kTileBytes + 1024;   // Q, dO, then L[128], D[128]; keeps 1 KB alignment
constexpr int kKvSmemTc = 1024 + 2 * kTileBytes + kKvStages * kQStage + 256;
constexpr int kXCol = 0, kPtCol = 128, kDstCol = 192, kDvCol = 256, kDkCol = 384;
static_assert(kQStage % 1024 == 0 && kTileBytes % 1024 == 0,
              "128-byte-swizzled TMA tiles need 1 KB-aligned shared-memory addresses");
static_assert(kKvSmemTc <= 232448 && kDqSmem <= 232448 && kSmem <= 232448, "shared memory per CTA");

template <bool kWin>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap map_qkv,  // qkv, box 64 x 128 (K, V, Q)
                            const __grid_constant__ CUtensorMap map_do,   // dO, box 64 x 128
                            const __grid_constant__ CUtensorMap map_out,  // dqkv, box 64 x 128
                            const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = smem, *sV = sK + kTileBytes;
  uint8_t *sQS = sV + kTileBytes;                 // stage s at s*kQStage: Q, dO, L, D
  uint64_t *bars = reinterpret_cast<uint64_t *>(sQS + kKvStages * kQStage);
  // kv_full, q_full[S] (Q, dO tiles), ld_full[S] (L, D), q_empty[S], then the hand-offs below
  constexpr int kB = 1 + 3 * kKvStages;
  static_assert((kB + 10) * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit their 256 bytes");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kB + 10);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t kv_full = smem_u32(bars);
  auto q_full = [&](int s) { return smem_u32(bars + 1 + s); };
  auto ld_full = [&](int s) { return smem_u32(bars + 1 + kKvStages + s); };
  auto q_empty = [&](int s) { return smem_u32(bars + 1 + 2 * kKvStages + s); };
  const uint32_t s_full = smem_u32(bars + kB), dp_full = smem_u32(bars + kB + 1);      // MMA -> element-wise
  const uint32_t s_taken = smem_u32(bars + kB + 2), dp_taken = smem_u32(bars + kB + 3);  // X loaded
  const uint32_t p_full = smem_u32(bars + kB + 4), p_empty = smem_u32(bars + kB + 5);
  const uint32_t ds_full = smem_u32(bars + kB + 6), ds_empty = smem_u32(bars + kB + 7);
  const uint32_t fin = smem_u32(bars + kB + 8), drain = smem_u32(bars + kB + 9);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA -> (key tile, piece, row b): pieces of key tile 0 (the most work) first
  const int b = (int)blockIdx.x % p.B;
  int kt = 0, piece = (int)blockIdx.x / p.B, n_it = 0, n_pieces = 1;
  for (;; ++kt) {
    n_it = dkdv_iters(kt, p.n_tiles, p.H, p.window, kWin);
    n_pieces = dkdv_pieces(n_it, p.chunk);
    if (piece < n_pieces || kt == p.n_tiles - 1) break;
    piece -= n_pieces;
  }
  const int it0 = (int)((int64_t)piece * n_it / n_pieces), it1 = (int)((int64_t)(piece + 1) * n_it / n_pieces);
  const int my_n = it1 - it0;  // this CTA's iterations it0 .. it1 - 1
  const int k0 = kt * kQ;
  const int C = p.H * kD;
  const int first = k0 / kBQ2;
  const int n_q = n_it / p.H;  // iteration it: head it / n_q, query tile first + it % n_q
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(ld_full(s), 32);
      mbar_init(q_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(s_taken, kSoft);
    mbar_init(dp_taken, kSoft);
    mbar_init(p_full, kSoft);
    mbar_init(p_empty, 1);
    mbar_init(ds_full, kSoft);
    mbar_init(ds_empty, 1);
    mbar_init(fin, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer warp: TMA for tiles, plain loads for lse and D ----------------
    if (lane == 0) {
      mbar_expect_tx(kv_full, 2 * kTileBytes);
      for (int i = 0; i < 2; ++i) {
        tma_load_3d(smem_u32(sK) + i * 16384, &map_qkv, C + 64 * i, k0, b, kv_full);
        tma_load_3d(smem_u32(sV) + i * 16384, &map_qkv, C + kD + 64 * i, k0, b, kv_full);
      }
    }
    int issued = 0;
    for (int j = 0; j < my_n; ++j) {
      const int it = it0 + j, st = j % kKvStages;
      const bool okw = mbar_wait(q_empty(st), ((j / kKvStages) & 1) ^ 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, okw)) break;
      const int hh = it / n_q, qq0 = (first + it % n_q) * kBQ2;
      uint8_t *stage = sQS + st * kQStage;
      // lse and D of the tile's queries: 4-byte asynchronous copies whose
      // completion arrives on the stage's barrier, so this warp never blocks
      const uint32_t ls_dst = smem_u32(stage + 2 * kTileBytes), ds_dst = ls_dst + kBQ2 * 4;
      for (int i = lane; i < kBQ2; i += 32) {
        const int q = min(qq0 + i, p.T - 1);
        const int64_t gi = ((int64_t)b * p.H + hh) * p.T + q;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(ls_dst + 4 * i), "l"(p.lse + gi) : "memory");
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(ds_dst + 4 * i), "l"(p.Drow + gi) : "memory");
      }
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(ld_full(st)) : "memory");
      if (lane == 0) {
        mbar_expect_tx(q_full(st), 2 * kTileBytes);
        const uint32_t dst = smem_u32(stage);
        for (int i = 0; i < 2; ++i) {
          tma_load_3d(dst + i * 16384, &map_qkv, hh * kD + 64 * i, qq0, b, q_full(st));
          tma_load_3d(dst + kTileBytes + i * 16384, &map_do, hh * kD + 64 * i, qq0, b, q_full(st));
        }
      }
      ++issued;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try(kv_full, 0) && globaltimer() - t0 < kWaitNs) {}
      for (int it = max(0, issued - kKvStages); it < issued; ++it) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(q_full(it % kKvStages), (it / kKvStages) & 1) && globaltimer() - t1 < kWaitNs) {}
        while (!mbar_try(ld_full(it % kKvStages), (it / kKvStages) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_x = make_idesc(0, 0, kQ, kBQ2);  // K Q^T, V dO^T
      const uint32_t idesc_g = make_idesc(0, 1, kQ, kD);    // P^T dO, dS^T Q: A from TMEM, B MN-major
      // Descriptors built once; (byte offset >> 4) added moves the start
      // address (no carry: shared addresses are below 2^18).
      const uint64_t dKd = smem_desc(smem_u32(sK), 16, 1024), dVd = smem_desc(smem_u32(sV), 16, 1024);
      const uint64_t dQs = smem_desc(smem_u32(sQS), 16, 1024);     // K-major view of stage 0
      const uint64_t dQm = smem_desc(smem_u32(sQS), 16384, 1024);  // MN-major view of stage 0
      constexpr uint32_t kGo = kTileBytes >> 4;                    // Q -> dO within a stage
      bool ok = mbar_wait(kv_full, 0, abort_flag, p.status);
      auto x_mma = [&](uint64_t a, uint64_t bq) {
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
          const uint32_t o = ((s >> 2) * 16384 + (s & 3) * 32) >> 4;
          tc_mma(tmem + kXCol, a + o, bq + o, idesc_x, s > 0);
        }
      };
      auto g_mma = [&](uint32_t d_col, uint32_t a_col, uint64_t bq, bool first_tile) {
#pragma unroll
        for (int s = 0; s < kBQ2 / 16; ++s)
          tc_mma_ts(tmem + d_col, tmem + a_col + 8 * s, bq + ((s * 2048) >> 4), idesc_g,
                    (!first_tile || s > 0) ? 1u : 0u);
      };
      // S^T_0
      if (ok) ok = mbar_wait(q_full(0), 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        x_mma(dKd, dQs);
        tc_commit(s_full);
      }
      for (int j = 0; j < my_n && ok; ++j) {
        const int st = j % kKvStages;
        const uint64_t qs = dQs + (uint64_t)((st * kQStage) >> 4), qm = dQm + (uint64_t)((st * kQStage) >> 4);
        const uint32_t par = j & 1;
        // dP^T_j = V dO_j^T once S^T_j has left X
        if (!(ok = mbar_wait(s_taken, par, abort_flag, p.status))) break;
        tc_fence_after();
        x_mma(dVd, qs + kGo);
        tc_commit(dp_full);
        // dV += P^T_j dO_j
        if (!(ok = mbar_wait(p_full, par, abort_flag, p.status))) break;
        tc_fence_after();
        g_mma(kDvCol, kPtCol, qm + kGo, j == 0);
        tc_commit(p_empty);
        // S^T_{j+1} = K Q_{j+1}^T once dP^T_j has left X
        if (j + 1 < my_n) {
          const int st1 = (j + 1) % kKvStages;
          if (!(ok = mbar_wait(dp_taken, par, abort_flag, p.status))) break;
          if (!(ok = mbar_wait(q_full(st1), ((j + 1) / kKvStages) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          x_mma(dKd, dQs + (uint64_t)((st1 * kQStage) >> 4));
          tc_commit(s_full);
        }
        // dK += dS^T_j Q_j; the stage is free after this
        if (!(ok = mbar_wait(ds_full, par, abort_flag, p.status))) break;
        tc_fence_after();
        g_mma(kDkCol, kDstCol, qm, j == 0);
        tc_commit(ds_empty);
        tc_commit(q_empty(st));
      }
      tc_commit(fin);
      tc_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try(drain, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ---------------- element-wise warps: thread = key row, half g of the queries ----------------
    const int quarter = warp & 3, g = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int key = k0 + r;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = rsqrtf((float)kD) * kLog2e;
    const int c0 = g * 64;  // this thread's 64 queries of the 128-query tile
    bool ok = true;
    for (int j = 0; j < my_n; ++j) {
      const int st = j % kKvStages;
      const uint32_t par = j & 1;
      const int qq0 = (first + (it0 + j) % n_q) * kBQ2 + c0;
      ok = mbar_wait(s_full, par, abort_flag, p.status) &&
           mbar_wait(ld_full(st), (j / kKvStages) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t xv[64];
      tmem_ld32_nw(lane_base + kXCol + c0, *reinterpret_cast<uint32_t(*)[32]>(xv));
      tmem_ld32_nw(lane_base + kXCol + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(xv + 32));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_taken);  // X may take dP^T now
      const float *Ls = reinterpret_cast<const float *>(sQS + st * kQStage + 2 * kTileBytes) + c0;
      const float *Ds = Ls + kBQ2;
      const bool need_mask = qq0 < key + 1 || qq0 + 64 > p.T || (kWin && qq0 + 63 - key >= p.window);
      // P^T = 2^(s sc - lse log2 e), two queries at a time (f32x2)
      const uint64_t sc2 = f2(sc, sc), nl2e = f2(-kLog2e, -kLog2e);
      float pr[64];
      uint32_t pk[32];
#pragma unroll
      for (int i4 = 0; i4 < 16; ++i4) {
        const float4 l4 = reinterpret_cast<const float4 *>(Ls)[i4];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int qi = 4 * i4 + 2 * h2;
          const uint64_t nl = mul2(h2 ? f2(l4.z, l4.w) : f2(l4.x, l4.y), nl2e);
          const uint64_t x = fma2(f2(__uint_as_float(xv[qi]), __uint_as_float(xv[qi + 1])), sc2, nl);
          float v0, v1;
          if (h2 && (i4 & 1)) {
            ex2_poly2(x, v0, v1);  // one pair in four on the FMA pipe: MUFU bounds this loop
          } else {
            float x0, x1;
            f2split(x, x0, x1);
            v0 = ex2(x0);
            v1 = ex2(x1);
          }
          if (need_mask) {
            if (qq0 + qi < key || qq0 + qi >= p.T || (kWin && qq0 + qi - key >= p.window)) v0 = 0.f;
            if (qq0 + qi + 1 < key || qq0 + qi + 1 >= p.T || (kWin && qq0 + qi + 1 - key >= p.window)) v1 = 0.f;
          }
          pr[qi] = v0;
          pr[qi + 1] = v1;
          pk[qi / 2] = pack2(v0, v1);
        }
      }
      // P^T once dV += P^T_{it-1} dO has read the previous one
      ok = mbar_wait(p_empty, par ^ 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tmem_st32(lane_base + kPtCol + 32 * g, pk);
      tc_fence_before();
      mbar_arrive(p_full);
      ok = mbar_wait(dp_full, par, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      tmem_ld32_nw(lane_base + kXCol + c0, *reinterpret_cast<uint32_t(*)[32]>(xv));
      tmem_ld32_nw(lane_base + kXCol + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(xv + 32));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(dp_taken);  // X may take the next S^T now
      // dS^T = P^T (dP^T - D), two queries at a time (f32x2)
#pragma unroll
      for (int i4 = 0; i4 < 16; ++i4) {
        const float4 d4 = reinterpret_cast<const float4 *>(Ds)[i4];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int qi = 4 * i4 + 2 * h2;
          const uint64_t t = add2(f2(__uint_as_float(xv[qi]), __uint_as_float(xv[qi + 1])),
                                  h2 ? f2(-d4.z, -d4.w) : f2(-d4.x, -d4.y));
          float d0, d1;
          f2split(mul2(f2(pr[qi], pr[qi + 1]), t), d0, d1);
          pk[qi / 2] = pack2(d0, d1);
        }
      }
      ok = mbar_wait(ds_empty, par ^ 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tmem_st32(lane_base + kDstCol + 32 * g, pk);
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok) ok = mbar_wait(fin, 0, abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    const bool split = n_pieces > 1;
    // a piece of a split key tile: its fp32 rows (dK | dV, unscaled) go to the
    // idle Q/dO stages, 16-byte unit u of row r at unit (u ^ (r & 7)), then out
    // to its partial-sum slot with coalesced stores
    float *stg = reinterpret_cast<float *>(sQS);
    if (ok && split) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + (g == 0 ? kDkCol : kDvCol) + c * 32, rr);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int u = 32 * g + 8 * c + q;
          *reinterpret_cast<float4 *>(stg + r * 256 + ((u ^ (r & 7)) << 2)) =
              make_float4(__uint_as_float(rr[4 * q]), __uint_as_float(rr[4 * q + 1]), __uint_as_float(rr[4 * q + 2]),
                          __uint_as_float(rr[4 * q + 3]));
        }
      }
    } else if (ok) {
      tc_fence_after();
      // warpgroup 0 drains dK (scaled) into the K tile, warpgroup 1 dV into the V tile
      uint8_t *dst = g == 0 ? sK : sV;
      const float f = g == 0 ? rsqrtf((float)kD) : 1.f;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + (g == 0 ? kDkCol : kDvCol) + c * 32, rr);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack2(__uint_as_float(rr[8 * u + 0]) * f, __uint_as_float(rr[8 * u + 1]) * f);
          w.y = pack2(__uint_as_float(rr[8 * u + 2]) * f, __uint_as_float(rr[8 * u + 3]) * f);
          w.z = pack2(__uint_as_float(rr[8 * u + 4]) * f, __uint_as_float(rr[8 * u + 5]) * f);
          w.w = pack2(__uint_as_float(rr[8 * u + 6]) * f, __uint_as_float(rr[8 * u + 7]) * f);
          *reinterpret_cast<uint4 *>(dst + tile_unit(r, c * 4 + u)) = w;
        }
      }
    }
    fence_proxy_async();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ok && split) {
      float4 *dst = reinterpret_cast<float4 *>(p.part + (size_t)blockIdx.x * kQ * 2 * kD);
      for (int q = (int)threadIdx.x - 64; q < kQ * 64; q += kSoft) {
        const int row = q >> 6, u = q & 63;
        dst[q] = *reinterpret_cast<const float4 *>(stg + row * 256 + ((u ^ (row & 7)) << 2));
      }
    } else if (ok && warp == 2 && lane == 0) {
      for (int i = 0; i < 2; ++i) {
        tma_store_3d(&map_out, smem_u32(sK) + i * 16384, C + 64 * i, k0, b);
        tma_store_3d(&map_out, smem_u32(sV) + i * 16384, C + kD + 64 * i, k0, b);
      }
      bulk_commit();
      bulk_wait0();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// dK, dV of the key tiles cut into pieces: the pieces' partial sums added in
// piece order (a fixed order: the result does not depend on which piece
// finished first), dK scaled by 1/sqrt(128), both written to dqkv in bf16.
// Block = (key tile, row b); tiles left whole were written by their CTA.
__global__ void __launch_bounds__(256) attn_bwd_dkdv_reduce_kernel(const BwdParams p, bool win, bf16 *dqkv) {
  const int kt = (int)blockIdx.x / p.B, b = (int)blockIdx.x % p.B;
  int prefix = 0;
  for (int t = 0; t < kt; ++t) prefix += dkdv_pieces(dkdv_iters(t, p.n_tiles, p.H, p.window, win), p.chunk);
  const int np = dkdv_pieces(dkdv_iters(kt, p.n_tiles, p.H, p.window, win), p.chunk);
  if (np == 1) return;
  const float f = rsqrtf((float)kD);
  const int C = p.H * kD;
  for (int q = threadIdx.x; q < kQ * 64; q += blockDim.x) {
    const int row = q >> 6, u = q & 63;  // 4 columns of dK (u < 32) or dV
    const int key = kt * kQ + row;
    if (key >= p.T) break;  // rows are visited in order: the rest are past T too
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < np; ++c) {
      const float4 v = reinterpret_cast<const float4 *>(p.part + ((size_t)(prefix + c) * p.B + b) * kQ * 2 * kD)[q];
      a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    }
    if (u < 32) { a.x *= f; a.y *= f; a.z *= f; a.w *= f; }
    uint2 o;
    o.x = pack2(a.x, a.y);
    o.y = pack2(a.z, a.w);
    *reinterpret_cast<uint2 *>(dqkv + ((size_t)b * p.T + key) * p.ld + C + 4 * u) = o;
  }
}

// ------------------------------- host side -------------------------------

// 3-D bf16 map over [B][T][cols] with row stride ld elements.
inline bool make_map3(CUtensorMap *map, const void *base, int B, int T, int cols, int64_t ld, int box_rows) {
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2 * T};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kWin>
inline cudaError_t init_variant() {
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<kWin>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_fwd_pp_kernel<kWin>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);

  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<kWin>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDqSmem);

  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel<kWin>, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmemTc);
  return e;
}
inline cudaError_t init() {
  cudaError_t e = init_variant<false>();
  return e == cudaSuccess ? init_variant<true>() : e;
}

// A window that covers every earlier key is the plain causal mask: only a
// window shorter than the sequence takes the windowed kernels.
inline bool windowed(int window, int T) { return window > 0 && window < T; }

// Operands the TMA tiles can take: 16-byte aligned bases and row strides.
inline bool aligned(const void *qkv, int64_t ld, const void *O) {
  return (ld % 8) == 0 && ((uintptr_t)qkv & 15) == 0 && ((uintptr_t)O & 15) == 0;
}
inline bool supported(const void *qkv, int64_t ld, const void *O) {
  return encode_fn() != nullptr && aligned(qkv, ld, O);
}

// Process-wide cap on the CTAs of the persistent attention kernels (0: one
// per SM): fewer CTAs leave SMs to other streams and give each CTA more items.
inline std::atomic<int> &persistent_cap() {
  static std::atomic<int> cap{0};
  return cap;
}
inline int persistent_ctas(int num_sms) {
  const int c = persistent_cap().load();
  return c > 0 && c < num_sms ? c : num_sms;
}

// pingpong: the kernel with two softmax warpgroups on alternating key tiles,
// persistent over grid = min(items, CTAs) CTAs (num_sms = 0: one CTA per item)
inline cudaError_t launch_fwd(const bf16 *qkv, int64_t ld, bf16 *O, float *lse, int B, int T, int H, int window,
                              bool pingpong, int num_sms, int *status, cudaStream_t st) {
  CUtensorMap mqk, mv, mo;
  const int C = H * kD;
  if (!make_map3(&mqk, qkv, B, T, (int)ld, ld, 128) || !make_map3(&mv, qkv, B, T, (int)ld, ld, 64) ||
      !make_map3(&mo, O, B, T, C, C, 128))
    return cudaErrorInvalidValue;
  FwdParams p;
  p.T = T;
  p.H = H;
  p.n_qt = (T + kQ - 1) / kQ;
  p.lse = lse;
  p.status = status;
  p.window = window;
  p.B = B;
  const int grid = B * H * p.n_qt;
  const bool win = windowed(window, T);
  if (pingpong) {
    const int ctas = num_sms > 0 ? persistent_ctas(num_sms) : 0;
    const int g = ctas > 0 && ctas < grid ? ctas : grid;
    if (win) attn_fwd_pp_kernel<true><<<g, kPpThreads, kSmem, st>>>(mqk, mv, mo, p);
    else attn_fwd_pp_kernel<false><<<g, kPpThreads, kSmem, st>>>(mqk, mv, mo, p);
  } else {
    if (win) attn_fwd_tc_kernel<true><<<grid, kFwdThreads, kSmem, st>>>(mqk, mv, mo, p);
    else attn_fwd_tc_kernel<false><<<grid, kFwdThreads, kSmem, st>>>(mqk, mv, mo, p);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) fprintf(stderr, "nanochat_b200: attention forward launch: %s\n", cudaGetErrorString(e));
  return e;
}

}  // namespace fatc
}  // namespace nc

namespace nc {
namespace fatc {

// Piece size of the dK/dV schedule.  0 (no cut) while the heaviest key tile
// carries at most 1.25 SM shares of the iterations: whole tiles, heaviest
// first, then pack the SMs within a few percent (d20: 160 against 147), and
// every piece costs a prologue, a K/V load and a partial-sum round trip.
// Otherwise pieces of two thirds of a share (at least 4 iterations).
inline int dkdv_chunk(int B, int T, int H, int window, int num_sms) {
  const int n_tiles = (T + kQ - 1) / kQ;
  const bool win = windowed(window, T);
  int64_t total = 0;
  int most = 0;
  for (int kt = 0; kt < n_tiles; ++kt) {
    const int n = dkdv_iters(kt, n_tiles, H, window, win);
    total += n;
    most = max(most, n);
  }
  total *= B;
  const int64_t share = (total + num_sms - 1) / num_sms;
  if (4 * (int64_t)most <= 5 * share) return 0;
  const int64_t piece = (2 * total + 3 * (int64_t)num_sms - 1) / (3 * (int64_t)num_sms);
  const int chunk = (int)(piece > 4 ? piece : 4);
  return most > chunk ? chunk : 0;
}

// CTAs of the dK/dV kernel for a piece size.
inline int dkdv_grid(int B, int T, int H, int window, int chunk) {
  const int n_tiles = (T + kQ - 1) / kQ;
  const bool win = windowed(window, T);
  int pieces = 0;
  for (int kt = 0; kt < n_tiles; ++kt) pieces += dkdv_pieces(dkdv_iters(kt, n_tiles, H, window, win), chunk);
  return pieces * B;
}

// Bytes of partial sums the cut schedule needs (0 when nothing is cut).
inline size_t dkdv_scratch_bytes(int B, int T, int H, int window, int num_sms) {
  const int chunk = dkdv_chunk(B, T, H, window, num_sms);
  return chunk ? (size_t)dkdv_grid(B, T, H, window, chunk) * kQ * 2 * kD * sizeof(float) : 0;
}

// part: scratch for the cut dK/dV schedule (part_bytes >= dkdv_scratch_bytes);
// nullptr: every key tile in one CTA.
inline cudaError_t launch_bwd(const bf16 *qkv, int64_t ld, const bf16 *O, const bf16 *dO, const float *lse,
                              float *Drow, float *part, size_t part_bytes, bf16 *dqkv, int B, int T, int H,
                              int window, int num_sms, int *status, cudaStream_t st, int *launched = nullptr) {
  CUtensorMap mq128, mdo128, mout;
  const int C = H * kD;
  if (!make_map3(&mq128, qkv, B, T, (int)ld, ld, 128) || !make_map3(&mdo128, dO, B, T, C, C, 128) ||
      !make_map3(&mout, dqkv, B, T, (int)ld, ld, 128))
    return cudaErrorInvalidValue;
  BwdParams p;
  p.T = T;
  p.H = H;
  p.ld = (int)ld;
  p.lse = lse;
  p.Drow = Drow;
  p.O = O;
  p.status = status;
  p.n_tiles = (T + kQ - 1) / kQ;
  p.window = window;
  p.B = B;
  p.chunk = 0;
  p.part = nullptr;
  if (part && part_bytes >= dkdv_scratch_bytes(B, T, H, window, num_sms)) {
    p.chunk = dkdv_chunk(B, T, H, window, num_sms);
    p.part = part;
  }
  const int grid_kv = dkdv_grid(B, T, H, window, p.chunk);
  const bool win = windowed(window, T);
  // dQ: persistent, one CTA per SM over the B * H * n_tiles query tiles
  const int dq_items = B * H * p.n_tiles;
  const int dq_ctas = persistent_ctas(num_sms);
  const int grid_dq = dq_ctas > 0 && dq_ctas < dq_items ? dq_ctas : dq_items;
  if (win) attn_bwd_dq_tc_kernel<true><<<grid_dq, kBwdThreads, kDqSmem, st>>>(mq128, mdo128, mout, p);
  else attn_bwd_dq_tc_kernel<false><<<grid_dq, kBwdThreads, kDqSmem, st>>>(mq128, mdo128, mout, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "nanochat_b200: attention dQ launch: %s\n", cudaGetErrorString(e));
    return e;
  }
  if (win) attn_bwd_dkdv_tc_kernel<true><<<grid_kv, kBwdThreads, kKvSmemTc, st>>>(mq128, mdo128, mout, p);
  else attn_bwd_dkdv_tc_kernel<false><<<grid_kv, kBwdThreads, kKvSmemTc, st>>>(mq128, mdo128, mout, p);
  if (p.chunk) attn_bwd_dkdv_reduce_kernel<<<B * p.n_tiles, 256, 0, st>>>(p, win, dqkv);
  if (launched) *launched = p.chunk ? 3 : 2;
  return cudaGetLastError();
}

inline bool aligned_bwd(const void *qkv, int64_t ld, const void *O, const void *dO, const void *dqkv) {
  return aligned(qkv, ld, dO) && ((uintptr_t)dqkv & 15) == 0 && ((uintptr_t)O & 15) == 0;
}
inline bool supported_bwd(const void *qkv, int64_t ld, const void *O, const void *dO, const void *dqkv) {
  return encode_fn() != nullptr && aligned_bwd(qkv, ld, O, dO, dqkv);
}

}  // namespace fatc
}  // namespace nc
