// Causal multi-query attention forward on the 5th-generation tensor cores
// (energyai.berlin page, "Multi-Query Attention (MQA)": one key/value head
// shared by the H query heads; scores q.k / sqrt(128), keys j <= i).
//
// CTA = 128 queries of one (row b, head h); keys in tiles of 128.
//   warp 0      TMA: Q once, then K and V tiles into a 2-stage ring
//   warp 1      MMA: S_j = Q K_j^T into one of two TMEM score tiles,
//               O += P_j V_j into a TMEM accumulator
//   warps 2..5  softmax, one thread per query row: S row out of TMEM, running
//               max / sum, P_j as bf16 into shared memory (the next MMA's
//               A operand), O rescaled in TMEM only when the row max grows by
//               more than 2^8 (the exponent base may lag the true max by up to
//               8 in the log2 domain, which changes no result: P and the sum
//               carry the same factor)
// S_{j+1} is issued before P_j is ready, so the tensor core works on the next
// scores while the softmax warps finish the current tile.
//
// Operands, all bf16 with 128-byte swizzle: Q, K as K-major (d contiguous)
// tiles of 2 boxes [64 d x 128 rows]; V as an MN-major B operand (d
// contiguous) of 4 boxes [64 d x 64 keys]; P as a K-major A operand of 2
// blocks [64 keys x 128 rows] written by the softmax threads.
#pragma once

#include "tc_common.cuh"

namespace nc {
namespace fatc {

using namespace tc;

constexpr int kQ = 128, kKV = 128, kD = 128;
constexpr int kThreads = 192;
constexpr int kTileBytes = kQ * kD * 2;      // 32 KB: Q, K, V or P tile
constexpr int kStageBytes = 2 * kTileBytes;  // K + V
constexpr int kSmem = 1024 + kTileBytes /*Q*/ + 2 * kStageBytes + kTileBytes /*P*/ + 256;
constexpr int kTmemCols = 512;               // S0 [0,128), S1 [128,256), O [256,384)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
  int T, H, n_qt;
  float *lse;   // [B, H, T]
  int *status;
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_qk,   // qkv [B][T][ld], box 64 x 128
                       const __grid_constant__ CUtensorMap map_v,    // qkv, box 64 x 64
                       const __grid_constant__ CUtensorMap map_o,    // O [B][T][C], box 64 x 128
                       const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sKV = sQ + kTileBytes;                 // stage s: K at s*64K, V at s*64K + 32K
  uint8_t *sP = sKV + 2 * kStageBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sP + kTileBytes);
  // bars: q_full, kv_full[2], kv_empty[2], s_full[2], s_empty[2], p_full, o_done, drain
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 12);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t q_full = smem_u32(bars + 0);
  auto kv_full = [&](int s) { return smem_u32(bars + 1 + s); };
  auto kv_empty = [&](int s) { return smem_u32(bars + 3 + s); };
  auto s_full = [&](int s) { return smem_u32(bars + 5 + s); };
  auto s_empty = [&](int s) { return smem_u32(bars + 7 + s); };
  const uint32_t p_full = smem_u32(bars + 9);
  const uint32_t o_done = smem_u32(bars + 10);
  const uint32_t drain = smem_u32(bars + 11);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = gridDim.x / p.n_qt;
  const int qt = p.n_qt - 1 - (int)blockIdx.x / BH;  // latest query tiles (most keys) first
  const int h = ((int)blockIdx.x % BH) % p.H, b = ((int)blockIdx.x % BH) / p.H;
  const int q0 = qt * kQ;
  const int n_kv = (min(q0 + kQ, p.T) + kKV - 1) / kKV;  // = qt + 1
  const int C = p.H * kD;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(s_empty(s), 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
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
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(kv_empty(st), ((j >> 1) & 1) ^ 1, abort_flag, p.status)) break;
        const uint32_t k_dst = smem_u32(sKV) + st * kStageBytes, v_dst = k_dst + kTileBytes;
        mbar_expect_tx(kv_full(st), kStageBytes);
        for (int i = 0; i < 2; ++i) tma_load_3d(k_dst + i * 16384, &map_qk, C + 64 * i, j * kKV, b, kv_full(st));
        for (int hh = 0; hh < 2; ++hh)
          for (int a = 0; a < 2; ++a)
            tma_load_3d(v_dst + hh * 16384 + a * 8192, &map_v, C + kD + 64 * a, j * kKV + 64 * hh, b, kv_full(st));
        ++issued;
      }
      // no copy of ours may still be landing when the CTA exits
      const uint64_t t0 = globaltimer();
      while (!mbar_try(q_full, 0) && globaltimer() - t0 < kWaitNs) {}
      for (int j = max(0, issued - 2); j < issued; ++j) {
        const uint64_t t1 = globaltimer();
        while (!mbar_try(kv_full(j & 1), (j >> 1) & 1) && globaltimer() - t1 < kWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc_s = make_idesc(0, 0, kQ, kKV);   // Q K^T: both K-major
      const uint32_t idesc_o = make_idesc(0, 1, kQ, kD);    // P V: V is MN-major
      const uint32_t aQ = smem_u32(sQ), aP = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(kv_full(st), (j >> 1) & 1, abort_flag, p.status)) return false;
        if (!mbar_wait(s_empty(st), ((j >> 1) & 1) ^ 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t bK = smem_u32(sKV) + st * kStageBytes;
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
          const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
          tc_mma(tmem + st * kKV, smem_desc(aQ + off, 16, 1024), smem_desc(bK + off, 16, 1024), idesc_s,
                 s > 0 ? 1u : 0u);
        }
        tc_commit(s_full(st));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv && !issue_s(j + 1)) break;
        if (!mbar_wait(p_full, j & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t bV = smem_u32(sKV) + (j & 1) * kStageBytes + kTileBytes;
#pragma unroll
        for (int s = 0; s < kKV / 16; ++s) {
          const uint32_t a_off = (s >> 2) * 16384 + (s & 3) * 32;    // P: K-major, k = keys
          const uint32_t b_off = (s >> 2) * 16384 + (s & 3) * 2048;  // V: MN-major, k rows
          tc_mma(tmem + 2 * kKV, smem_desc(aP + a_off, 16, 1024), smem_desc(bV + b_off, 8192, 1024), idesc_o,
                 (j > 0 || s > 0) ? 1u : 0u);
        }
        tc_commit(o_done);
        tc_commit(kv_empty(j & 1));
      }
      tc_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try(drain, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ---------------- softmax warps 2..5: thread = query row ----------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int row = q0 + r;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = rsqrtf((float)kD) * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j & 1;
      ok = mbar_wait(s_full(st), (j >> 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float s[kKV];
#pragma unroll
      for (int c = 0; c < kKV / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + st * kKV + c * 32, rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(rr[i]) * sc;
      }
      tc_fence_before();
      mbar_arrive(s_empty(st));
      const int kv0 = j * kKV;
      if (kv0 + kKV > q0 || kv0 + kKV > p.T) {
#pragma unroll
        for (int i = 0; i < kKV; ++i)
          if (kv0 + i > row || kv0 + i >= p.T) s[i] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kKV; ++i) mx = fmaxf(mx, s[i]);
      // P_{j-1} V_{j-1} must be done before P_j overwrites P and before O is touched
      if (j > 0) {
        ok = mbar_wait(o_done, (j - 1) & 1, abort_flag, p.status);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      const bool grow = mx > m_used + kRescaleLog2;
      if (j == 0) {
        m_used = mx;
      } else if (__any_sync(0xffffffffu, grow)) {
        const float corr = grow ? ex2(m_used - mx) : 1.f;
        if (grow) {
          l *= corr;
          m_used = mx;
        }
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(lane_base + 2 * kKV + c * 32, rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * corr);
          tmem_st32(lane_base + 2 * kKV + c * 32, rr);
        }
      }
      float sum = 0.f;
#pragma unroll
      for (int u = 0; u < kKV / 8; ++u) {
        float e[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          e[i] = ex2(s[8 * u + i] - m_used);
          sum += e[i];
        }
        uint4 w;
        w.x = pack2(e[0], e[1]);
        w.y = pack2(e[2], e[3]);
        w.z = pack2(e[4], e[5]);
        w.w = pack2(e[6], e[7]);
        *reinterpret_cast<uint4 *>(sP + tile_unit(r, u)) = w;
      }
      l += sum;
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // ---------------- epilogue: O / l, lse ----------------
    if (ok) ok = mbar_wait(o_done, (n_kv - 1) & 1, abort_flag, p.status);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(lane_base + 2 * kKV + c * 32, rr);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack2(__uint_as_float(rr[8 * u + 0]) * inv, __uint_as_float(rr[8 * u + 1]) * inv);
          w.y = pack2(__uint_as_float(rr[8 * u + 2]) * inv, __uint_as_float(rr[8 * u + 3]) * inv);
          w.z = pack2(__uint_as_float(rr[8 * u + 4]) * inv, __uint_as_float(rr[8 * u + 5]) * inv);
          w.w = pack2(__uint_as_float(rr[8 * u + 6]) * inv, __uint_as_float(rr[8 * u + 7]) * inv);
          *reinterpret_cast<uint4 *>(sQ + tile_unit(r, c * 4 + u)) = w;  // Q is no longer read
        }
      }
      if (row < p.T) p.lse[((int64_t)b * p.H + h) * p.T + row] = (m_used + __log2f(l)) * (1.f / kLog2e);
    }
    fence_proxy_async();
    asm volatile("bar.sync 1, 128;" ::: "memory");
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

inline cudaError_t init() {
  return cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
}

inline bool supported(const void *qkv, int64_t ld, const void *O) {
  return encode_fn() != nullptr && (ld % 8) == 0 && ((uintptr_t)qkv & 15) == 0 && ((uintptr_t)O & 15) == 0;
}

inline cudaError_t launch_fwd(const bf16 *qkv, int64_t ld, bf16 *O, float *lse, int B, int T, int H, int *status,
                              cudaStream_t st) {
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
  attn_fwd_tc_kernel<<<B * H * p.n_qt, kThreads, kSmem, st>>>(mqk, mv, mo, p);
  return cudaGetLastError();
}

}  // namespace fatc
}  // namespace nc
