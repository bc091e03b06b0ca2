// bf16 GEMM on the 5th-generation tensor cores (sm_100a):
//   TMA (128-byte swizzle) -> 4-stage shared-memory ring -> tcgen05.mma
//   (cta_group::1, M=128, N=256, K=16, fp32 accumulate in TMEM) -> tcgen05.ld
//   -> fused epilogue -> global.
// Persistent: one CTA per SM walks a static list of (tile, k-split) units.
// Warp roles: warp 0 issues TMA, warp 1 owns TMEM and issues MMAs (one
// elected lane), warps 2..5 drain the accumulator (each warp reads the 32
// TMEM lanes its warp index selects).  Two TMEM accumulators (2 x 256 fp32
// columns) let the epilogue of one tile overlap the main loop of the next.
//
// Operand layouts (see gemm_common.cuh): a K-major operand is loaded as one
// box of [64 k x rows] (128 bytes of k per row, 8-row swizzle atoms of 1 KB);
// an MN-major operand as boxes of [64 mn x 64 k] (128 bytes of mn per k-row),
// stacked 8 KB apart along mn.  The shared-memory descriptors encode both
// canonical forms.
//
// Every wait is bounded: after kWaitNs without progress a CTA raises its
// abort flag, records kStatusTimeout in the status word, drains what it has
// in flight (again bounded), frees TMEM and returns.
#pragma once

#include <cuda.h>

#include "gemm_common.cuh"
#include "tc_common.cuh"

namespace nc {
namespace tc {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                // 16 KB
constexpr int B_BYTES = BN * BK * 2;                // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;      // 48 KB
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
// bf16 outputs leave through a 128 x 128 staging tile (two 64-column boxes of
// 128 rows x 128 B, 128-byte swizzle) written by TMA bulk stores
constexpr int STAGING_BYTES = 2 * BM * 128;          // 32 KB
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct Unit {
  int m_blk, n_blk, kb0, kb1;
};

struct Params {
  int M, N, K;
  int n_m, n_n;        // tile counts
  int splits, kblocks;  // k-splits per tile, k-blocks of BK in K
  int units;
  int a_mn, b_mn;
  void *D;
  int64_t ldd;
  int epi;
  int atomic_out;       // split-K: reduce fp32 output with red.global.add
  int *status;
};

__device__ __forceinline__ Unit unit_of(const Params &p, int u) {
  // Units in flight at once should share operand panels in L2.  k-splits are
  // the slowest index, so a wave works on one K slice of many tiles.  With
  // few N tiles the N tiles of an M block are consecutive (its A panel is read
  // once per wave); with many, tiles are grouped 16 M blocks at a time with M
  // fastest (each B panel serves 16 M blocks).
  const int tiles = p.n_m * p.n_n;
  const int split = u / tiles, tile = u % tiles;
  Unit x;
  if (p.n_n <= 16) {
    x.m_blk = tile / p.n_n;
    x.n_blk = tile % p.n_n;
  } else {
    const int G = 16;
    const int per_group = G * p.n_n;
    const int g = tile / per_group;
    const int first_m = g * G;
    const int gsize = min(p.n_m - first_m, G);
    const int r = tile % per_group;
    x.m_blk = first_m + r % gsize;
    x.n_blk = r / gsize;
  }
  const int per = (p.kblocks + p.splits - 1) / p.splits;
  x.kb0 = split * per;
  x.kb1 = min(p.kblocks, x.kb0 + per);
  return x;
}

// Epilogue of 32 consecutive columns [n, n+32) of row m.
__device__ __forceinline__ void epilogue_chunk(const Params &p, int m, int n, const uint32_t (&r)[32]) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (epi_f32(p.epi)) {
    float *d = reinterpret_cast<float *>(p.D) + (size_t)m * p.ldd + n;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int c = n + 4 * q;
      if (c + 4 <= p.N) {
        if (p.atomic_out) red_add_v4(d + 4 * q, v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        else *reinterpret_cast<float4 *>(d + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
        for (int j = 0; j < 4; ++j)
          if (c + j < p.N) {
            if (p.atomic_out) atomicAdd(d + 4 * q + j, v[4 * q + j]);
            else d[4 * q + j] = v[4 * q + j];
          }
      }
    }
    return;
  }
  bf16 *d = reinterpret_cast<bf16 *>(p.D) + (size_t)m * p.ldd + n;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = n + 8 * q;
    float o[8], old[8];
    const bool full = c + 8 <= p.N;
    if (p.epi == EPI_ADD || p.epi == EPI_DRELU2) {
      if (full) Vec8<bf16>::load(d + 8 * q, old);
      else
        for (int j = 0; j < 8; ++j) old[j] = (c + j < p.N) ? __bfloat162float(d[8 * q + j]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float a = v[8 * q + j];
      switch (p.epi) {
        case EPI_ADD: o[j] = old[j] + a; break;
        case EPI_RELU2: { const float t = fmaxf(a, 0.f); o[j] = t * t; } break;
        case EPI_DRELU2: o[j] = a * 2.f * sqrtf(old[j]); break;
        case EPI_SOFTCAP: o[j] = softcap_fast(a); break;
        default: o[j] = a; break;
      }
    }
    if (full) Vec8<bf16>::store(d + 8 * q, o);
    else
      for (int j = 0; j < 8; ++j)
        if (c + j < p.N) d[8 * q + j] = __float2bfloat16_rn(o[j]);
  }
}

// relu(h) = sqrt(relu(h)^2): the hardware approximation (relative error near
// 2^-23, exact 0 at 0) is far below the bf16 rounding of the result, and
// avoids the IEEE square root's slow path in the epilogue's inner loop.
__device__ __forceinline__ float sqrt_fast(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16 epilogue of 32 columns (chunk c of the 128-column half) of staging row r:
// 16-byte unit u of the row sits at (u ^ (r & 7)) within its 128-byte box row.
__device__ __forceinline__ void epilogue_stage(int epi, uint8_t *staging, int r, int c, const uint32_t (&acc)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int unit = c * 4 + q;  // 0..15 over the 128 columns
    uint8_t *ptr = staging + (unit >> 3) * (BM * 128) + r * 128 + (((unit & 7) ^ (r & 7)) << 4);
    float old[8], o[8];
    if (epi == EPI_ADD || epi == EPI_DRELU2) Vec8<bf16>::load(reinterpret_cast<const bf16 *>(ptr), old);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float a = __uint_as_float(acc[8 * q + j]);
      switch (epi) {
        case EPI_ADD: o[j] = old[j] + a; break;
        case EPI_RELU2: { const float t = fmaxf(a, 0.f); o[j] = t * t; } break;
        case EPI_DRELU2: o[j] = a * 2.f * sqrt_fast(old[j]); break;
        case EPI_SOFTCAP: o[j] = softcap_fast(a); break;
        default: o[j] = a; break;
      }
    }
    Vec8<bf16>::store(reinterpret_cast<bf16 *>(ptr), o);
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_d, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *staging = smem + STAGES * STAGE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(staging + STAGING_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain, aux
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 6);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * STAGES + 2 + a); };
  const uint32_t drain_bar = smem_u32(bars + 2 * STAGES + 4);
  const uint32_t aux_bar = smem_u32(bars + 2 * STAGES + 5);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    mbar_init(aux_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit x = unit_of(p, u);
        for (int kb = x.kb0; kb < x.kb1; ++kb) {
          if (!mbar_wait<true>(empty_bar(stage), phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          mbar_expect_tx(full_bar(stage), STAGE_BYTES);
          const int k0 = kb * BK;
          if (!p.a_mn) {
            tma_load_2d(sa, &map_a, k0, x.m_blk * BM, full_bar(stage));
          } else {
#pragma unroll
            for (int i = 0; i < BM / 64; ++i) tma_load_2d(sa + i * 8192, &map_a, x.m_blk * BM + 64 * i, k0, full_bar(stage));
          }
          if (!p.b_mn) {
            tma_load_2d(sb, &map_b, k0, x.n_blk * BN, full_bar(stage));
          } else {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i) tma_load_2d(sb + i * 8192, &map_b, x.n_blk * BN + 64 * i, k0, full_bar(stage));
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // make sure no copy of ours is still landing before the CTA can exit:
      // wait (bounded) on the last min(issued, STAGES) stages we filled
      for (int i = 0; i < min(issued, STAGES); ++i) {
        if (--stage < 0) { stage = STAGES - 1; phase ^= 1; }
        const uint64_t t0 = globaltimer();
        while (!mbar_try(full_bar(stage), phase) && globaltimer() - t0 < kWaitNs) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = make_idesc(p.a_mn, p.b_mn, BM, BN);
      // descriptor offsets: K-major -> SBO 1 KB (8-row atoms), k step 32 B;
      // MN-major -> LBO 8 KB (64-wide mn atoms), SBO 1 KB (8 k-rows), k step 2 KB
      const uint32_t a_lbo = p.a_mn ? 8192 : 16, a_sbo = 1024, a_kstep = p.a_mn ? 2048 : 32;
      const uint32_t b_lbo = p.b_mn ? 8192 : 16, b_sbo = 1024, b_kstep = p.b_mn ? 2048 : 32;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit x = unit_of(p, u);
        if (!mbar_wait<true>(tempty_bar(acc), acc_phase ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = x.kb0; kb < x.kb1; ++kb) {
          if (!mbar_wait<true>(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc(sa + kk * a_kstep, a_lbo, a_sbo);
            const uint64_t bd = smem_desc(sb + kk * b_kstep, b_lbo, b_sbo);
            tc_mma(d_tmem, ad, bd, idesc, (kb > x.kb0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // every MMA this thread issued has completed once the drain barrier flips
      tc_commit(drain_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try(drain_bar, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ---------------- epilogue warps 2..5 ----------------
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const int r = quarter * 32 + lane;  // tile row owned by this thread
    const bool leader = warp == 2 && lane == 0;  // issues the epilogue's TMA copies
    const bool f32_out = epi_f32(p.epi);
    const bool aux = p.epi == EPI_ADD || p.epi == EPI_DRELU2;
    const uint32_t st_addr = smem_u32(staging);
    int acc = 0;
    uint32_t acc_phase = 0, aux_phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const Unit x = unit_of(p, u);
      // every lane waits; the vote over all epilogue threads keeps their
      // branches (and named barriers) uniform and re-converges each warp
      ok = epi_vote_all(mbar_wait<true>(tfull_bar(acc), acc_phase, abort_flag, p.status));
      __syncwarp();
      if (!ok) break;
      tc_fence_after();
      const int m0 = x.m_blk * BM;
      const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      if (f32_out) {
        const int m = m0 + r;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int n = x.n_blk * BN + c * 32;
          if (n >= p.N) break;  // warp-uniform
          uint32_t rr[32];
          tmem_ld32(t_row + c * 32, rr);
          if (m < p.M) epilogue_chunk(p, m, n, rr);
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(acc));
      } else {
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          // half 0 always starts inside N; half 1 runs only if half 0 did not reach N
          const int n_half = x.n_blk * BN + half * 128;
          const bool box1 = n_half + 64 < p.N;
          if (leader) {
            bulk_wait_read0();  // the previous stores have finished reading the staging tile
            if (aux) {
              mbar_expect_tx(aux_bar, box1 ? 2 * BM * 128 : BM * 128);
              tma_load_2d(st_addr, &map_d, n_half, m0, aux_bar);
              if (box1) tma_load_2d(st_addr + BM * 128, &map_d, n_half + 64, m0, aux_bar);
            }
          }
          if (aux) {
            ok = epi_vote_all(mbar_wait<true>(aux_bar, aux_phase, abort_flag, p.status));
            aux_phase ^= 1;
            if (!ok) break;
          } else {
            epi_bar();
          }
          __syncwarp();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t rr[32];
            tmem_ld32(t_row + half * 128 + c * 32, rr);
            epilogue_stage(p.epi, staging, r, c, rr);
          }
          if (half == 1 || n_half + 128 >= p.N) {
            // accumulator fully read: hand TMEM back to the MMA warp
            tc_fence_before();
            mbar_arrive(tempty_bar(acc));
          }
          fence_proxy_async();
          epi_bar();
          if (leader) {
            tma_store_2d(&map_d, st_addr, n_half, m0);
            if (box1) tma_store_2d(&map_d, st_addr + BM * 128, n_half + 64, m0);
            bulk_commit();
          }
          if (n_half + 128 >= p.N) break;
        }
        if (!ok) break;
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (leader) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

// ===========================================================================
// Two-CTA version (cta_group::2): a cluster of 2 CTAs on neighbouring SMs
// computes a 256 x 256 tile.  CTA r owns rows [128r, 128r+128) of the tile
// (its A slice and its half of the accumulator) and loads half of B
// (tile columns [128r, 128r+128)); the leader (r = 0) issues every MMA, which
// reads A and B from both CTAs' shared memory.  Per SM a k-block moves 32 KB
// instead of 48 KB for the same flops, so six stages fit (five, plus a second
// staging tile, for the epilogues that read their output tile first) and L2
// traffic for the B operand halves.  Both CTAs' TMA loads complete on the leader's "full"
// barrier; the leader's commits arrive on both CTAs' "empty" and "tmem full"
// barriers; both CTAs' epilogue threads release the accumulator on the
// leader's "tmem empty" barrier.
constexpr int BN2 = 256, BH2 = 128;                  // tile N, B rows per CTA
constexpr int STAGES2 = 6;
// Eight epilogue warps (2..9): two per TMEM lane quarter (warp % 4), each
// taking one of the two column groups of every half tile, so an epilogue
// that reads its output tile first keeps pace with the main loop.
constexpr int EPI_WARPS2 = 8;
constexpr int NUM_THREADS2 = 64 + 32 * EPI_WARPS2;
constexpr int STAGE_BYTES2 = A_BYTES + BH2 * BK * 2;  // 32 KB
constexpr int SMEM_BYTES2 = STAGES2 * STAGE_BYTES2 + STAGING_BYTES + 1024 + 256;
static_assert(SMEM_BYTES2 <= 232448, "shared memory per CTA");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// arrive on the barrier at the same offset in CTA `rank` of the cluster
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar, uint32_t rank) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(bar),
      "r"(rank)
      : "memory");
}
// shared::cluster address of the location at this offset in CTA `rank`
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// TMA load into this CTA's shared memory whose completion is counted on the
// barrier `bar_cluster` (a shared::cluster address: the pair leader's barrier)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// commit of the pair's MMAs, arriving on the barrier at this offset in every CTA of `mask`.
// This is an mbarrier arrive inside the 2-CTA cluster of this GPU, not a
// load: no TMA or bulk copy in this file uses cluster multicast.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// barrier, and barrier with an AND vote, among the 256 epilogue threads of the two-CTA kernel
__device__ __forceinline__ void epi_bar2() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ bool epi_vote_all2(bool v) {
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

__device__ __forceinline__ Unit unit_of2(const Params &p, int u) {
  // p.n_m counts 256-row blocks here
  return unit_of(p, u);
}

__global__ void __launch_bounds__(NUM_THREADS2, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const __grid_constant__ CUtensorMap map_d, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *staging = smem + STAGES2 * STAGE_BYTES2;
  uint64_t *bars = reinterpret_cast<uint64_t *>(staging + STAGING_BYTES);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain, aux[2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES2 + 7);
  static_assert((2 * STAGES2 + 7) * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit their 256 bytes");
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES2 + s); };
  auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * STAGES2 + a); };
  auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * STAGES2 + 2 + a); };
  const uint32_t drain_bar = smem_u32(bars + 2 * STAGES2 + 4);
  auto aux_bar = [&](int b) { return smem_u32(bars + 2 * STAGES2 + 5 + b); };
  // An epilogue that reads its output tile first (residual add, relu^2
  // backward) runs the ring with one stage fewer and takes that stage's 32 KB
  // as a second staging tile: the input of the next half tile loads into one
  // while the current half is computed and stored from the other.
  const bool aux_pipe = (p.epi == EPI_ADD || p.epi == EPI_DRELU2) && !epi_f32(p.epi);
  const int nst = aux_pipe ? STAGES2 - 1 : STAGES2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * 32 * EPI_WARPS2);  // both CTAs' epilogue threads
    }
    mbar_init(drain_bar, 1);
    mbar_init(aux_bar(0), 1);
    mbar_init(aux_bar(1), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int u = cluster; u < p.units && ok; u += n_clusters) {
        const Unit x = unit_of2(p, u);
        const int m_row = x.m_blk * 256 + (int)rank * BM;
        const int n_row = x.n_blk * BN2 + (int)rank * BH2;
        for (int kb = x.kb0; kb < x.kb1; ++kb) {
          if (!mbar_wait<true>(empty_bar(stage), phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES2);
          const uint32_t sb = sa + A_BYTES;
          if (leader) mbar_expect_tx(full_bar(stage), 2 * STAGE_BYTES2);
          const uint32_t fb = cluster_addr(full_bar(stage), 0);
          const int k0 = kb * BK;
          if (!p.a_mn) {
            tma_load_2d_pair(sa, &map_a, k0, m_row, fb);
          } else {
#pragma unroll
            for (int i = 0; i < BM / 64; ++i) tma_load_2d_pair(sa + i * 8192, &map_a, m_row + 64 * i, k0, fb);
          }
          if (!p.b_mn) {
            tma_load_2d_pair(sb, &map_b, k0, n_row, fb);
          } else {
#pragma unroll
            for (int i = 0; i < BH2 / 64; ++i) tma_load_2d_pair(sb + i * 8192, &map_b, n_row + 64 * i, k0, fb);
          }
          ++issued;
          if (++stage == nst) { stage = 0; phase ^= 1; }
        }
      }
      // our copies complete on the leader's barriers; every one of them is
      // consumed by an MMA before the leader's final commit, which the final
      // cluster barrier orders before either CTA exits
      (void)issued;
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = make_idesc(p.a_mn, p.b_mn, 256, BN2);
      const uint32_t a_lbo = p.a_mn ? 8192 : 16, a_kstep = p.a_mn ? 2048 : 32;
      const uint32_t b_lbo = p.b_mn ? 8192 : 16, b_kstep = p.b_mn ? 2048 : 32;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = cluster; u < p.units && ok; u += n_clusters) {
        const Unit x = unit_of2(p, u);
        if (!mbar_wait<true>(tempty_bar(acc), acc_phase ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN2;
        for (int kb = x.kb0; kb < x.kb1; ++kb) {
          if (!mbar_wait<true>(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES2);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_pair(d_tmem, smem_desc(sa + kk * a_kstep, a_lbo, 1024), smem_desc(sb + kk * b_kstep, b_lbo, 1024),
                        idesc, (kb > x.kb0 || kk > 0) ? 1u : 0u);
          tc_commit_pair(empty_bar(stage), 0x3);
          if (++stage == nst) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair(tfull_bar(acc), 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      tc_commit_pair(drain_bar, 0x1);
      const uint64_t t0 = globaltimer();
      while (!mbar_try(drain_bar, 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ---------------- epilogue warps 2..9 (both CTAs) ----------------
    const int quarter = warp & 3;
    const int cg = (warp - 2) >> 2;  // column group: chunks [2 cg, 2 cg + 2) of each half tile
    const int r = quarter * 32 + lane;
    const bool ep_leader = warp == 2 && lane == 0;
    const bool f32_out = epi_f32(p.epi);
    const bool aux = aux_pipe;
    // staging tile 0 is the one after the ring; tile 1 (aux epilogues only)
    // is the ring's last stage, which their ring does not use
    auto stg_tile = [&](int b) { return b ? smem + (STAGES2 - 1) * STAGE_BYTES2 : staging; };
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t aux_phases = 0;    // bit b: the phase of aux_bar(b)
    int halves = 0;             // half tiles this CTA has taken (their staging tile alternates)
    uint32_t aux_inflight = 0;  // ep_leader, bit b: a load into tile b not yet waited for
    bool ok = true;
    auto release_tmem = [&](int a) {
      tc_fence_before();
      if (leader) mbar_arrive(tempty_bar(a));
      else mbar_arrive_remote(tempty_bar(a), 0);
    };
    // ep_leader: this CTA's rows of half `hh` of unit `uu`, read from D into staging tile `b`
    auto load_aux = [&](int uu, int hh, int b) {
      const Unit y = unit_of2(p, uu);
      const int ym0 = y.m_blk * 256 + (int)rank * BM;
      const int yn = y.n_blk * BN2 + hh * 128;
      const bool yb1 = yn + 64 < p.N;
      const uint32_t dst = smem_u32(stg_tile(b));
      mbar_expect_tx(aux_bar(b), yb1 ? 2 * BM * 128 : BM * 128);
      tma_load_2d(dst, &map_d, yn, ym0, aux_bar(b));
      if (yb1) tma_load_2d(dst + BM * 128, &map_d, yn + 64, ym0, aux_bar(b));
      aux_inflight |= 1u << b;
    };
    if (aux && ep_leader && cluster < p.units) load_aux(cluster, 0, 0);
    for (int u = cluster; u < p.units && ok; u += n_clusters) {
      const Unit x = unit_of2(p, u);
      ok = epi_vote_all2(mbar_wait<true>(tfull_bar(acc), acc_phase, abort_flag, p.status));
      __syncwarp();
      if (!ok) break;
      tc_fence_after();
      const int m0 = x.m_blk * 256 + (int)rank * BM;
      const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN2;
      if (f32_out) {
        const int m = m0 + r;
#pragma unroll 1
        for (int c = 4 * cg; c < 4 * cg + 4; ++c) {
          const int n = x.n_blk * BN2 + c * 32;
          if (n >= p.N) break;  // warp-uniform
          uint32_t rr[32];
          tmem_ld32(t_row + c * 32, rr);
          if (m < p.M) epilogue_chunk(p, m, n, rr);
        }
        release_tmem(acc);
      } else {
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const int n_half = x.n_blk * BN2 + half * 128;
          const bool box1 = n_half + 64 < p.N;
          const bool last_half = half == 1 || n_half + 128 >= p.N;
          const int b = aux ? (halves & 1) : 0;
          uint8_t *const stg = stg_tile(b);
          const uint32_t st_addr = smem_u32(stg);
          if (aux) {
            if (ep_leader) {
              // the next half tile's input goes to the other staging tile as
              // soon as the store that last read it (the previous half's) is done
              const int nu = last_half ? u + n_clusters : u, nh = last_half ? 0 : 1;
              if (nu < p.units) {
                bulk_wait_read0();
                load_aux(nu, nh, b ^ 1);
              }
            }
            ok = epi_vote_all2(mbar_wait<true>(aux_bar(b), (aux_phases >> b) & 1u, abort_flag, p.status));
            if (!ok) break;
            aux_phases ^= 1u << b;
            aux_inflight &= ~(1u << b);
            ++halves;
          } else {
            if (ep_leader) bulk_wait_read0();  // the previous stores have read the staging tile
            epi_bar2();
          }
          __syncwarp();
#pragma unroll 1
          for (int c = 2 * cg; c < 2 * cg + 2; ++c) {
            uint32_t rr[32];
            tmem_ld32(t_row + half * 128 + c * 32, rr);
            epilogue_stage(p.epi, stg, r, c, rr);
          }
          if (last_half) release_tmem(acc);
          fence_proxy_async();
          epi_bar2();
          if (ep_leader) {
            tma_store_2d(&map_d, st_addr, n_half, m0);
            if (box1) tma_store_2d(&map_d, st_addr + BM * 128, n_half + 64, m0);
            bulk_commit();
          }
          if (n_half + 128 >= p.N) break;
        }
        if (!ok) break;
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    if (ep_leader) {
      bulk_wait0();
      // only after an abort: loads issued for halves that were never taken
      // land before the CTA's shared memory goes away (bounded)
      for (int b = 0; b < 2; ++b) {
        if (!((aux_inflight >> b) & 1u)) continue;
        const uint64_t t0 = globaltimer();
        while (!mbar_try(aux_bar(b), (aux_phases >> b) & 1u) && globaltimer() - t0 < kWaitNs) {}
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer can still signal or read it
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------- host side -------------------------------

// 2D bf16 map over a row-major [rows, cols] matrix with row stride ld
// elements; box = box_cols (innermost, 64 = 128 bytes) x box_rows.
inline bool make_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int64_t ld,
                     int box_cols, int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Split K over several units when the tile count would leave SMs idle:
// choose the split count that best fills whole waves, with a small cost per
// extra split (each split adds one fp32 reduction pass over the tile).
inline int choose_splits(int tiles, int kblocks, int num_sms) {
  if (tiles >= 2 * num_sms) return 1;
  int best = 1;
  double best_score = -1.0;
  for (int s = 1; s <= 16; ++s) {
    if (s > 1 && kblocks / s < 8) break;
    const int units = tiles * s;
    const int waves = (units + num_sms - 1) / num_sms;
    const double eff = (double)units / (double)(waves * num_sms);
    const double score = eff - 0.015 * (s - 1);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = s;
    }
  }
  return best;
}

}  // namespace tc

inline cudaError_t tc_init() {
  if (!tc::encode_fn()) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    tc::encode_fn() = reinterpret_cast<tc::EncodeTiledFn>(fn);
  }
  cudaError_t e = cudaFuncSetAttribute(tc::gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       tc::SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tc::gemm_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES2);
  return e;
}

// Operands the TMA tiles can take: 16-byte aligned bases and row strides.
inline bool tc_gemm_aligned(const GemmProblem &p) {
  if (p.M < 1 || p.N < 1 || p.K < 1) return false;
  if ((p.lda % 8) || (p.ldb % 8)) return false;
  if (((uintptr_t)p.A & 15) || ((uintptr_t)p.B & 15) || ((uintptr_t)p.D & 15)) return false;
  if (epi_f32(p.epi) ? (p.ldd % 4) : (p.ldd % 8)) return false;
  return true;
}

template <typename T>
inline bool tc_gemm_supported(const GemmProblem &p) {
  return sizeof(T) == 2 && tc_gemm_aligned(p) && tc::encode_fn() != nullptr;
}

inline cudaError_t launch_gemm_tc2(const GemmProblem &g, int num_sms, int *status, cudaStream_t st);

// pair = 1: the two-CTA kernel (M >= 256), pair = 0: the one-CTA kernel
inline cudaError_t launch_gemm_tc(const GemmProblem &g, int num_sms, int *status, cudaStream_t st,
                                  int pair = 1) {
  if (pair && g.M >= 256) return launch_gemm_tc2(g, num_sms, status, st);
  using namespace tc;
  CUtensorMap ma, mb;
  bool ok;
  if (!g.a_mn) ok = make_map(&ma, g.A, g.M, g.K, g.lda, 64, BM);
  else ok = make_map(&ma, g.A, g.K, g.M, g.lda, 64, 64);
  if (!ok) return cudaErrorInvalidValue;
  if (!g.b_mn) ok = make_map(&mb, g.B, g.N, g.K, g.ldb, 64, BN);
  else ok = make_map(&mb, g.B, g.K, g.N, g.ldb, 64, 64);
  if (!ok) return cudaErrorInvalidValue;
  CUtensorMap md = ma;  // fp32 outputs are written directly; the map is unused
  if (!epi_f32(g.epi) && !make_map(&md, g.D, g.M, g.N, g.ldd, 64, BM)) return cudaErrorInvalidValue;
  Params p;
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.n_m = (g.M + BM - 1) / BM;
  p.n_n = (g.N + BN - 1) / BN;
  p.kblocks = (g.K + BK - 1) / BK;
  const int tiles = p.n_m * p.n_n;
  p.splits = epi_f32(g.epi) ? choose_splits(tiles, p.kblocks, num_sms) : 1;
  {
    // every split must own at least one k-block
    const int per = (p.kblocks + p.splits - 1) / p.splits;
    p.splits = (p.kblocks + per - 1) / per;
  }
  p.units = tiles * p.splits;
  p.a_mn = g.a_mn; p.b_mn = g.b_mn;
  p.D = g.D; p.ldd = g.ldd; p.epi = g.epi;
  // split-K partial sums, and accumulation into an existing D, add with red.global.add
  p.atomic_out = p.splits > 1 || g.epi == EPI_ACC_F32;
  p.status = status;
  if (p.splits > 1 && g.epi == EPI_STORE_F32) {
    // fp32 partial sums are added into a zeroed output
    cudaError_t e = cudaMemset2DAsync(g.D, (size_t)g.ldd * 4, 0, (size_t)g.N * 4, (size_t)g.M, st);
    if (e != cudaSuccess) return e;
  }
  const int grid = p.units < num_sms ? p.units : num_sms;
  gemm_tc_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(ma, mb, md, p);
  return cudaGetLastError();
}

}  // namespace nc

namespace nc {

inline cudaError_t launch_gemm_tc2(const GemmProblem &g, int num_sms, int *status, cudaStream_t st) {
  using namespace tc;
  CUtensorMap ma, mb;
  bool ok;
  if (!g.a_mn) ok = make_map(&ma, g.A, g.M, g.K, g.lda, 64, BM);
  else ok = make_map(&ma, g.A, g.K, g.M, g.lda, 64, 64);
  if (!ok) return cudaErrorInvalidValue;
  if (!g.b_mn) ok = make_map(&mb, g.B, g.N, g.K, g.ldb, 64, BH2);
  else ok = make_map(&mb, g.B, g.K, g.N, g.ldb, 64, 64);
  if (!ok) return cudaErrorInvalidValue;
  CUtensorMap md = ma;
  if (!epi_f32(g.epi) && !make_map(&md, g.D, g.M, g.N, g.ldd, 64, BM)) return cudaErrorInvalidValue;
  Params p;
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.n_m = (g.M + 255) / 256;
  p.n_n = (g.N + BN2 - 1) / BN2;
  p.kblocks = (g.K + BK - 1) / BK;
  const int n_clusters = num_sms / 2;
  const int tiles = p.n_m * p.n_n;
  p.splits = epi_f32(g.epi) ? choose_splits(tiles, p.kblocks, n_clusters) : 1;
  {
    const int per = (p.kblocks + p.splits - 1) / p.splits;
    p.splits = (p.kblocks + per - 1) / per;
  }
  p.units = tiles * p.splits;
  p.a_mn = g.a_mn; p.b_mn = g.b_mn;
  p.D = g.D; p.ldd = g.ldd; p.epi = g.epi;
  // split-K partial sums, and accumulation into an existing D, add with red.global.add
  p.atomic_out = p.splits > 1 || g.epi == EPI_ACC_F32;
  p.status = status;
  if (p.splits > 1 && g.epi == EPI_STORE_F32) {
    cudaError_t e = cudaMemset2DAsync(g.D, (size_t)g.ldd * 4, 0, (size_t)g.N * 4, (size_t)g.M, st);
    if (e != cudaSuccess) return e;
  }
  const int clusters = p.units < n_clusters ? p.units : n_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(NUM_THREADS2);
  cfg.dynamicSmemBytes = SMEM_BYTES2;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel, ma, mb, md, p);
}

}  // namespace nc
