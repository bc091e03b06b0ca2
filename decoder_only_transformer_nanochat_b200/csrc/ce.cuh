// Softcap + log-sum-exp + token cross-entropy, forward and backward fused, in
// place over the unembedding output z [M, ldz]:
//   s = 15 tanh(z / 15)             ("ten modern departures": logit softcap 15,
//                                     computed in fp32)
//   loss_i = logsumexp(s_i) - s_i[target_i]
//   dz = (softmax(s_i) - onehot(target_i)) (1 - (s/15)^2) / M   written over z
// No fp32 copy of the logits is ever materialised: each row is read once and
// written once.
#pragma once

#include "common.cuh"

namespace nc {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// tanh in the precision of the storage type: the hardware approximation
// (relative error ~2^-11) for bf16 logits, whose storage rounding (2^-9) is
// larger; the accurate library routine for fp32.
template <typename T> __device__ __forceinline__ float softcap_tanh(float x);
template <> __device__ __forceinline__ float softcap_tanh<bf16>(float x) { return tanh_fast(x); }
template <> __device__ __forceinline__ float softcap_tanh<float>(float x) { return tanhf(x); }
template <typename T> __device__ __forceinline__ float exp_t(float x);
template <> __device__ __forceinline__ float exp_t<bf16>(float x) { return ex2_fast(x * kLog2e); }
template <> __device__ __forceinline__ float exp_t<float>(float x) { return expf(x); }

// ---------------------------------------------------------------------------
// bf16 rows of V = 1024 threads * 8 * NVEC values (65,536 for NVEC = 8),
// persistent: one CTA per SM walks rows b, b + grid, ...  tanh(z/15) is kept
// per element as fp16 in registers (|t| <= 1, 11-bit mantissa: finer than the
// bf16 logit it came from).
// Each row (V bf16 = 128 KB at V = 65,536) arrives in shared memory by TMA
// bulk copies; as soon as every thread has its slice in registers the copy of
// the CTA's next row is issued, so the load of row i+1 and the store of dz for
// row i stream while row i's tanh / exp work runs.
constexpr int kCeThreads = 1024;
constexpr int kCeCopy = 32768;  // bytes per bulk copy

__device__ __forceinline__ bool ce_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok = 0;
  const uint64_t t0 = [] { uint64_t t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }();
  for (uint32_t i = 0;; ++i) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((i & 255) == 255) {
      uint64_t t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > 4000000000ull) return false;
    }
  }
}

__device__ __forceinline__ void ce_fetch_row(uint32_t dst, const bf16 *src, int bytes, uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  for (int o = 0; o < bytes; o += kCeCopy)
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst + o),
        "l"(reinterpret_cast<const uint8_t *>(src) + o), "r"(kCeCopy), "r"(bar)
        : "memory");
}

template <int NVEC>
__global__ void __launch_bounds__(kCeThreads, 1) ce_fused_bf16_persistent_kernel(
    bf16 *__restrict__ z, int64_t ldz, const int32_t *__restrict__ targets,
    float *__restrict__ token_loss, int M, int V, float inv_M, int *status) {
  extern __shared__ __align__(128) uint8_t ce_smem[];
  __shared__ float red[32];
  __shared__ float s_target;
  __shared__ __align__(8) uint64_t bar_storage;
  const uint32_t bar = static_cast<uint32_t>(__cvta_generic_to_shared(&bar_storage));
  const uint32_t buf = static_cast<uint32_t>(__cvta_generic_to_shared(ce_smem));
  const int row_bytes = V * 2;
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  int row = blockIdx.x;
  if (threadIdx.x == 0 && row < M) ce_fetch_row(buf, z + (size_t)row * ldz, row_bytes, bar);
  uint32_t phase = 0;
  for (; row < M; row += gridDim.x) {
    const bool ok = ce_wait(bar, phase);
    phase ^= 1;
    if (!__syncthreads_and(ok)) {
      if (threadIdx.x == 0) set_status(status, kStatusTimeout);
      break;
    }
    int tgt = targets[row];
    if (tgt < 0 || tgt >= V) {
      if (threadIdx.x == 0) set_status(status, kStatusRange);
      tgt = tgt < 0 ? 0 : V - 1;
    }
    if (threadIdx.x == 0) {
      // the target's softcapped logit, rounded exactly as in the sweep below
      const float zt = __bfloat162float(reinterpret_cast<const bf16 *>(ce_smem)[tgt]);
      s_target = kSoftcap * __half2float(__float2half_rn(tanh_fast(zt * (1.f / kSoftcap))));
    }
    __half2 t[NVEC][4];
    __half2 hmax = __float2half2_rn(-1.f);
#pragma unroll
    for (int k = 0; k < NVEC; ++k) {
      const uint4 zr = *reinterpret_cast<const uint4 *>(ce_smem + (threadIdx.x + k * kCeThreads) * 16);
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&zr);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h[j]);
        t[k][j] = __floats2half2_rn(tanh_fast(f.x * (1.f / kSoftcap)), tanh_fast(f.y * (1.f / kSoftcap)));
        hmax = __hmax2(hmax, t[k][j]);
      }
    }
    const float tmax = fmaxf(__low2float(hmax), __high2float(hmax));
    __syncthreads();  // the buffer is free: fetch the next row while this one is finished
    if (threadIdx.x == 0 && row + (int)gridDim.x < M)
      ce_fetch_row(buf, z + (size_t)(row + gridDim.x) * ldz, row_bytes, bar);
    const float smax2 = kSoftcap * kLog2e * block_max(tmax, red);
    // e = exp(s - smax); t is replaced by w = e (1 - t^2), the row's gradient
    // up to the factor 1 / (sum M), so the write-out needs no second
    // exponential (two MUFU operations per logit instead of three).  w lies in
    // [0, 1]; in fp16 it keeps 11 bits where it matters and flushes only
    // entries far below the bf16 resolution of the row's largest ones.
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < NVEC; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 r = __half22float2(t[k][j]);
        const float ea = ex2_fast(kSoftcap * kLog2e * r.x - smax2);
        const float eb = ex2_fast(kSoftcap * kLog2e * r.y - smax2);
        sum += ea + eb;
        t[k][j] = __floats2half2_rn(ea * (1.f - r.x * r.x), eb * (1.f - r.y * r.y));
      }
    sum = block_sum(sum, red);  // contains __syncthreads: s_target is visible after it
    const float lse2 = smax2 + __log2f(sum);  // log-sum-exp in the log2 domain
    if (threadIdx.x == 0) token_loss[row] = lse2 * kLn2 - s_target;
    const float scale = inv_M / sum;
    bf16 *zrow = z + (size_t)row * ldz;
#pragma unroll
    for (int k = 0; k < NVEC; ++k) {
      const int v = threadIdx.x + k * kCeThreads;
      uint4 u;
      __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 w = __half22float2(t[k][j]);
        h[j] = __floats2bfloat162_rn(w.x * scale, w.y * scale);
      }
      // the one-hot term of the target lives in exactly one thread's vector;
      // its p and 1 - t^2 come from the target's own softcapped logit
      if ((unsigned)(tgt - v * 8) < 8u) {
        const int j = (tgt - v * 8) >> 1;
        const float rt = s_target * (1.f / kSoftcap);
        const float pt = ex2_fast(kLog2e * s_target - lse2) - 1.f;
        const bf16 val = __float2bfloat16_rn(pt * (1.f - rt * rt) * inv_M);
        if (tgt & 1) h[j].y = val;
        else h[j].x = val;
      }
      *reinterpret_cast<uint4 *>(zrow + v * 8) = u;
    }
    __syncthreads();  // s_target and red are reused by the next row
  }
}

// ---------------------------------------------------------------------------
// General version, any V and either dtype: two sweeps over the row (the
// second is served by L2), online max/sum in the first.
template <typename T>
__global__ void __launch_bounds__(256) ce_fused_generic_kernel(
    T *__restrict__ z, int64_t ldz, const int32_t *__restrict__ targets,
    float *__restrict__ token_loss, int M, int V, float inv_M, int *status) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  if (row >= M) return;
  T *zr = z + (size_t)row * ldz;
  int tgt = targets[row];
  if (tgt < 0 || tgt >= V) {
    if (threadIdx.x == 0) set_status(status, kStatusRange);
    tgt = tgt < 0 ? 0 : V - 1;
  }
  float m = -INFINITY, l = 0.f;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    const float s = kSoftcap * softcap_tanh<T>(to_f(zr[v]) * (1.f / kSoftcap));
    if (s > m) {
      l = l * exp_t<T>(m - s) + 1.f;
      m = s;
    } else {
      l += exp_t<T>(s - m);
    }
  }
  const float gm = block_max(m, red);
  const float part = (m == -INFINITY) ? 0.f : l * exp_t<T>(m - gm);
  const float s_t = kSoftcap * softcap_tanh<T>(to_f(zr[tgt]) * (1.f / kSoftcap));
  const float tot = block_sum(part, red);  // syncs: every read of zr[tgt] precedes the writes
  const float lse = gm + logf(tot);
  if (threadIdx.x == 0) token_loss[row] = lse - s_t;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    const float tt = softcap_tanh<T>(to_f(zr[v]) * (1.f / kSoftcap));
    const float p = exp_t<T>(kSoftcap * tt - lse) - (v == tgt ? 1.f : 0.f);
    zr[v] = from_f<T>(p * (1.f - tt * tt) * inv_M);
  }
}

// loss = mean of the per-token losses; flags a non-finite result.
__global__ void __launch_bounds__(1024) loss_mean_kernel(const float *__restrict__ token_loss,
                                                         int M, float *__restrict__ loss,
                                                         int *status) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < M; i += blockDim.x) s += (double)token_loss[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) {
      const float r = (float)(s / (double)M);
      *loss = r;
      if (!isfinite(r)) set_status(status, kStatusNonFinite);
    }
  }
}

}  // namespace nc
