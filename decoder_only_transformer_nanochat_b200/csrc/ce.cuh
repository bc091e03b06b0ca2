// Softcap + log-sum-exp + token cross-entropy, forward and backward fused, in
// place over the unembedding output z [M, ldz]:
//   s = 15 tanh(z / 15)             ("ten modern departures": logit softcap 15,
//                                     computed in fp32)
//   loss_i = logsumexp(s_i) - s_i[target_i]
//   dz = (softmax(s_i) - onehot(target_i)) (1 - (s/15)^2) g   written over z
// with g the gradient scale (1/M for the mean loss).  No fp32 copy of the
// logits is ever materialised: each row is read once and written once.
//
// Precision.  tanh and 1 - tanh^2 are formed to fp32 accuracy from one
// exponential, E = exp(-2|x|), x = z/15:
//   u = 1 - |t| = 2E / (1 + E),   t = sign(x)(1 - u),   1 - t^2 = u (2 - u),
// so 1 - t^2 keeps its relative precision where tanh saturates (a hardware
// tanh of relative error 2^-11 would leave it none at |z| ~ 45).  The row
// max comes from the raw logits (tanh is increasing).  The target's term is
// kept out of the running sum, so 1 - p_target = rest / (rest + e_target)
// has no cancellation when the target dominates the row.
#pragma once

#include "common.cuh"

namespace nc {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// t = tanh(z/15) and 1 - t^2 for a bf16 model: E by the MUFU exponential
// (relative error ~2^-22), 1/(1+E) on the FMA pipe by three Newton steps from
// the best linear guess on [1, 2] (relative error 1/17, squared by each step).
__device__ __forceinline__ void softcap_parts_fast(float z, float &t, float &sech2) {
  const float E = ex2_fast(fabsf(z) * (-2.f * kLog2e / kSoftcap));
  const float y = 1.f + E;
  float r = fmaf(-8.f / 17.f, y, 24.f / 17.f);
  r = fmaf(r, fmaf(-y, r, 1.f), r);
  r = fmaf(r, fmaf(-y, r, 1.f), r);
  r = fmaf(r, fmaf(-y, r, 1.f), r);
  const float u = 2.f * E * r;
  t = copysignf(1.f - u, z);
  sech2 = u * (2.f - u);
}

// The same for two logits at once, the FMA-pipe steps in packed f32x2 form
// (each lane rounds exactly as the scalar form above, so the results are
// bit-identical to two softcap_parts_fast calls).
__device__ __forceinline__ void softcap_parts_fast2(float za, float zb, float &ta, float &tb, float &sa,
                                                    float &sb) {
  constexpr float c = -2.f * kLog2e / kSoftcap;
  const uint64_t E = f2(ex2_fast(fabsf(za) * c), ex2_fast(fabsf(zb) * c));
  const uint64_t one = f2(1.f, 1.f), m1 = f2(-1.f, -1.f);
  const uint64_t y = add2(one, E);
  const uint64_t ny = fma2(E, m1, m1);  // -(1 + E), exactly
  uint64_t r = fma2(f2(-8.f / 17.f, -8.f / 17.f), y, f2(24.f / 17.f, 24.f / 17.f));
  r = fma2(r, fma2(ny, r, one), r);
  r = fma2(r, fma2(ny, r, one), r);
  r = fma2(r, fma2(ny, r, one), r);
  const uint64_t two = f2(2.f, 2.f);
  const uint64_t u = mul2(mul2(two, E), r);
  float va, vb;
  f2split(fma2(u, m1, one), va, vb);  // 1 - u
  ta = copysignf(va, za);
  tb = copysignf(vb, zb);
  f2split(mul2(u, fma2(u, m1, two)), sa, sb);  // u (2 - u)
}

// Two floats packed into one 32-bit register as fp16 / bf16 (lo in the low half).
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ float2 unpack_h2(uint32_t u) {
  __half2 h;
  memcpy(&h, &u, 4);
  return __half22float2(h);
}
__device__ __forceinline__ float2 unpack_bf2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// The same for an fp32 model with the library's accurate exponential and a
// correctly rounded division.
__device__ __forceinline__ void softcap_parts_precise(float z, float &t, float &sech2) {
  const float E = expf(fabsf(z) * (-2.f / kSoftcap));
  const float u = 2.f * E / (1.f + E);
  t = copysignf(1.f - u, z);
  sech2 = u * (2.f - u);
}

template <typename T> __device__ __forceinline__ void softcap_parts(float z, float &t, float &sech2);
template <> __device__ __forceinline__ void softcap_parts<bf16>(float z, float &t, float &s2) {
  softcap_parts_fast(z, t, s2);
}
template <> __device__ __forceinline__ void softcap_parts<float>(float z, float &t, float &s2) {
  softcap_parts_precise(z, t, s2);
}
template <typename T> __device__ __forceinline__ float exp_t(float x);
template <> __device__ __forceinline__ float exp_t<bf16>(float x) { return ex2_fast(x * kLog2e); }
template <> __device__ __forceinline__ float exp_t<float>(float x) { return expf(x); }

// ---------------------------------------------------------------------------
// bf16 rows of V <= 1024 threads * 8 * NVEC values, V % 8 == 0, persistent:
// one CTA per SM walks rows b, b + grid, ...  Each row (V bf16 = 128 KB at
// V = 65,536) arrives in shared memory by TMA bulk copies; as soon as every
// thread has its slice in registers the copy of the CTA's next row is
// issued, so the load of row i+1 and the store of dz for row i stream while
// row i's exponentials run.  Per thread the raw logits, then w = e (1 - t^2)
// (fp16, w <= 1), are kept packed in registers.  A row takes two block-wide
// barriers: one publishes the warps' maxima (and frees the buffer), one their
// sums.  The small shared values alternate between two slots by row parity,
// so a warp that has stored its part of row i goes on to row i+1 without
// waiting for the others; the next row's target id is read a row ahead.
constexpr int kCeThreads = 1024;
constexpr int kCeCopy = 32768;  // bytes per bulk copy

__device__ __forceinline__ bool ce_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok = 0;
  const uint64_t t0 = [] { uint64_t t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }();
  for (uint32_t i = 0;; ++i) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "n"(1u << 20)  // sleep in hardware until the row lands (<= ~1 ms)
        : "memory");
    if (ok) return true;
    if ((i & 15) == 15) {
      uint64_t t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > 4000000000ull) return false;
    }
  }
}

// One row of `bytes` (a multiple of 16) into shared memory, in copies of at
// most kCeCopy bytes, completing on `bar`.
__device__ __forceinline__ void ce_fetch_row(uint32_t dst, const bf16 *src, int bytes, uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  for (int o = 0; o < bytes; o += kCeCopy) {
    const int n = bytes - o < kCeCopy ? bytes - o : kCeCopy;
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst + o),
        "l"(reinterpret_cast<const uint8_t *>(src) + o), "r"(n), "r"(bar)
        : "memory");
  }
}

template <int NVEC>
__global__ void __launch_bounds__(kCeThreads, 1) ce_fused_bf16_persistent_kernel(
    bf16 *__restrict__ z, int64_t ldz, const int32_t *__restrict__ targets,
    float *__restrict__ token_loss, int M, int V, float grad_scale, int *status) {
  extern __shared__ __align__(128) uint8_t ce_smem[];
  constexpr int kWarps = kCeThreads / 32;
  static_assert(kWarps == 32, "one warp reads every warp's partial, one per lane");
  __shared__ float red_max[2][kWarps], red_sum[2][kWarps];
  __shared__ float s_target[2], sech2_target[2];
  __shared__ __align__(8) uint64_t bar_storage;
  const uint32_t bar = static_cast<uint32_t>(__cvta_generic_to_shared(&bar_storage));
  const uint32_t buf = static_cast<uint32_t>(__cvta_generic_to_shared(ce_smem));
  const int row_bytes = V * 2;
  const int n8 = V >> 3;  // 16-byte chunks of a row
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  int row = blockIdx.x;
  if (threadIdx.x == 0 && row < M) ce_fetch_row(buf, z + (size_t)row * ldz, row_bytes, bar);
  uint32_t phase = 0;
  const float k2 = kSoftcap * kLog2e;
  int tgt_next = row < M ? targets[row] : 0;
  for (int par = 0; row < M; row += gridDim.x, par ^= 1) {
    int tgt = tgt_next;
    if (row + (int)gridDim.x < M) tgt_next = targets[row + gridDim.x];  // used by the next row
    const bool ok = ce_wait(bar, phase);
    phase ^= 1;
    if (tgt < 0 || tgt >= V) {
      if (threadIdx.x == 0) set_status(status, kStatusRange);
      tgt = tgt < 0 ? 0 : V - 1;
    }
    if (threadIdx.x == 0) {
      float tt, s2;
      softcap_parts_fast(__bfloat162float(reinterpret_cast<const bf16 *>(ce_smem)[tgt]), tt, s2);
      s_target[par] = kSoftcap * tt;
      sech2_target[par] = s2;
    }
    // raw logits into registers, their max (tanh is increasing)
    uint32_t pk[NVEC][4];
    __nv_bfloat162 hmax = __float2bfloat162_rn(-INFINITY);
#pragma unroll
    for (int k = 0; k < NVEC; ++k) {
      const int c = threadIdx.x + k * kCeThreads;
      if (c < n8) {
        const uint4 u = *reinterpret_cast<const uint4 *>(ce_smem + c * 16);
        pk[k][0] = u.x; pk[k][1] = u.y; pk[k][2] = u.z; pk[k][3] = u.w;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __nv_bfloat162 h;
          memcpy(&h, &pk[k][j], 4);
          hmax = __hmax2(hmax, h);
        }
      }
    }
    {
      const float wm = warp_max(fmaxf(__low2float(hmax), __high2float(hmax)));
      if (lane == 0) red_max[par][wid] = wm;
    }
    // every slice is in registers (the buffer may take the next row), the
    // warps' maxima and the target's terms are visible, and all threads agree
    // that the row arrived
    if (!__syncthreads_and(ok)) {
      if (threadIdx.x == 0) set_status(status, kStatusTimeout);
      break;
    }
    if (threadIdx.x == 0 && row + (int)gridDim.x < M)
      ce_fetch_row(buf, z + (size_t)(row + gridDim.x) * ldz, row_bytes, bar);
    const float zmax = warp_max(red_max[par][lane]);
    float tmax, s2max;
    softcap_parts_fast(zmax, tmax, s2max);
    const float m2 = k2 * tmax;  // row max of s, log2 domain
    // e = exp(s - max) summed without the target's term; w = e (1 - t^2)
    // replaces the logits (the row's gradient up to 1 / sum)
    float rest = 0.f;
#pragma unroll
    for (int k = 0; k < NVEC; ++k) {
      const int c = threadIdx.x + k * kCeThreads;
      if (c < n8) {
        float e[8], part = 0.f;
        uint64_t part2 = f2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_bf2(pk[k][j]);
          float ta, sa, tb, sb;
          softcap_parts_fast2(f.x, f.y, ta, tb, sa, sb);
          float xa, xb;
          f2split(fma2(f2(k2, k2), f2(ta, tb), f2(-m2, -m2)), xa, xb);
          e[2 * j] = ex2_fast(xa);
          e[2 * j + 1] = ex2_fast(xb);
          const uint64_t ee = f2(e[2 * j], e[2 * j + 1]);
          part2 = add2(part2, ee);
          float wa, wb;
          f2split(mul2(ee, f2(sa, sb)), wa, wb);
          pk[k][j] = pack_h2(wa, wb);
        }
        {
          float pa, pb;
          f2split(part2, pa, pb);
          part = pa + pb;
        }
        if ((unsigned)(tgt - c * 8) < 8u) {  // the target's chunk: its term stays out
          part = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c * 8 + j != tgt) part += e[j];
        }
        rest += part;
      }
    }
    {
      const float ws = warp_sum(rest);
      if (lane == 0) red_sum[par][wid] = ws;
    }
    __syncthreads();
    rest = warp_sum(red_sum[par][lane]);
    const float s_t = s_target[par];
    const float e_t = ex2_fast(fmaf(kLog2e, s_t, -m2));
    const float sum = rest + e_t;
    const float lse2 = m2 + __log2f(sum);  // log-sum-exp in the log2 domain
    if (threadIdx.x == 0) token_loss[row] = lse2 * kLn2 - s_t;
    const float scale = grad_scale / sum;
    // 1 - p_target = rest / sum: no cancellation when the target dominates
    const bf16 dz_t = __float2bfloat16_rn(-(rest / sum) * sech2_target[par] * grad_scale);
    bf16 *zrow = z + (size_t)row * ldz;
#pragma unroll
    for (int k = 0; k < NVEC; ++k) {
      const int c = threadIdx.x + k * kCeThreads;
      if (c < n8) {
        uint32_t o[4];
        const uint64_t scale2 = f2(scale, scale);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack_h2(pk[k][j]);
          float oa, ob;
          f2split(mul2(f2(f.x, f.y), scale2), oa, ob);
          o[j] = pack_bf2(oa, ob);
        }
        if ((unsigned)(tgt - c * 8) < 8u) {
          const int j = (tgt - c * 8) >> 1;
          const uint32_t b = __bfloat16_as_ushort(dz_t);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            if (jj == j) o[jj] = (tgt & 1) ? ((o[jj] & 0xffffu) | (b << 16)) : ((o[jj] & 0xffff0000u) | b);
        }
        const uint4 u = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4 *>(zrow + c * 8) = u;
      }
    }
    // no barrier here: the next row writes the other parity's slots, and this
    // row's slots are rewritten only after both of the next row's barriers
  }
}

// ---------------------------------------------------------------------------
// General version, any V and either dtype: three sweeps over the row (the
// second and third are served by L2): the max of the raw logits, the sum of
// exp(s - max) without the target's term, the write-out.
template <typename T>
__global__ void __launch_bounds__(256) ce_fused_generic_kernel(
    T *__restrict__ z, int64_t ldz, const int32_t *__restrict__ targets,
    float *__restrict__ token_loss, int M, int V, float grad_scale, int *status) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  if (row >= M) return;
  T *zr = z + (size_t)row * ldz;
  int tgt = targets[row];
  if (tgt < 0 || tgt >= V) {
    if (threadIdx.x == 0) set_status(status, kStatusRange);
    tgt = tgt < 0 ? 0 : V - 1;
  }
  float zm = -INFINITY;
  for (int v = threadIdx.x; v < V; v += blockDim.x) zm = fmaxf(zm, to_f(zr[v]));
  zm = block_max(zm, red);
  float tm, s2m, tt, s2t;
  softcap_parts<T>(zm, tm, s2m);
  softcap_parts<T>(to_f(zr[tgt]), tt, s2t);
  const float m = kSoftcap * tm, s_t = kSoftcap * tt;
  float rest = 0.f;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    float t, s2;
    softcap_parts<T>(to_f(zr[v]), t, s2);
    if (v != tgt) rest += exp_t<T>(kSoftcap * t - m);
  }
  rest = block_sum(rest, red);  // syncs: every read of zr precedes the writes
  const float sum = rest + exp_t<T>(s_t - m);
  const float lse = m + logf(sum);
  if (threadIdx.x == 0) token_loss[row] = lse - s_t;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    float t, s2;
    softcap_parts<T>(to_f(zr[v]), t, s2);
    const float p = v == tgt ? -(rest / sum) : exp_t<T>(kSoftcap * t - lse);
    zr[v] = from_f<T>(p * s2 * grad_scale);
  }
}

// Dynamic shared memory of the persistent kernel: one row.
inline int ce_persistent_smem(int V) { return V * 2; }

// Whether the persistent bf16 kernel takes these rows: V a multiple of 8 up
// to 65,536, 16-byte aligned rows.
inline bool ce_persistent_ok(const void *z, int64_t ldz, int V) {
  return V >= 8 && V <= 65536 && (V % 8) == 0 && (ldz % 8) == 0 && ((uintptr_t)z & 15) == 0;
}

inline cudaError_t ce_init() {
  return cudaFuncSetAttribute(ce_fused_bf16_persistent_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              ce_persistent_smem(65536));
}

// Softcap + CE over M rows of z (dtype T), in place; token losses to
// token_loss.  The bf16 rows the persistent kernel takes go there.
template <typename T>
inline cudaError_t launch_ce(T *z, int64_t ldz, const int32_t *targets, float *token_loss, int M, int V,
                             float grad_scale, int num_sms, int *status, cudaStream_t st) {
  if (sizeof(T) == 2 && ce_persistent_ok(z, ldz, V)) {
    const int grid = M < num_sms ? M : num_sms;
    ce_fused_bf16_persistent_kernel<8><<<grid, kCeThreads, ce_persistent_smem(V), st>>>(
        (bf16 *)z, ldz, targets, token_loss, M, V, grad_scale, status);
  } else {
    ce_fused_generic_kernel<T><<<M, 256, 0, st>>>(z, ldz, targets, token_loss, M, V, grad_scale, status);
  }
  return cudaGetLastError();
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
