// Bandwidth-bound kernels of the decoder step: embedding gather + RMSNorm,
// RMSNorm, RoPE + QK-norm, their backward passes and the embedding
// scatter-add.  One warp owns one row; a row of C values is held in registers
// (8 contiguous values per 16-byte access, C/8 accesses spread over the lanes)
// so each row is read once and written once.
//
// Parameterless RMSNorm y = x / sqrt(mean(x^2) + eps) ("A Llama-class
// transformer with ten modern departures": bare F.rms_norm after the
// embedding, before attention, before the MLP and before the head).
// Backward: dx = r (dy - y mean(dy y)), r = 1/sqrt(mean(x^2) + eps).
#pragma once

#include "common.cuh"

namespace nc {

// NV = 16-byte accesses per lane: a row of C values needs NV = ceil(C / 256).
// Rows up to C = 32 lanes * 16 * 8 = 4096 are supported.
constexpr int kMaxVecPerLane = 16;

#define NC_DISPATCH_NV(C, KERNEL_CALL)                 \
  do {                                                 \
    const int nv_ = ((C) / 8 + 31) / 32;               \
    switch (nv_) {                                     \
      case 1: { constexpr int NV = 1; KERNEL_CALL; } break; \
      case 2: { constexpr int NV = 2; KERNEL_CALL; } break; \
      case 3: { constexpr int NV = 3; KERNEL_CALL; } break; \
      case 4: { constexpr int NV = 4; KERNEL_CALL; } break; \
      case 5: { constexpr int NV = 5; KERNEL_CALL; } break; \
      case 6: { constexpr int NV = 6; KERNEL_CALL; } break; \
      case 7: { constexpr int NV = 7; KERNEL_CALL; } break; \
      case 8: { constexpr int NV = 8; KERNEL_CALL; } break; \
      default: { constexpr int NV = 16; KERNEL_CALL; } break; \
    }                                                  \
  } while (0)

// ---------------------------------------------------------------------------
// x = rmsnorm(wte[tok]); r0 = 1/rms.  Token ids outside [0, V) are flagged
// and clamped so the gather stays in bounds.
template <typename T, int NV>
__global__ void __launch_bounds__(256) embed_norm_kernel(
    const int32_t *__restrict__ tokens, const T *__restrict__ wte, T *__restrict__ x,
    float *__restrict__ r_out, int M, int C, int V, int *status) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  int tok = tokens[row];
  if (tok < 0 || tok >= V) {
    if (lane == 0) set_status(status, kStatusRange);
    tok = tok < 0 ? 0 : V - 1;
  }
  const int nv = C >> 3;
  const T *src = wte + (size_t)tok * C;
  float v[NV][8];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (lane + 32 * i);
    if (c < nv) {
      Vec8<T>::load(src + c * 8, v[i]);
#pragma unroll
      for (int j = 0; j < 8; ++j) ss += v[i][j] * v[i][j];
    }
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)C + kEps);
  T *dst = x + (size_t)row * C;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (lane + 32 * i);
    if (c < nv) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[i][j] *= r;
      Vec8<T>::store(dst + c * 8, v[i]);
    }
  }
  if (lane == 0) r_out[row] = r;
}

// y = rmsnorm(x) row-wise; r = 1/rms saved for the backward pass.
template <typename T, int NV>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const T *__restrict__ x, T *__restrict__ y,
                                                      float *__restrict__ r_out, int M, int C) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const int nv = C >> 3;
  const T *src = x + (size_t)row * C;
  float v[NV][8];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (lane + 32 * i);
    if (c < nv) {
      Vec8<T>::load(src + c * 8, v[i]);
#pragma unroll
      for (int j = 0; j < 8; ++j) ss += v[i][j] * v[i][j];
    }
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)C + kEps);
  T *dst = y + (size_t)row * C;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (lane + 32 * i);
    if (c < nv) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[i][j] *= r;
      Vec8<T>::store(dst + c * 8, v[i]);
    }
  }
  if (lane == 0) r_out[row] = r;
}

// RMSNorm backward with the residual-stream accumulation:
//   g = r (dy - y mean(dy y));  dx = g (+ dx_old if accumulate)
// dy is a GEMM output in T, y the saved normalised value, dx kept in fp32
// and also written in T as the next GEMM's operand.
template <typename T, int NV>
__global__ void __launch_bounds__(256) rmsnorm_bwd_kernel(
    const T *__restrict__ dy, const T *__restrict__ y, const float *__restrict__ r,
    float *__restrict__ dx, T *__restrict__ dx_t, int M, int C, int accumulate) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const int nv = C >> 3;
  const size_t base = (size_t)row * C;
  // Pass 1: dot(dy, y) over the row, with the fp32 dx_old it will add to
  // requested into L2 meanwhile.  Nothing is kept across the reduction, so
  // the kernel runs at a register count that keeps many rows in flight.
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (lane + 32 * i);
    if (c < nv) {
      float g[8], yy[8];
      Vec8<T>::load(dy + base + c * 8, g);
      Vec8<T>::load(y + base + c * 8, yy);
#pragma unroll
      for (int j = 0; j < 8; ++j) dot += g[j] * yy[j];
      if (accumulate) asm volatile("prefetch.global.L2 [%0];" ::"l"(dx + base + c * 8));
    }
  }
  dot = warp_sum(dot) / (float)C;
  const float rr = r[row];
  // Pass 2: dy and y again (now in L1 or L2), then dx and its copy in T.
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (lane + 32 * i);
    if (c < nv) {
      float g[8], yy[8], old[8];
      Vec8<T>::load(dy + base + c * 8, g);
      Vec8<T>::load(y + base + c * 8, yy);
      if (accumulate) Vec8<float>::load(dx + base + c * 8, old);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        g[j] = rr * (g[j] - yy[j] * dot);
        if (accumulate) g[j] += old[j];
      }
      Vec8<float>::store(dx + base + c * 8, g);
      Vec8<T>::store(dx_t + base + c * 8, g);
    }
  }
}

// ---------------------------------------------------------------------------
// RoPE then QK-norm, in place on the q heads and the shared k head of the
// fused qkv rows [M, ld] = [q (H*128) | k (128) | v (128)].
// RoPE ("ten modern departures": theta 10,000) on half-split pairs (i, i+64):
//   y_i = x_i cos - x_{i+64} sin,  y_{i+64} = x_i sin + x_{i+64} cos,
// angle = pos * theta^(-i/64), pos = token index within its row of T.
// QK-norm after RoPE: per-head parameterless RMSNorm over the 128 dims.
template <typename T> struct Pair2;
template <> struct Pair2<bf16> {
  static __device__ __forceinline__ float2 load(const bf16 *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
  }
  static __device__ __forceinline__ void store(bf16 *p, float2 v) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v.x, v.y);
  }
};
template <> struct Pair2<float> {
  static __device__ __forceinline__ float2 load(const float *p) {
    return *reinterpret_cast<const float2 *>(p);
  }
  static __device__ __forceinline__ void store(float *p, float2 v) {
    *reinterpret_cast<float2 *>(p) = v;
  }
};

// One warp per token: the q heads and the k head of a token are H+1
// contiguous 128-wide rows; each half-warp holds one head, so a warp covers
// two heads per step.  Lane j of the half-warp holds both members of its four
// RoPE pairs, dims 4j..4j+3 and 64+4j..64+4j+3 (two 8-byte loads for bf16), so
// the rotation needs no data from other lanes; the head's sum of squares is a
// 16-lane reduction.
template <typename T>
__device__ __forceinline__ void rope_pair_tables(const float *cos_t, const float *sin_t, int pos, int j,
                                                 float (&c)[4], float (&s)[4]) {
  const float4 c4 = *reinterpret_cast<const float4 *>(cos_t + pos * 64 + 4 * j);
  const float4 s4 = *reinterpret_cast<const float4 *>(sin_t + pos * 64 + 4 * j);
  c[0] = c4.x; c[1] = c4.y; c[2] = c4.z; c[3] = c4.w;
  s[0] = s4.x; s[1] = s4.y; s[2] = s4.z; s[3] = s4.w;
}

__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Value embedding (full reference block): with ve != nullptr the shared v
// head of the row also gets gate * ve[token] added ("ten modern departures":
// a gated embedding lookup added to V at alternating layers); v is neither
// roped nor normed.
// KV cache (inference): with kc != nullptr the finished k and v of the row
// are also written to the cache at [row b, position pos] (stride `cstride`
// elements between rows b), b = tok / T_len; pos = positions[b] when given
// (decode: one token per row), else tok % T_len (prefill).
template <typename T>
struct KvCacheOut {
  T *kc = nullptr, *vc = nullptr;
  int64_t cstride = 0;
  const int32_t *positions = nullptr;
  int tmax = 0;        // positions past the cache are clamped and flagged
  int *status = nullptr;
};

template <typename T>
__global__ void __launch_bounds__(256) rope_qknorm_kernel(
    T *__restrict__ qkv, int ld, float *__restrict__ rq, float *__restrict__ rk,
    const float *__restrict__ cos_t, const float *__restrict__ sin_t, int M, int T_len, int H,
    const int32_t *__restrict__ tokens = nullptr, const T *__restrict__ ve = nullptr,
    const T *__restrict__ ve_gate = nullptr, int V = 0, KvCacheOut<T> cache = KvCacheOut<T>()) {
  const int tok = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= M) return;
  int pos = cache.positions ? cache.positions[tok / T_len] : tok % T_len;
  if (cache.positions && (pos < 0 || pos >= cache.tmax)) {
    if (lane == 0) set_status(cache.status, kStatusRange);
    pos = pos < 0 ? 0 : cache.tmax - 1;
  }
  T *kc_row = cache.kc ? cache.kc + (size_t)(tok / T_len) * cache.cstride + (size_t)pos * kHeadDim : nullptr;
  if ((ve || cache.kc) && lane < kHeadDim / 8) {
    T *vrow = qkv + (size_t)tok * ld + (H + 1) * kHeadDim + lane * 8;
    float v[8];
    Vec8<T>::load(vrow, v);
    if (ve) {
      const int id = min(max(tokens[tok], 0), V - 1);
      const float g = to_f(ve_gate[0]);
      float e[8];
      Vec8<T>::load(ve + (size_t)id * kHeadDim + lane * 8, e);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] += g * e[i];
      Vec8<T>::store(vrow, v);
    }
    if (cache.kc) Vec8<T>::store(cache.vc + (kc_row - cache.kc) + lane * 8, v);
  }
  const int hw = lane >> 4, j = lane & 15;
  float c[4], s[4];
  rope_pair_tables<T>(cos_t, sin_t, pos, j, c, s);
  T *row = qkv + (size_t)tok * ld;
  for (int h0 = 0; h0 < H + 1; h0 += 2) {
    const int h = h0 + hw;
    const bool live = h < H + 1;  // uniform per half-warp
    float a[4], b[4];             // dims 4j.. and 64 + 4j..
    if (live) {
      Vec4<T>::load(row + h * kHeadDim + 4 * j, a);
      Vec4<T>::load(row + h * kHeadDim + 64 + 4 * j, b);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = 0.f; b[i] = 0.f; }
    }
    float ya[4], yb[4], ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // y_i = x_i cos - x_{i+64} sin ;  y_{i+64} = x_i sin + x_{i+64} cos
      ya[i] = a[i] * c[i] - b[i] * s[i];
      yb[i] = a[i] * s[i] + b[i] * c[i];
      ss += ya[i] * ya[i] + yb[i] * yb[i];
    }
    ss = half_warp_sum(ss);
    const float r = rsqrtf(ss / (float)kHeadDim + kEps);
#pragma unroll
    for (int i = 0; i < 4; ++i) { ya[i] *= r; yb[i] *= r; }
    if (live) {
      Vec4<T>::store(row + h * kHeadDim + 4 * j, ya);
      Vec4<T>::store(row + h * kHeadDim + 64 + 4 * j, yb);
      if (h == H && kc_row) {
        Vec4<T>::store(kc_row + 4 * j, ya);
        Vec4<T>::store(kc_row + 64 + 4 * j, yb);
      }
      if (j == 0) {
        if (h < H) rq[(size_t)tok * H + h] = r;
        else rk[tok] = r;
      }
    }
  }
}

// Backward of QK-norm then RoPE, in place on the q and k parts of dqkv:
//   g = r (dy - y mean(dy y)) with y the saved normalised q/k,
//   dx_i = g_i cos + g_{i+64} sin,  dx_{i+64} = -g_i sin + g_{i+64} cos.
template <typename T>
__global__ void __launch_bounds__(256) rope_qknorm_bwd_kernel(
    T *__restrict__ dqkv, const T *__restrict__ qkv, int ld, const float *__restrict__ rq,
    const float *__restrict__ rk, const float *__restrict__ cos_t,
    const float *__restrict__ sin_t, int M, int T_len, int H) {
  const int tok = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= M) return;
  const int pos = tok % T_len;
  const int hw = lane >> 4, j = lane & 15;
  float c[4], s[4];
  rope_pair_tables<T>(cos_t, sin_t, pos, j, c, s);
  T *drow = dqkv + (size_t)tok * ld;
  const T *yrow = qkv + (size_t)tok * ld;
  for (int h0 = 0; h0 < H + 1; h0 += 2) {
    const int h = h0 + hw;
    const bool live = h < H + 1;
    float da[4], db[4], ya[4], yb[4];  // dims 4j.. and 64 + 4j..
    if (live) {
      Vec4<T>::load(drow + h * kHeadDim + 4 * j, da);
      Vec4<T>::load(drow + h * kHeadDim + 64 + 4 * j, db);
      Vec4<T>::load(yrow + h * kHeadDim + 4 * j, ya);
      Vec4<T>::load(yrow + h * kHeadDim + 64 + 4 * j, yb);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) { da[i] = 0.f; db[i] = 0.f; ya[i] = 0.f; yb[i] = 0.f; }
    }
    const float r = live ? (h < H ? rq[(size_t)tok * H + h] : rk[tok]) : 0.f;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) dot += da[i] * ya[i] + db[i] * yb[i];
    dot = half_warp_sum(dot) / (float)kHeadDim;
    float oa[4], ob[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float ga = r * (da[i] - ya[i] * dot), gb = r * (db[i] - yb[i] * dot);
      // dx_i = g_i cos + g_{i+64} sin ;  dx_{i+64} = -g_i sin + g_{i+64} cos
      oa[i] = ga * c[i] + gb * s[i];
      ob[i] = gb * c[i] - ga * s[i];
    }
    if (live) {
      Vec4<T>::store(drow + h * kHeadDim + 4 * j, oa);
      Vec4<T>::store(drow + h * kHeadDim + 64 + 4 * j, ob);
    }
  }
}

// ---------------------------------------------------------------------------
// Residual scalars of the full reference block ("ten modern departures":
// resid_lambdas and x0_lambdas mixing each layer's stream with the
// normalised embedding).  At block entry
//   x_in = lam_r x + lam_0 x0,   xn = rmsnorm(x_in)
// x_in is the stream the block's residual adds then go into (written to
// x_out, a buffer of its own, so x stays for the backward).
template <typename T, int NV>
__global__ void __launch_bounds__(256) mix_rmsnorm_kernel(
    const T *__restrict__ x, const T *__restrict__ x0, const T *__restrict__ lam_r, const T *__restrict__ lam_0,
    T *__restrict__ x_out, T *__restrict__ y, float *__restrict__ r_out, int M, int C) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float a = to_f(lam_r[0]), b = to_f(lam_0[0]);
  const int nv = C >> 3;
  const size_t base = (size_t)row * C;
  float v[NV][8];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (lane + 32 * i);
    if (c < nv) {
      float e[8];
      Vec8<T>::load(x + base + c * 8, v[i]);
      Vec8<T>::load(x0 + base + c * 8, e);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[i][j] = a * v[i][j] + b * e[j];
        ss += v[i][j] * v[i][j];
      }
      Vec8<T>::store(x_out + base + c * 8, v[i]);
    }
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)C + kEps);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (lane + 32 * i);
    if (c < nv) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[i][j] *= r;
      Vec8<T>::store(y + base + c * 8, v[i]);
    }
  }
  if (lane == 0) r_out[row] = r;
}

// Backward of the block entry, fused into the norm backward of xn:
//   dx_in = dx_old + r (dy - y mean(dy y))
//   dx    = lam_r dx_in          (the stream gradient below the block; fp32 and T)
//   dx0  (+)= lam_0 dx_in        (first != 0: written, else accumulated)
//   partial[block] = (sum dx_in x, sum dx_in x0) over the block's rows, in a
//   fixed order (the scalars' gradients, finished by ordered_sum_rows_kernel)
template <typename T, int NV>
__global__ void __launch_bounds__(256) rmsnorm_bwd_mix_kernel(
    const T *__restrict__ dy, const T *__restrict__ y, const float *__restrict__ r, float *__restrict__ dx,
    T *__restrict__ dx_t, const T *__restrict__ x, const T *__restrict__ x0, const T *__restrict__ lam_r,
    const T *__restrict__ lam_0, float *__restrict__ dx0, int first, float *__restrict__ part_r,
    float *__restrict__ part_0, int M, int C) {
  __shared__ float sh_r[8], sh_0[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  float sum_r = 0.f, sum_0 = 0.f;
  if (row < M) {
    const float a = to_f(lam_r[0]), b = to_f(lam_0[0]);
    const int nv = C >> 3;
    const size_t base = (size_t)row * C;
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = (lane + 32 * i);
      if (c < nv) {
        float g[8], yy[8];
        Vec8<T>::load(dy + base + c * 8, g);
        Vec8<T>::load(y + base + c * 8, yy);
#pragma unroll
        for (int j = 0; j < 8; ++j) dot += g[j] * yy[j];
        asm volatile("prefetch.global.L2 [%0];" ::"l"(dx + base + c * 8));
      }
    }
    dot = warp_sum(dot) / (float)C;
    const float rr = r[row];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = (lane + 32 * i);
      if (c < nv) {
        float g[8], yy[8], old[8], xv[8], x0v[8], acc0[8];
        Vec8<T>::load(dy + base + c * 8, g);
        Vec8<T>::load(y + base + c * 8, yy);
        Vec8<float>::load(dx + base + c * 8, old);
        Vec8<T>::load(x + base + c * 8, xv);
        Vec8<T>::load(x0 + base + c * 8, x0v);
        if (!first) Vec8<float>::load(dx0 + base + c * 8, acc0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float din = old[j] + rr * (g[j] - yy[j] * dot);
          sum_r += din * xv[j];
          sum_0 += din * x0v[j];
          g[j] = a * din;
          acc0[j] = (first ? 0.f : acc0[j]) + b * din;
        }
        Vec8<float>::store(dx + base + c * 8, g);
        Vec8<T>::store(dx_t + base + c * 8, g);
        Vec8<float>::store(dx0 + base + c * 8, acc0);
      }
    }
    sum_r = warp_sum(sum_r);
    sum_0 = warp_sum(sum_0);
  }
  if (lane == 0) {
    sh_r[warp] = sum_r;
    sh_0[warp] = sum_0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f, b = 0.f;
    for (int w = 0; w < 8; ++w) {
      a += sh_r[w];
      b += sh_0[w];
    }
    part_r[blockIdx.x] = a;
    part_0[blockIdx.x] = b;
  }
}

// out[row * out_stride] (+)= sum of partial[row * n .. row * n + n) in a fixed order.
__global__ void __launch_bounds__(256) ordered_sum_rows_kernel(const float *__restrict__ partial, int n,
                                                               float *__restrict__ out, int out_stride,
                                                               int accumulate) {
  __shared__ float sh[32];
  const float *p = partial + (size_t)blockIdx.x * n;
  float s = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += p[i];
  s = block_sum(s, sh);
  float *o = out + (size_t)blockIdx.x * out_stride;
  if (threadIdx.x == 0) *o = s + (accumulate ? *o : 0.f);
}

// Value-embedding gate gradient, first stage: partial[block] = sum over the
// block's 64 positions of dv_i . ve[tok_i] (dv: v part of dqkv, stride ld), in
// a fixed order; ordered_sum_kernel adds the partials.
template <typename T>
__global__ void __launch_bounds__(256) ve_gate_partial_kernel(const T *__restrict__ dv, int64_t ld,
                                                              const int32_t *__restrict__ tokens,
                                                              const T *__restrict__ ve, int V, int M,
                                                              float *__restrict__ partial) {
  __shared__ float sh[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc = 0.f;
  for (int t = 0; t < 8; ++t) {
    const int i = blockIdx.x * 64 + warp * 8 + t;
    if (i < M && lane < kHeadDim / 8) {
      const int id = min(max(tokens[i], 0), V - 1);
      float a[8], e[8];
      Vec8<T>::load(dv + (size_t)i * ld + lane * 8, a);
      Vec8<T>::load(ve + (size_t)id * kHeadDim + lane * 8, e);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc += a[j] * e[j];
    }
  }
  acc = warp_sum(acc);
  if (lane == 0) sh[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += sh[w];
    partial[blockIdx.x] = s;
  }
}

// D[b,h,t] = sum_c dO[t,h,c] O[t,h,c]  (the softmax-backward row term).
template <typename T>
__global__ void __launch_bounds__(256) attn_rowdot_kernel(const T *__restrict__ dO,
                                                          const T *__restrict__ O,
                                                          float *__restrict__ D, int M,
                                                          int T_len, int H) {
  const int item = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (item >= M * H) return;
  const int tok = item / H, h = item % H;
  const size_t off = (size_t)tok * H * kHeadDim + h * kHeadDim + lane * 4;
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 4; j += 2) {
    float2 a = Pair2<T>::load(dO + off + j), b = Pair2<T>::load(O + off + j);
    s += a.x * b.x + a.y * b.y;
  }
  s = warp_sum(s);
  if (lane == 0) {
    const int bb = tok / T_len, t = tok % T_len;
    D[((size_t)bb * H + h) * T_len + t] = s;
  }
}

}  // namespace nc
