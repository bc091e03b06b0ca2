// Causal multi-query attention on CUDA cores with fp32 arithmetic: the
// exact-fp32 path of the fp32 model.  One shared key/value head serves all H
// query heads (energyai.berlin page, "Multi-Query Attention (MQA)"); scores
// are q.k / sqrt(128) with keys j <= i.
//
// Layout: qkv rows [M, ld] = [q (H*128) | k (128) | v (128)], M = B*T;
// O [M, H*128]; lse and D [B, H, T] fp32.
//
// Each query (or key) row is owned by 8 threads; thread `sub` owns dims
// sub + 8*c, c < 16, and dot products are finished with 3 shuffles.
// window > 0 limits query i to keys j with i - j < window (sliding window);
// window <= 0 is the plain causal mask.
#pragma once

#include "elementwise.cuh"
#include "attn_tc.cuh"
#include "common.cuh"

namespace nc {

constexpr int kSimtRows = 16;   // rows per block (16 rows * 8 threads = 128 threads)
constexpr int kSimtKeys = 32;   // keys / queries per shared-memory tile

__device__ __forceinline__ float sub8_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  return v;
}

template <typename T>
__global__ void __launch_bounds__(128) attn_fwd_simt_kernel(const T *__restrict__ qkv, int ld,
                                                            T *__restrict__ O,
                                                            float *__restrict__ lse, int T_len,
                                                            int H, int window) {
  __shared__ float Ks[kSimtKeys][kHeadDim + 1];
  __shared__ float Vs[kSimtKeys][kHeadDim + 1];
  const int b = blockIdx.z, h = blockIdx.y;
  const int r = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const int i = blockIdx.x * kSimtRows + r;  // query position
  const int C = H * kHeadDim;
  const size_t row0 = (size_t)b * T_len;
  const float scale = rsqrtf((float)kHeadDim);
  float q[16], acc[16];
  const bool valid = i < T_len;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    q[c] = valid ? to_f(qkv[(row0 + i) * ld + h * kHeadDim + sub + 8 * c]) * scale : 0.f;
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int w = window > 0 ? window : T_len;
  const int last = min(T_len - 1, blockIdx.x * kSimtRows + kSimtRows - 1);
  const int j_first = max(0, (int)blockIdx.x * kSimtRows - w + 1) / kSimtKeys * kSimtKeys;
  for (int j0 = j_first; j0 <= last; j0 += kSimtKeys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kSimtKeys * kHeadDim; e += blockDim.x) {
      const int jj = e / kHeadDim, c = e % kHeadDim;
      const int j = j0 + jj;
      const bool ok = j < T_len;
      Ks[jj][c] = ok ? to_f(qkv[(row0 + j) * ld + C + c]) : 0.f;
      Vs[jj][c] = ok ? to_f(qkv[(row0 + j) * ld + C + kHeadDim + c]) : 0.f;
    }
    __syncthreads();
    float s[kSimtKeys];
    float tmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kSimtKeys; ++jj) {
      float d = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) d = fmaf(q[c], Ks[jj][sub + 8 * c], d);
      d = sub8_sum(d);
      s[jj] = (j0 + jj <= i && i - (j0 + jj) < w) ? d : -INFINITY;
      tmax = fmaxf(tmax, s[jj]);
    }
    if (tmax == -INFINITY) continue;  // every key of this tile is in the future
    const float mnew = fmaxf(m, tmax);
    const float corr = expf(m - mnew);
    l *= corr;
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] *= corr;
#pragma unroll
    for (int jj = 0; jj < kSimtKeys; ++jj) {
      const float pj = expf(s[jj] - mnew);
      l += pj;
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[c] = fmaf(pj, Vs[jj][sub + 8 * c], acc[c]);
    }
    m = mnew;
  }
  if (!valid) return;
  const float inv = 1.f / l;
#pragma unroll
  for (int c = 0; c < 16; ++c)
    O[(row0 + i) * C + h * kHeadDim + sub + 8 * c] = from_f<T>(acc[c] * inv);
  if (sub == 0) lse[((size_t)b * H + h) * T_len + i] = m + logf(l);
}

// dq_i = sum_j ds_ij k_j / sqrt(d),  ds_ij = p_ij (dO_i . v_j - D_i),
// p_ij = exp(q_i.k_j/sqrt(d) - lse_i).  Written into the q part of dqkv.
template <typename T>
__global__ void __launch_bounds__(128) attn_bwd_dq_simt_kernel(
    const T *__restrict__ qkv, int ld, const T *__restrict__ dO, const float *__restrict__ lse,
    const float *__restrict__ Dr, T *__restrict__ dqkv, int T_len, int H, int window) {
  __shared__ float Ks[kSimtKeys][kHeadDim + 1];
  __shared__ float Vs[kSimtKeys][kHeadDim + 1];
  const int b = blockIdx.z, h = blockIdx.y;
  const int w = window > 0 ? window : T_len;
  const int r = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const int i = blockIdx.x * kSimtRows + r;
  const int C = H * kHeadDim;
  const size_t row0 = (size_t)b * T_len;
  const float scale = rsqrtf((float)kHeadDim);
  const bool valid = i < T_len;
  float q[16], g[16], dq[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    q[c] = valid ? to_f(qkv[(row0 + i) * ld + h * kHeadDim + sub + 8 * c]) * scale : 0.f;
    g[c] = valid ? to_f(dO[(row0 + i) * C + h * kHeadDim + sub + 8 * c]) : 0.f;
    dq[c] = 0.f;
  }
  const size_t li = ((size_t)b * H + h) * T_len + (valid ? i : 0);
  const float L = lse[li], Di = Dr[li];
  const int last = min(T_len - 1, blockIdx.x * kSimtRows + kSimtRows - 1);
  const int j_first = max(0, (int)blockIdx.x * kSimtRows - w + 1) / kSimtKeys * kSimtKeys;
  for (int j0 = j_first; j0 <= last; j0 += kSimtKeys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kSimtKeys * kHeadDim; e += blockDim.x) {
      const int jj = e / kHeadDim, c = e % kHeadDim;
      const int j = j0 + jj;
      const bool ok = j < T_len;
      Ks[jj][c] = ok ? to_f(qkv[(row0 + j) * ld + C + c]) : 0.f;
      Vs[jj][c] = ok ? to_f(qkv[(row0 + j) * ld + C + kHeadDim + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < kSimtKeys; ++jj) {
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        s = fmaf(q[c], Ks[jj][sub + 8 * c], s);
        dp = fmaf(g[c], Vs[jj][sub + 8 * c], dp);
      }
      s = sub8_sum(s);
      dp = sub8_sum(dp);
      const float p = (j0 + jj <= i && i - (j0 + jj) < w) ? expf(s - L) : 0.f;
      const float ds = p * (dp - Di) * scale;
#pragma unroll
      for (int c = 0; c < 16; ++c) dq[c] = fmaf(ds, Ks[jj][sub + 8 * c], dq[c]);
    }
  }
  if (!valid) return;
#pragma unroll
  for (int c = 0; c < 16; ++c) dqkv[(row0 + i) * ld + h * kHeadDim + sub + 8 * c] = from_f<T>(dq[c]);
}

// dv_j = sum_h sum_{i>=j} p_ij dO_i ;  dk_j = sum_h sum_{i>=j} ds_ij q_i / sqrt(d)
// (the shared head's gradients sum over every query head).  Written into the
// k and v parts of dqkv.
template <typename T>
__global__ void __launch_bounds__(128) attn_bwd_dkdv_simt_kernel(
    const T *__restrict__ qkv, int ld, const T *__restrict__ dO, const float *__restrict__ lse,
    const float *__restrict__ Dr, T *__restrict__ dqkv, int T_len, int H, int window) {
  __shared__ float Qs[kSimtKeys][kHeadDim + 1];
  __shared__ float Gs[kSimtKeys][kHeadDim + 1];
  __shared__ float Ls[kSimtKeys], Ds[kSimtKeys];
  const int b = blockIdx.z;
  const int r = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const int j = blockIdx.x * kSimtRows + r;  // key position
  const int C = H * kHeadDim;
  const size_t row0 = (size_t)b * T_len;
  const float scale = rsqrtf((float)kHeadDim);
  const bool valid = j < T_len;
  float k[16], v[16], dk[16], dv[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    k[c] = valid ? to_f(qkv[(row0 + j) * ld + C + sub + 8 * c]) : 0.f;
    v[c] = valid ? to_f(qkv[(row0 + j) * ld + C + kHeadDim + sub + 8 * c]) : 0.f;
    dk[c] = 0.f;
    dv[c] = 0.f;
  }
  const int first = blockIdx.x * kSimtRows;  // earliest query that sees a key of this block
  const int w = window > 0 ? window : T_len;
  const int i_end = min(T_len, first + kSimtRows - 1 + w);  // past the last query that sees one
  for (int h = 0; h < H; ++h) {
    for (int i0 = (first / kSimtKeys) * kSimtKeys; i0 < i_end; i0 += kSimtKeys) {
      __syncthreads();
      for (int e = threadIdx.x; e < kSimtKeys * kHeadDim; e += blockDim.x) {
        const int ii = e / kHeadDim, c = e % kHeadDim;
        const int i = i0 + ii;
        const bool ok = i < T_len;
        Qs[ii][c] = ok ? to_f(qkv[(row0 + i) * ld + h * kHeadDim + c]) : 0.f;
        Gs[ii][c] = ok ? to_f(dO[(row0 + i) * C + h * kHeadDim + c]) : 0.f;
      }
      if (threadIdx.x < kSimtKeys) {
        const int i = i0 + threadIdx.x;
        const bool ok = i < T_len;
        Ls[threadIdx.x] = ok ? lse[((size_t)b * H + h) * T_len + i] : 0.f;
        Ds[threadIdx.x] = ok ? Dr[((size_t)b * H + h) * T_len + i] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int ii = 0; ii < kSimtKeys; ++ii) {
        const int i = i0 + ii;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          s = fmaf(Qs[ii][sub + 8 * c], k[c], s);
          dp = fmaf(Gs[ii][sub + 8 * c], v[c], dp);
        }
        s = sub8_sum(s) * scale;
        dp = sub8_sum(dp);
        const bool live = valid && i < T_len && i >= j && i - j < w;
        const float p = live ? expf(s - Ls[ii]) : 0.f;
        const float ds = p * (dp - Ds[ii]) * scale;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          dv[c] = fmaf(p, Gs[ii][sub + 8 * c], dv[c]);
          dk[c] = fmaf(ds, Qs[ii][sub + 8 * c], dk[c]);
        }
      }
    }
  }
  if (!valid) return;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    dqkv[(row0 + j) * ld + C + sub + 8 * c] = from_f<T>(dk[c]);
    dqkv[(row0 + j) * ld + C + kHeadDim + sub + 8 * c] = from_f<T>(dv[c]);
  }
}

// Decode attention over the KV cache ("nanochat - full-stack ChatGPT in ~8k
// lines", section "6. Inference": a KV cache with per-row sequence lengths):
// one new query per row b at position p_b = pos[b], against the cached keys
// j <= p_b of that row (window > 0: p_b - j < window).  qkv holds the new
// token's rows [B, ld] (q heads already roped and normed; its k and v already
// in the cache).  CTA per (head h, row b), 128 threads: scores into shared
// memory, their softmax, then thread d sums p_j v_j[d] over the keys (one
// coalesced 256-byte V row per step).  Bandwidth-bound: the cache of the
// shared head is read once per query head from L2.
template <typename T>
__global__ void __launch_bounds__(128) attn_decode_kernel(const T *__restrict__ qkv, int ld,
                                                          const T *__restrict__ kc, const T *__restrict__ vc,
                                                          int64_t cstride, const int32_t *__restrict__ pos,
                                                          int tmax, int H, int window, T *__restrict__ O) {
  extern __shared__ float dsm[];
  __shared__ float red[32];
  float *q = dsm, *pj = dsm + kHeadDim;
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int p = min(max(pos[b], 0), tmax - 1);
  const int j0 = window > 0 ? max(0, p - window + 1) : 0;
  const T *krow0 = kc + (size_t)b * cstride, *vrow0 = vc + (size_t)b * cstride;
  q[t] = to_f(qkv[(size_t)b * ld + h * kHeadDim + t]) * rsqrtf((float)kHeadDim);
  __syncthreads();
  float m = -INFINITY;
  for (int j = j0 + t; j <= p; j += blockDim.x) {
    const T *kr = krow0 + (size_t)j * kHeadDim;
    float d = 0.f;
#pragma unroll
    for (int c = 0; c < kHeadDim / 8; ++c) {
      float k8[8];
      Vec8<T>::load(kr + 8 * c, k8);
#pragma unroll
      for (int i = 0; i < 8; ++i) d = fmaf(q[8 * c + i], k8[i], d);
    }
    pj[j - j0] = d;
    m = fmaxf(m, d);
  }
  m = block_max(m, red);
  float l = 0.f;
  for (int j = j0 + t; j <= p; j += blockDim.x) {
    const float e = expf(pj[j - j0] - m);
    pj[j - j0] = e;
    l += e;
  }
  l = block_sum(l, red);  // its barriers also publish every p_j
  float acc = 0.f;
  for (int j = j0; j <= p; ++j) acc = fmaf(pj[j - j0], to_f(vrow0[(size_t)j * kHeadDim + t]), acc);
  O[(size_t)b * H * kHeadDim + h * kHeadDim + t] = from_f<T>(acc / l);
}

// Shared memory of the decode kernel: the query and one score per cached key.
inline size_t attn_decode_smem(int tmax) { return (size_t)(kHeadDim + tmax) * sizeof(float); }

template <typename T>
inline cudaError_t launch_attn_decode(const T *qkv, int ld, const T *kc, const T *vc, int64_t cstride,
                                      const int32_t *pos, int tmax, int B, int H, int window, T *O,
                                      cudaStream_t st) {
  attn_decode_kernel<T><<<dim3(H, B), kHeadDim, attn_decode_smem(tmax), st>>>(qkv, ld, kc, vc, cstride, pos, tmax,
                                                                               H, window, O);
  return cudaGetLastError();
}

// pos[b] += 1 after a decode step; pos[b] = T after a prefill of T tokens.
__global__ void seqlens_kernel(int32_t *__restrict__ pos, int B, int set_to) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) pos[b] = set_to >= 0 ? set_to : pos[b] + 1;
}

template <typename T>
inline cudaError_t launch_attn_simt_fwd(const T *qkv, int ld, T *O, float *lse, int B, int T_len,
                                        int H, int window, cudaStream_t st) {
  dim3 grid((T_len + kSimtRows - 1) / kSimtRows, H, B);
  attn_fwd_simt_kernel<T><<<grid, 128, 0, st>>>(qkv, ld, O, lse, T_len, H, window);
  return cudaGetLastError();
}

template <typename T>
inline cudaError_t launch_attn_simt_bwd(const T *qkv, int ld, const T *dO, const float *lse,
                                        const float *Dr, T *dqkv, int B, int T_len, int H, int window,
                                        cudaStream_t st) {
  dim3 g1((T_len + kSimtRows - 1) / kSimtRows, H, B);
  attn_bwd_dq_simt_kernel<T><<<g1, 128, 0, st>>>(qkv, ld, dO, lse, Dr, dqkv, T_len, H, window);
  dim3 g2((T_len + kSimtRows - 1) / kSimtRows, 1, B);
  attn_bwd_dkdv_simt_kernel<T><<<g2, 128, 0, st>>>(qkv, ld, dO, lse, Dr, dqkv, T_len, H, window);
  return cudaGetLastError();
}

}  // namespace nc

namespace nc {

// engine 0: the path of the model step -- tcgen05 tensor cores for bf16 (the
// caller checks fatc::supported / supported_bwd first and reports a
// misaligned operand; there is no slower fallback), CUDA cores for fp32;
// engine 1: the CUDA-core kernels for either dtype (a test engine).
template <typename T>
inline cudaError_t launch_attn_fwd(const T *qkv, int ld, T *O, float *lse, int B, int T_len, int H, int window,
                                   int engine, int *status, cudaStream_t st, int num_sms = 148) {
  if (sizeof(T) == 2 && (engine == 0 || engine == 2 || engine == 3)) {
    if (!fatc::supported(qkv, ld, O)) return cudaErrorInvalidValue;
    const bool pp = engine == 3 || (engine == 0) == fatc::kFwdPingPongDefault;
    return fatc::launch_fwd((const bf16 *)qkv, ld, (bf16 *)O, lse, B, T_len, H, window, pp,
                            engine == 3 ? 0 : num_sms, status, st);
  }
  return launch_attn_simt_fwd<T>(qkv, ld, O, lse, B, T_len, H, window, st);
}

// D = rowsum(dO * O) is computed inside the tcgen05 dQ kernel; the CUDA-core
// engine gets it from attn_rowdot_kernel first.  Drow is [B, H, T] scratch.
// part: scratch that lets the tcgen05 dK/dV kernel cut large key tiles into
// pieces (fatc::dkdv_scratch_bytes; nullptr: no cut).
template <typename T>
inline cudaError_t launch_attn_bwd(const T *qkv, int ld, const T *O, const T *dO, const float *lse, float *Dr,
                                   T *dqkv, int B, int T_len, int H, int window, int engine, int *status,
                                   cudaStream_t st, float *part = nullptr, size_t part_bytes = 0,
                                   int num_sms = 148, int *launched = nullptr) {
  if (sizeof(T) == 2 && engine == 0) {
    if (!fatc::supported_bwd(qkv, ld, O, dO, dqkv)) return cudaErrorInvalidValue;
    return fatc::launch_bwd((const bf16 *)qkv, ld, (const bf16 *)O, (const bf16 *)dO, lse, Dr, part, part_bytes,
                            (bf16 *)dqkv, B, T_len, H, window, num_sms, status, st, launched);
  }
  if (launched) *launched = 3;
  const int M = B * T_len;
  attn_rowdot_kernel<T><<<(unsigned)(((size_t)M * H + 7) / 8), 256, 0, st>>>(dO, O, Dr, M, T_len, H);
  return launch_attn_simt_bwd<T>(qkv, ld, dO, lse, Dr, dqkv, B, T_len, H, window, st);
}

}  // namespace nc
