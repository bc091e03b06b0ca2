// The optimizer step: Muon for the block matrices, AdamW for the embeddings,
// the unembedding and the scalars ("Nanochat: full-stack LLM training in 8,000
// lines for $72", section "A Llama-class transformer with ten modern
// departures": a dual optimizer, Muon for the matrices, AdamW for embeddings
// and scalars; "nanochat - full-stack ChatGPT in ~8k lines", section "2.
// Pretrain").  State, all fp32, laid out like the weights: the master copy,
// m (AdamW's first moment, or Muon's momentum) and v (AdamW's second moment).
//
// AdamW, element-wise with bias correction and decoupled decay:
//   m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2
//   w = w - lr (m bc1) / (sqrt(v bc2) + eps) - lr wd w,   bc = 1 / (1 - b^t)
// Muon, per matrix M [n, k]: buf = mu buf + g; X = buf / |buf|_F; then the
// cubic Newton-Schulz step X = 1.5 X - 0.5 X X^T X (written through the small
// Gram matrix of the shorter side), and w = w - lr X - lr wd w.  The
// Newton-Schulz products run on the library's GEMMs (tensor cores for bf16
// models); the rest is element-wise here.
#pragma once

#include "common.cuh"

namespace nc {

constexpr int kOptBlocks = 296;  // fixed grid of the norm's partial sums: a fixed summation order

template <typename T>
__global__ void __launch_bounds__(256) adamw_kernel(T *__restrict__ w, float *__restrict__ master,
                                                    const float *__restrict__ g, float *__restrict__ m,
                                                    float *__restrict__ v, int64_t n, float lr, float b1, float b2,
                                                    float eps, float wd, float bc1, float bc2) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float gi = g[i];
    const float mi = b1 * m[i] + (1.f - b1) * gi;
    const float vi = b2 * v[i] + (1.f - b2) * gi * gi;
    m[i] = mi;
    v[i] = vi;
    const float wi = master[i];
    const float nw = wi - lr * (mi * bc1) / (sqrtf(vi * bc2) + eps) - lr * wd * wi;
    master[i] = nw;
    w[i] = from_f<T>(nw);
  }
}

// buf = mu buf + g over one matrix; partial[block] = sum of buf^2 over a fixed
// set of elements (grid kOptBlocks), added in a fixed order afterwards.
__global__ void __launch_bounds__(256) muon_momentum_kernel(const float *__restrict__ g, float *__restrict__ buf,
                                                            int64_t n, float mu, float *__restrict__ partial) {
  __shared__ float sh[32];
  float s = 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float b = mu * buf[i] + g[i];
    buf[i] = b;
    s += b * b;
  }
  s = block_sum(s, sh);
  if (threadIdx.x == 0) partial[blockIdx.x] = s;
}

// X = buf / sqrt(sumsq) in T (X = 0 for a zero momentum).
template <typename T>
__global__ void __launch_bounds__(256) muon_scale_kernel(const float *__restrict__ buf, int64_t n,
                                                         const float *__restrict__ sumsq, T *__restrict__ X) {
  const float s = *sumsq;
  const float inv = s > 0.f ? rsqrtf(s) : 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    X[i] = from_f<T>(buf[i] * inv);
}

// Bm = 1.5 I - 0.5 A for the k x k Gram matrix A (fp32), in T.
template <typename T>
__global__ void __launch_bounds__(256) ns_coeff_kernel(const float *__restrict__ A, int k, T *__restrict__ Bm) {
  const int64_t n = (int64_t)k * k;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / k), c = (int)(i % k);
    Bm[i] = from_f<T>((r == c ? 1.5f : 0.f) - 0.5f * A[i]);
  }
}

// w = w - lr X - lr wd w on the master copy, and its copy in T.
template <typename T>
__global__ void __launch_bounds__(256) muon_apply_kernel(float *__restrict__ master, const T *__restrict__ X,
                                                         T *__restrict__ w, int64_t n, float lr, float wd) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float wi = master[i];
    const float nw = wi - lr * to_f(X[i]) - lr * wd * wi;
    master[i] = nw;
    w[i] = from_f<T>(nw);
  }
}

// master = the weights, widened; m = v = 0.
template <typename T>
__global__ void __launch_bounds__(256) optim_init_kernel(const T *__restrict__ w, float *__restrict__ master,
                                                         float *__restrict__ m, float *__restrict__ v, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    master[i] = to_f(w[i]);
    m[i] = 0.f;
    v[i] = 0.f;
  }
}

inline unsigned ew_grid(int64_t n, int num_sms) {
  const int64_t want = (n + 255) / 256;
  const int64_t cap = (int64_t)num_sms * 8;
  return (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace nc
