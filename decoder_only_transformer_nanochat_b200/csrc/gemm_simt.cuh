// CUDA-core GEMM with fp32 accumulation: the exact-fp32 path of the fp32
// model (tensor-core TF32 would miss its 1e-5 tolerance), usable for bf16
// operands as well.  128x128 output tile, 256 threads, 8x8 outputs per
// thread, k-slices of 16 staged through shared memory in [k][m] order for
// either operand layout.
#pragma once

#include "gemm_common.cuh"

namespace nc {

constexpr int kSimtBM = 128, kSimtBN = 128, kSimtBK = 16;

template <typename T>
__device__ __forceinline__ void simt_stage(const T *__restrict__ X, int64_t ld, int mn_major,
                                           int rows, int K, int r0, int k0,
                                           float (*S)[kSimtBM + 4]) {
  // stage X(r0 + r, k0 + k) for r < 128, k < 16 into S[k][r]
  const int tid = threadIdx.x;
  if (!mn_major) {
    // contiguous along k: thread reads 8 consecutive k of one row
    const int r = tid >> 1, kk = (tid & 1) * 8;
    const int gr = r0 + r;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gk = k0 + kk + j;
      S[kk + j][r] = (gr < rows && gk < K) ? to_f(X[(int64_t)gr * ld + gk]) : 0.f;
    }
  } else {
    // contiguous along rows: thread reads 8 consecutive rows of one k
    const int kk = tid >> 4, r = (tid & 15) * 8;
    const int gk = k0 + kk;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gr = r0 + r + j;
      S[kk][r + j] = (gr < rows && gk < K) ? to_f(X[(int64_t)gk * ld + gr]) : 0.f;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmProblem p) {
  __shared__ float As[kSimtBK][kSimtBM + 4];
  __shared__ float Bs[kSimtBK][kSimtBN + 4];
  const int m0 = blockIdx.y * kSimtBM, n0 = blockIdx.x * kSimtBN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const T *A = reinterpret_cast<const T *>(p.A);
  const T *B = reinterpret_cast<const T *>(p.B);
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < p.K; k0 += kSimtBK) {
    simt_stage<T>(A, p.lda, p.a_mn, p.M, p.K, m0, k0, As);
    simt_stage<T>(B, p.ldb, p.b_mn, p.N, p.K, n0, k0, Bs);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSimtBK; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n < p.N) epi_apply<T>(p.epi, acc[i][j], p.D, (size_t)m * p.ldd + n);
    }
  }
}

template <typename T>
inline cudaError_t launch_gemm_simt(const GemmProblem &p, cudaStream_t st) {
  dim3 grid((p.N + kSimtBN - 1) / kSimtBN, (p.M + kSimtBM - 1) / kSimtBM);
  gemm_simt_kernel<T><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace nc
