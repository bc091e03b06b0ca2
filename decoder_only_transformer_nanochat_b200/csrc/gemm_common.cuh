// GEMM problem description shared by the SIMT and the tcgen05 kernels.
//   D[m, n] = epilogue( sum_k A(m, k) B(n, k) )
// A(m, k) = A[m*lda + k] (K-major) or A[k*lda + m] (MN-major); likewise B(n, k).
// The three products of a linear layer y = x W^T map onto it as:
//   forward      y  = x  W^T : A = x  K-major,   B = W  K-major
//   input grad   dx = dy W   : A = dy K-major,   B = W  MN-major
//   weight grad  dW = dy^T x : A = dy MN-major,  B = x  MN-major
#pragma once

#include "common.cuh"

namespace nc {

enum Epilogue : int {
  EPI_STORE = 0,      // D = acc                      (D in T)
  EPI_STORE_F32 = 1,  // D = acc                      (D in fp32)
  EPI_ADD = 2,        // D = D + acc                  (residual add, D in T)
  EPI_RELU2 = 3,      // D = relu(acc)^2              (MLP activation, D in T)
  EPI_DRELU2 = 4,     // D = acc * 2 sqrt(D)          (relu^2 backward: D holds a = relu(h)^2,
                      //                               so relu(h) = sqrt(a); D in T)
  EPI_SOFTCAP = 5,    // D = 15 tanh(acc / 15)        (softcapped logits, D in T)
  EPI_ACC_F32 = 6     // D = D + acc                  (D in fp32: gradient accumulation)
};

// Epilogues whose output D is fp32.
__host__ __device__ inline bool epi_f32(int epi) { return epi == EPI_STORE_F32 || epi == EPI_ACC_F32; }

struct GemmProblem {
  int M, N, K;
  const void *A;
  int64_t lda;
  int a_mn;  // 0: K-major, 1: MN-major
  const void *B;
  int64_t ldb;
  int b_mn;
  void *D;
  int64_t ldd;
  int epi;
};

__device__ __forceinline__ float softcap_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x * (1.f / kSoftcap)));
  return kSoftcap * y;
}

template <typename T> __device__ __forceinline__ float epi_softcap(float acc);
template <> __device__ __forceinline__ float epi_softcap<bf16>(float acc) { return softcap_fast(acc); }
template <> __device__ __forceinline__ float epi_softcap<float>(float acc) {
  return kSoftcap * tanhf(acc * (1.f / kSoftcap));
}

// Apply the epilogue to one output element in place.
template <typename T>
__device__ __forceinline__ void epi_apply(int epi, float acc, void *D, size_t idx) {
  if (epi == EPI_STORE_F32) {
    reinterpret_cast<float *>(D)[idx] = acc;
    return;
  }
  if (epi == EPI_ACC_F32) {
    reinterpret_cast<float *>(D)[idx] += acc;
    return;
  }
  T *d = reinterpret_cast<T *>(D);
  float v;
  switch (epi) {
    case EPI_ADD: v = to_f(d[idx]) + acc; break;
    case EPI_RELU2: { const float r = fmaxf(acc, 0.f); v = r * r; } break;
    case EPI_DRELU2: v = acc * 2.f * sqrtf(to_f(d[idx])); break;
    case EPI_SOFTCAP: v = epi_softcap<T>(acc); break;
    default: v = acc; break;
  }
  d[idx] = from_f<T>(v);
}

}  // namespace nc
