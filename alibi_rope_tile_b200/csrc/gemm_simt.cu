// CUDA-core GEMM for the block projections when the tensor-core GEMM does not apply
// (fp32, or shapes that are not multiples of its tile): C = A @ W with A [M,K],
// W [K,N], C [M,N], all row-major, fp32 accumulation ("Write attention from scratch",
// worked example: x @ Wq, ..., ctx @ Wo with weights stored [in, out]).
// 64x64 output tile per 256-thread CTA, 4x4 outputs per thread, K staged by 16.
#include "kernels.h"

namespace attn {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ A,
                                                        const T* __restrict__ W, T* __restrict__ C,
                                                        int M, int N, int K) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Ws[TK][TN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int idx = tid; idx < TM * TK; idx += 256) {
      const int r = idx / TK, c = idx % TK;
      const int gm = m0 + r, gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? Elem<T>::load(A + (size_t)gm * K + gk) : 0.f;
    }
    for (int idx = tid; idx < TK * TN; idx += 256) {
      const int r = idx / TN, c = idx % TN;
      const int gk = k0 + r, gn = n0 + c;
      Ws[r][c] = (gk < K && gn < N) ? Elem<T>::load(W + (size_t)gk * N + gn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gm = m0 + ty + 16 * i, gn = n0 + tx + 16 * j;
      if (gm < M && gn < N) Elem<T>::store(C + (size_t)gm * N + gn, acc[i][j]);
    }
}

}  // namespace

cudaError_t launch_gemm_simt(const void* A, const void* W, void* C, int M, int N, int K, int dtype,
                             cudaStream_t s) {
  dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
  if (dtype == 0)
    gemm_simt_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(A),
                                                 static_cast<const float*>(W),
                                                 static_cast<float*>(C), M, N, K);
  else
    gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(W),
        static_cast<__nv_bfloat16*>(C), M, N, K);
  return cudaGetLastError();
}

}  // namespace attn
