// Pre-norm helpers of the fused attention sub-layer (attn_block_fused). RMSNorm ("Building a
// Transformer from Scratch", RMSNorm and Pre-LN residuals: x / sqrt(mean(x^2) + eps) * gamma)
// is not materialised: since (x / r) * gamma @ W = (x @ diag(gamma) W) / r for the row's
// r = sqrt(mean(x^2) + eps), the sub-layer multiplies x by the weights with gamma folded into
// their rows and scales each output row by 1 / r in the GEMM epilogue. Here: the per-row 1 / r,
// the folded weights, and the (cos, sin) table the key epilogue turns by.
#include "kernels.h"
namespace attn {
namespace {

// 1 / sqrt(mean(x^2) + eps) of each row: one warp per row, 16-byte loads, fp32 sum of squares.
__global__ void rms_inverse_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ rinv, int M, int d,
                                   float eps) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * d);
  float ss = 0.f;
  for (int c = lane; c < d / 8; c += 32) {
    const uint4 u = __ldg(xr + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = __uint_as_float(w[i] << 16), b = __uint_as_float(w[i] & 0xffff0000u);
      ss = fmaf(a, a, fmaf(b, b, ss));
    }
  }
  ss = warp_sum(ss);
  if (lane == 0) rinv[row] = 1.f / sqrtf(ss / (float)d + eps);
}

// Wg[k][n] = gamma[k] W[k][n] (bf16, rounded to nearest even), 8 elements per thread.
__global__ void fold_gamma_kernel(const __nv_bfloat16* __restrict__ W, const __nv_bfloat16* __restrict__ gamma,
                                  __nv_bfloat16* __restrict__ Wg, int d, int N) {
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;  // first element
  if (i >= (size_t)d * N) return;
  const float g = __bfloat162float(gamma[i / N]);  // N % 8 == 0: the 8 elements share a row
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(W + i));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(w[e] << 16) * g,
                                                   __uint_as_float(w[e] & 0xffff0000u) * g);
    o[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(Wg + i) = make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void rope_table_kernel(float2* __restrict__ cs, int T, int pos0, const RopeFreqs rope, int half) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * half) return;
  const int t = i / half, c = i - t * half;
  float co, si;
  rope_cos_sin(pos0 + t, rope.hi[c], rope.lo[c], co, si);
  cs[i] = make_float2(co, si);
}

}  // namespace

cudaError_t launch_rms_inverse(const void* x, float* rinv, int M, int d, float eps, cudaStream_t s) {
  rms_inverse_kernel<<<(M + 7) / 8, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), rinv, M, d, eps);
  return cudaGetLastError();
}

cudaError_t launch_fold_gamma(const void* W, const void* gamma, void* Wg, int d, int N, cudaStream_t s) {
  const size_t chunks = (size_t)d * N / 8;
  fold_gamma_kernel<<<(unsigned)((chunks + 255) / 256), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(W),
                                                                     static_cast<const __nv_bfloat16*>(gamma),
                                                                     static_cast<__nv_bfloat16*>(Wg), d, N);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* cs, int T, int pos0, const RopeFreqs& rope, int hd, cudaStream_t s) {
  const int n = T * (hd / 2);
  rope_table_kernel<<<(n + 255) / 256, 256, 0, s>>>(cs, T, pos0, rope, hd / 2);
  return cudaGetLastError();
}

}  // namespace attn
