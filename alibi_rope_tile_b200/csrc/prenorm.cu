// Pre-norm helpers of the fused attention sub-layer (attn_block_fused): RMSNorm of the block
// input and the (cos, sin) table the QKV GEMM's epilogue turns q and k by.
#include "kernels.h"
namespace attn {
namespace {

// y = x / sqrt(mean(x^2) + eps) * gamma per row ("Building a Transformer from Scratch", RMSNorm
// and Pre-LN residuals); one CTA per row, fp32 sum of squares.
__global__ void rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ gamma,
                               __nv_bfloat16* __restrict__ y, int d, float eps) {
  __shared__ float part[32];
  const size_t row = blockIdx.x;
  const __nv_bfloat16* xr = x + row * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const float v = __bfloat162float(xr[i]);
    ss = fmaf(v, v, ss);
  }
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (threadIdx.x == 0) part[0] = 1.f / sqrtf(t / (float)d + eps);
  }
  __syncthreads();
  const float inv = part[0];
  for (int i = threadIdx.x; i < d; i += blockDim.x)
    y[row * d + i] = __float2bfloat16_rn(__bfloat162float(xr[i]) * inv * __bfloat162float(gamma[i]));
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

cudaError_t launch_rmsnorm(const void* x, const void* gamma, void* y, int M, int d, float eps, cudaStream_t s) {
  rmsnorm_kernel<<<M, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(gamma),
                                   static_cast<__nv_bfloat16*>(y), d, eps);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* cs, int T, int pos0, const RopeFreqs& rope, int hd, cudaStream_t s) {
  const int n = T * (hd / 2);
  rope_table_kernel<<<(n + 255) / 256, 256, 0, s>>>(cs, T, pos0, rope, hd / 2);
  return cudaGetLastError();
}

}  // namespace attn
