// Per-head projections of latent attention ("Write attention from scratch", exercise 5):
// the key up-projection folded into the query, q'_h = W_uk[h] q_h (hd -> dc), and the value
// up-projection applied to the attention's latent output, out_h = o_h W_uv[h] (dc -> hd).
// Between them the decode over the latent cache runs as a one-key/value-head decode of head
// dimension dc (decode_tc.cu), whose keys and values are the same cached latents.
//
// One CTA per (head, group of SEQ sequences): W[h] (dc x hd bf16, at most 64 KB) is staged in
// shared memory once and serves the group's vectors; fp32 accumulation.
#include "kernels.h"

namespace attn {
namespace {

constexpr int SEQ = 8;        // sequences per CTA
constexpr int THREADS = 256;

// fold: y[b,h,m] = sum_e W[h,m,e] x[b,h,e]   (x [B,H,hd], y [B,H,dc])
// out:  y[b,h,e] = sum_m W[h,m,e] x[b,h,m]   (x [B,H,dc], y [B,H,hd])
template <bool FOLD>
__global__ void __launch_bounds__(THREADS)
    head_proj_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W,
                     __nv_bfloat16* __restrict__ y, int B, int H, int dc, int hd) {
  extern __shared__ float sh[];
  const int h = blockIdx.x, b0 = blockIdx.y * SEQ;
  const int nb = min(SEQ, B - b0);
  const int nin = FOLD ? hd : dc, nout = FOLD ? dc : hd;
  float* Ws = sh;                          // [dc][hd]
  float* xs = sh + (size_t)dc * hd;        // [SEQ][nin]
  const __nv_bfloat16* Wh = W + (size_t)h * dc * hd;
  for (int i = threadIdx.x; i < dc * hd; i += THREADS) Ws[i] = __bfloat162float(Wh[i]);
  for (int i = threadIdx.x; i < nb * nin; i += THREADS) {
    const int s = i / nin, k = i - s * nin;
    xs[i] = __bfloat162float(x[((size_t)(b0 + s) * H + h) * nin + k]);
  }
  __syncthreads();
  if (FOLD) {
    // one warp per output m: lanes stride over the row Ws[m][:], then a warp reduction
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = THREADS >> 5;
    for (int m = warp; m < dc; m += nw) {
      float acc[SEQ];
#pragma unroll
      for (int s = 0; s < SEQ; ++s) acc[s] = 0.f;
      for (int e = lane; e < hd; e += 32) {
        const float w = Ws[m * hd + e];
#pragma unroll
        for (int s = 0; s < SEQ; ++s) acc[s] = fmaf(w, xs[s * nin + e], acc[s]);
      }
#pragma unroll
      for (int s = 0; s < SEQ; ++s) {
        float v = acc[s];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && s < nb) y[((size_t)(b0 + s) * H + h) * nout + m] = __float2bfloat16_rn(v);
      }
    }
  } else {
    // one thread per output e (consecutive threads read consecutive Ws[m][e])
    for (int e = threadIdx.x; e < hd; e += THREADS) {
      float acc[SEQ];
#pragma unroll
      for (int s = 0; s < SEQ; ++s) acc[s] = 0.f;
#pragma unroll 4
      for (int m = 0; m < dc; ++m) {
        const float w = Ws[m * hd + e];
#pragma unroll
        for (int s = 0; s < SEQ; ++s) acc[s] = fmaf(w, xs[s * nin + m], acc[s]);
      }
#pragma unroll
      for (int s = 0; s < SEQ; ++s)
        if (s < nb) y[((size_t)(b0 + s) * H + h) * nout + e] = __float2bfloat16_rn(acc[s]);
    }
  }
}

}  // namespace

cudaError_t launch_head_proj(bool fold, const void* x, const void* W, void* y, int B, int H, int dc, int hd,
                             cudaStream_t s) {
  const dim3 grid(H, (B + SEQ - 1) / SEQ);
  const size_t smem = sizeof(float) * ((size_t)dc * hd + (size_t)SEQ * (fold ? hd : dc));
  const auto* xx = static_cast<const __nv_bfloat16*>(x);
  const auto* ww = static_cast<const __nv_bfloat16*>(W);
  auto* yy = static_cast<__nv_bfloat16*>(y);
  cudaError_t e;
  if (fold) {
    e = cudaFuncSetAttribute(head_proj_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    head_proj_kernel<true><<<grid, THREADS, smem, s>>>(xx, ww, yy, B, H, dc, hd);
  } else {
    e = cudaFuncSetAttribute(head_proj_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    head_proj_kernel<false><<<grid, THREADS, smem, s>>>(xx, ww, yy, B, H, dc, hd);
  }
  return cudaGetLastError();
}

}  // namespace attn

