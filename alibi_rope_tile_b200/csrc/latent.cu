// Per-head projections of latent attention ("Write attention from scratch", exercise 5):
// the key up-projection folded into the query, q'_h = W_uk[h] q_h (hd -> dc), and the value
// up-projection applied to the attention's latent output, out_h = o_h W_uv[h] (dc -> hd).
// Between them the decode over the latent cache runs as a one-key/value-head decode of head
// dimension dc (decode_tc.cu), whose keys and values are the same cached latents.
//
// Both projections are small (H x dc x hd weights, one vector per (sequence, head)) and
// L2-resident; one CTA per (head, sequence) with fp32 accumulation.
#include "kernels.h"

namespace attn {
namespace {

// fold: y[b,h,m] = sum_e W[h,m,e] x[b,h,e]   (W [H][dc][hd], x [B,H,hd], y [B,H,dc])
// out:  y[b,h,e] = sum_m W[h,m,e] x[b,h,m]   (W [H][dc][hd], x [B,H,dc], y [B,H,hd])
template <bool FOLD>
__global__ void head_proj_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W,
                                 __nv_bfloat16* __restrict__ y, int H, int dc, int hd) {
  extern __shared__ float xs[];
  const int h = blockIdx.x, b = blockIdx.y;
  const int nin = FOLD ? hd : dc, nout = FOLD ? dc : hd;
  const __nv_bfloat16* xv = x + ((size_t)b * H + h) * nin;
  for (int i = threadIdx.x; i < nin; i += blockDim.x) xs[i] = __bfloat162float(xv[i]);
  __syncthreads();
  const __nv_bfloat16* Wh = W + (size_t)h * dc * hd;
  __nv_bfloat16* yv = y + ((size_t)b * H + h) * nout;
  if (FOLD) {
    // one warp per output m: lanes stride over the contiguous row W[h,m,:]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int m = warp; m < dc; m += nw) {
      float acc = 0.f;
      for (int e = lane; e < hd; e += 32) acc = fmaf(__bfloat162float(Wh[(size_t)m * hd + e]), xs[e], acc);
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) yv[m] = __float2bfloat16_rn(acc);
    }
  } else {
    // one thread per output e: consecutive threads read consecutive W[h,m,e]
    for (int e = threadIdx.x; e < hd; e += blockDim.x) {
      float acc = 0.f;
      for (int m = 0; m < dc; ++m) acc = fmaf(__bfloat162float(Wh[(size_t)m * hd + e]), xs[m], acc);
      yv[e] = __float2bfloat16_rn(acc);
    }
  }
}

}  // namespace

cudaError_t launch_head_proj(bool fold, const void* x, const void* W, void* y, int B, int H, int dc, int hd,
                             cudaStream_t s) {
  const dim3 grid(H, B);
  const size_t smem = sizeof(float) * (size_t)(fold ? hd : dc);
  const auto* xx = static_cast<const __nv_bfloat16*>(x);
  const auto* ww = static_cast<const __nv_bfloat16*>(W);
  auto* yy = static_cast<__nv_bfloat16*>(y);
  if (fold)
    head_proj_kernel<true><<<grid, 128, smem, s>>>(xx, ww, yy, H, dc, hd);
  else
    head_proj_kernel<false><<<grid, 128, smem, s>>>(xx, ww, yy, H, dc, hd);
  return cudaGetLastError();
}

}  // namespace attn
