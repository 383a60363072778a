// The key up-projection of latent attention ("Write attention from scratch", exercise 5) folded
// into the query: q'_h = W_uk[h] q_h (hd -> dc). Between this and the value up-projection (done
// by the merge of decode.cu) the decode over the latent cache runs as a one-key/value-head
// decode of head dimension dc (decode_tc.cu), whose keys and values are the same latents.
//
// One CTA per (head, group of SEQ sequences): thread m computes output m of every sequence of
// the group from row m of W_uk[h] (hd numbers, loaded into registers 128 at a time by 16-byte
// loads issued before the group's queries are staged) and the queries in shared memory (fp32),
// which all threads of a warp read at the same address (a broadcast). Each output is one fp32
// FMA chain over e = 0, 1, ..., hd - 1, rounded once to bf16.
#include "kernels.h"

namespace attn {
namespace {

constexpr int SEQ = 8;        // sequences per CTA
constexpr int THREADS = 128;  // >= dc (64 or 128)
constexpr int EC = 128;       // elements of a weight row held in registers at once

__global__ void __launch_bounds__(THREADS)
    latent_fold_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W,
                       __nv_bfloat16* __restrict__ y, int B, int H, int dc, int hd) {
  extern __shared__ float xs[];  // [SEQ][hd]
  // the decode that follows may start its independent set-up now (it waits for q')
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int h = blockIdx.x, b0 = blockIdx.y * SEQ;
  const int nb = min(SEQ, B - b0);
  const int m = threadIdx.x;
  const uint4* wr = reinterpret_cast<const uint4*>(W + ((size_t)h * dc + (m < dc ? m : 0)) * hd);
  uint4 u[EC / 8];
  auto load_w = [&](int e0) {
#pragma unroll
    for (int r = 0; r < EC / 8; ++r)
      if (e0 + 8 * r < hd) u[r] = __ldg(wr + e0 / 8 + r);
  };
  load_w(0);
  for (int c = threadIdx.x; c < nb * hd / 8; c += THREADS) {
    const int sq = c / (hd / 8), e0 = (c - sq * (hd / 8)) * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + ((size_t)(b0 + sq) * H + h) * hd + e0));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xs[sq * hd + e0 + 2 * i] = __uint_as_float(w[i] << 16);
      xs[sq * hd + e0 + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __syncthreads();
  if (m >= dc) return;
  float acc[SEQ];
#pragma unroll
  for (int s = 0; s < SEQ; ++s) acc[s] = 0.f;
  for (int e0 = 0; e0 < hd; e0 += EC) {
    if (e0 > 0) load_w(e0);
#pragma unroll
    for (int r = 0; r < EC / 8; ++r) {
      if (e0 + 8 * r >= hd) break;
      const uint32_t w[4] = {u[r].x, u[r].y, u[r].z, u[r].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float w0 = __uint_as_float(w[i] << 16), w1 = __uint_as_float(w[i] & 0xffff0000u);
        const int e = e0 + 8 * r + 2 * i;
#pragma unroll
        for (int s = 0; s < SEQ; ++s) {
          if (s < nb) {
            const float2 x2 = *reinterpret_cast<const float2*>(xs + s * hd + e);
            acc[s] = fmaf(w1, x2.y, fmaf(w0, x2.x, acc[s]));
          }
        }
      }
    }
  }
#pragma unroll
  for (int s = 0; s < SEQ; ++s)
    if (s < nb) y[((size_t)(b0 + s) * H + h) * dc + m] = __float2bfloat16_rn(acc[s]);
}

}  // namespace

cudaError_t launch_latent_fold(const void* x, const void* W, void* y, int B, int H, int dc, int hd,
                               cudaStream_t s) {
  if (dc > THREADS) return cudaErrorInvalidValue;
  const dim3 grid(H, (B + SEQ - 1) / SEQ);
  const size_t smem = sizeof(float) * (size_t)SEQ * hd;
  cudaError_t e = cudaFuncSetAttribute(latent_fold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  latent_fold_kernel<<<grid, THREADS, smem, s>>>(static_cast<const __nv_bfloat16*>(x),
                                                 static_cast<const __nv_bfloat16*>(W),
                                                 static_cast<__nv_bfloat16*>(y), B, H, dc, hd);
  return cudaGetLastError();
}

}  // namespace attn
