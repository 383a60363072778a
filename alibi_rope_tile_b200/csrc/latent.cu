// The key up-projection of latent attention ("Write attention from scratch", exercise 5) folded
// into the query: q'_h = W_uk[h] q_h (hd -> dc). Between this and the value up-projection (done
// by the merge of decode.cu) the decode over the latent cache runs as a one-key/value-head
// decode of head dimension dc (decode_tc.cu), whose keys and values are the same latents.
//
// One CTA per (head, group of SEQ sequences): W_uk[h] (dc x hd) is staged transposed in shared
// memory (fp32, rows padded by one word) and serves the group: thread m accumulates output m
// of every sequence of the group, reading W^T[e][m] (consecutive threads, consecutive m: no
// bank conflicts) and the query elements e..e+3 of each sequence as one broadcast 16-byte read.
#include "kernels.h"

namespace attn {
namespace {

constexpr int SEQ = 8;        // sequences per CTA
constexpr int THREADS = 128;  // >= dc (64 or 128)

__global__ void __launch_bounds__(THREADS)
    latent_fold_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W,
                       __nv_bfloat16* __restrict__ y, int B, int H, int dc, int hd) {
  extern __shared__ float sh[];
  // the decode that follows may start its independent set-up now (it waits for q')
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int h = blockIdx.x, b0 = blockIdx.y * SEQ;
  const int nb = min(SEQ, B - b0);
  const int ld = dc + 1;
  float* WT = sh;                       // [hd][dc + 1]: WT[e][m] = W[h][m][e]
  float* xs = sh + (size_t)hd * ld;     // [SEQ][hd]
  const __nv_bfloat16* Wh = W + (size_t)h * dc * hd;
  // 16-byte loads (eight consecutive e of one row m each, hd % 8 == 0), issued eight at a
  // time before any of them is stored, so their latencies overlap
  const int nchunk = dc * hd / 8;
  for (int c0 = threadIdx.x; c0 < nchunk; c0 += 8 * THREADS) {
    uint4 u[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int c = c0 + r * THREADS;
      if (c < nchunk) u[r] = __ldg(reinterpret_cast<const uint4*>(Wh) + c);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int c = c0 + r * THREADS;
      if (c >= nchunk) break;
      const int m = c / (hd / 8), e0 = (c - m * (hd / 8)) * 8;
      const uint32_t w[4] = {u[r].x, u[r].y, u[r].z, u[r].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        WT[(e0 + 2 * i) * ld + m] = __uint_as_float(w[i] << 16);
        WT[(e0 + 2 * i + 1) * ld + m] = __uint_as_float(w[i] & 0xffff0000u);
      }
    }
  }
  for (int c = threadIdx.x; c < nb * hd / 8; c += THREADS) {
    const int sq = c / (hd / 8), e0 = (c - sq * (hd / 8)) * 8;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + ((size_t)(b0 + sq) * H + h) * hd + e0));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xs[sq * hd + e0 + 2 * i] = __uint_as_float(w[i] << 16);
      xs[sq * hd + e0 + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __syncthreads();
  const int m = threadIdx.x;
  if (m >= dc) return;
  float acc[SEQ];
#pragma unroll
  for (int s = 0; s < SEQ; ++s) acc[s] = 0.f;
  // four e per step: four W^T reads and one 16-byte (broadcast) query read per sequence
#pragma unroll 2
  for (int e = 0; e < hd; e += 4) {
    const float w0 = WT[e * ld + m], w1 = WT[(e + 1) * ld + m];
    const float w2 = WT[(e + 2) * ld + m], w3 = WT[(e + 3) * ld + m];
#pragma unroll
    for (int s = 0; s < SEQ; ++s) {
      const float4 x4 = *reinterpret_cast<const float4*>(xs + s * hd + e);
      acc[s] = fmaf(w3, x4.w, fmaf(w2, x4.z, fmaf(w1, x4.y, fmaf(w0, x4.x, acc[s]))));
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
  const size_t smem = sizeof(float) * ((size_t)hd * (dc + 1) + (size_t)SEQ * hd);
  cudaError_t e = cudaFuncSetAttribute(latent_fold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  latent_fold_kernel<<<grid, THREADS, smem, s>>>(static_cast<const __nv_bfloat16*>(x),
                                                 static_cast<const __nv_bfloat16*>(W),
                                                 static_cast<__nv_bfloat16*>(y), B, H, dc, hd);
  return cudaGetLastError();
}

}  // namespace attn
