// Key rotation pass: k [B,T,KV,hd] (bf16) -> kr, the same keys turned by the rotary
// embedding at positions pos0 + t, so that the attention kernel that follows reads keys
// already turned. Each key tile is then turned once in all, not once per CTA that reads it.
//
// Rotation: "Write attention from scratch" (worked example, rope): the interleaved pair
// (2c, 2c+1) of a key at position p turns by the angle p * base^(-2c/hd). Angles come from
// the exact-reduction helper the other kernels use (rope_cos_sin); the turn is computed in
// fp32 and rounded once to bf16.
//
// Layout of the work: a CTA owns RK_POS consecutive positions. Its threads first compute the
// (cos, sin) of every pair at those positions into shared memory, then stream the rows of all
// sequences and key heads at those positions: for one sequence they form one contiguous run of
// RK_POS * KV * hd elements, read and written in 16-byte pieces (four pairs each) by
// consecutive threads. The pass is bound by HBM: it reads and writes the key tensor once.
#include <cuda_bf16.h>

#include "kernels.h"

namespace attn {
namespace {

constexpr int RK_THREADS = 256;
constexpr int RK_POS = 4;     // positions per CTA
constexpr int RK_UNROLL = 4;  // 16-byte pieces in flight per thread

__device__ __forceinline__ uint32_t turn_bf2(uint32_t w, float2 cs) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w);
  float x = __low2float(h), y = __high2float(h);
  rotate_pair(x, y, cs.x, cs.y);
  __nv_bfloat162 o = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&o);
}

__global__ void __launch_bounds__(RK_THREADS) rope_keys_kernel(const uint4* __restrict__ k, uint4* __restrict__ kr,
                                                              int B, int T, int KV, int chunks, int pos0,
                                                              const RopeFreqs rope) {
  __shared__ float2 cs[RK_POS][ATTN_MAX_PAIRS];
  // the attention kernel that follows may be scheduled now; it waits for this grid's
  // completion before it reads a key
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t0 = blockIdx.x * RK_POS;
  const int np = min(RK_POS, T - t0);  // positions of this CTA
  const int half = chunks * 4;         // pairs per key
  for (int i = threadIdx.x; i < np * half; i += RK_THREADS) {
    const int pp = i / half, c = i - pp * half;
    float co, si;
    rope_cos_sin(pos0 + t0 + pp, rope.hi[c], rope.lo[c], co, si);
    cs[pp][c] = make_float2(co, si);
  }
  __syncthreads();
  const int row = KV * chunks;     // 16-byte pieces per position
  const int per_b = np * row;      // pieces of one sequence in this CTA (contiguous)
  const int n = B * per_b;
  for (int base = 0; base < n; base += RK_THREADS * RK_UNROLL) {
    uint4 w[RK_UNROLL];
    size_t at[RK_UNROLL];
#pragma unroll
    for (int e = 0; e < RK_UNROLL; ++e) {
      const int u = base + e * RK_THREADS + threadIdx.x;
      if (u < n) {
        const int b = u / per_b, r = u - b * per_b;
        at[e] = ((size_t)b * T + t0) * row + r;
        w[e] = __ldg(k + at[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < RK_UNROLL; ++e) {
      const int u = base + e * RK_THREADS + threadIdx.x;
      if (u < n) {
        const int r = u % per_b;
        const int pp = r / row, c4 = (r % chunks) * 4;
        uint4 o;
        o.x = turn_bf2(w[e].x, cs[pp][c4]);
        o.y = turn_bf2(w[e].y, cs[pp][c4 + 1]);
        o.z = turn_bf2(w[e].z, cs[pp][c4 + 2]);
        o.w = turn_bf2(w[e].w, cs[pp][c4 + 3]);
        kr[at[e]] = o;
      }
    }
  }
}

}  // namespace

cudaError_t launch_rope_keys(const void* k, void* kr, int B, int T, int KV, int hd, int pos0,
                             const RopeFreqs& rope, cudaStream_t s) {
  if (hd % 8 != 0 || hd > ATTN_MAX_HD || B < 1 || T < 1 || KV < 1) return cudaErrorInvalidValue;
  const int chunks = hd / 8;
  rope_keys_kernel<<<(unsigned)((T + RK_POS - 1) / RK_POS), RK_THREADS, 0, s>>>(
      static_cast<const uint4*>(k), static_cast<uint4*>(kr), B, T, KV, chunks, pos0, rope);
  return cudaGetLastError();
}

}  // namespace attn
