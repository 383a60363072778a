// Log-sum-exp merge of split-KV partial states (the FlashAttention combination rule of
// "Building a Transformer from Scratch", Part 3): partial p of one (sequence, head) holds
// its maximum m_p (natural-log units), denominator l_p and unnormalised output O_p; the
// merged output is sum_p e^(m_p - M) O_p / sum_p e^(m_p - M) l_p with M = max_p m_p.
#pragma once
#include "common.cuh"

namespace attn {

// Merges n partials in one warp. Partial p's maximum and sum are at m0[p * mstride] and
// l0[p * mstride], its output at O0 + p * ostride (hd floats). The lanes read the maxima
// and sums in parallel, then each lane adds up output features lane, lane + 32, ... with
// several partials' loads in flight. Returns the unnormalised sums in acc, the maximum in
// M and the denominator in den (all lanes). A partial that saw no key (m = -inf) wrote no
// output and gets weight 0.
template <int NI>
__device__ __forceinline__ void warp_merge(const float* m0, const float* l0, const float* O0, size_t mstride,
                                           size_t ostride, int n, int hd, int lane, float (&acc)[NI],
                                           float& M, float& den) {
  M = -INFINITY;
  for (int c = lane; c < n; c += 32) M = fmaxf(M, m0[c * mstride]);
  M = warp_max(M);
  den = 0.f;
#pragma unroll
  for (int i = 0; i < NI; ++i) acc[i] = 0.f;
  if (M == -INFINITY) return;
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int c = c0 + lane;
    const float mc = c < n ? m0[c * mstride] : -INFINITY;
    const float wc = mc == -INFINITY ? 0.f : expf(mc - M);
    if (wc != 0.f) den += wc * l0[c * mstride];
    const int k1 = min(32, n - c0);
#pragma unroll 4
    for (int k = 0; k < k1; ++k) {
      const float w = __shfl_sync(0xffffffffu, wc, k);
      const float* Oc = O0 + (size_t)(c0 + k) * ostride;
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const int d = lane + 32 * i;
        const float o = d < hd ? Oc[d] : 0.f;
        acc[i] = fmaf(w, w != 0.f ? o : 0.f, acc[i]);
      }
    }
  }
  den = warp_sum(den);
}

}  // namespace attn
