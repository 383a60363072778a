// CUDA-core flash prefill for fp32 (and bf16 shapes the tensor-core kernel does not
// take). It follows the key-block recurrences of "Building grouped-query attention with
// RoPE and Flash Attention from scratch", Step 3: a running maximum m, a running
// denominator l and a rescaled partial output per query row, divided by l at the end.
//
// One CTA of 128 threads owns BQ = 16 query rows of one (batch, query head); each warp
// owns 4 rows. Key/value blocks of BK = 32 rows are staged in shared memory as fp32,
// with the keys turned by the rotary embedding as they are loaded (RoPE on load); the
// query rows are turned once when the CTA starts. Lane j of a warp scores key j of the
// block; lane d accumulates output feature d (and d + 32, ...).
//
// Masked pairs get weight exactly 0 and every sum runs in an order fixed by the tile
// structure alone, so a row's result never depends on the keys it may not see.
#include "kernels.h"

namespace attn {
namespace {

constexpr int BQ = 16;
constexpr int BK = 32;
constexpr int ROWS_PER_WARP = BQ / 4;
constexpr int MAX_NT = ATTN_MAX_HD / 32;

template <typename T>
__global__ void __launch_bounds__(128) prefill_simt_kernel(const PrefillParams p) {
  extern __shared__ float smem[];
  const int hd = p.hd;
  const int half = hd / 2;
  float* Qs = smem;                       // [BQ][hd]
  float* Ks = Qs + BQ * hd;               // [BK][hd + 1]
  float* Vs = Ks + BK * (hd + 1);         // [BK][hd]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * BQ;
  const int g = h / (p.H / p.KV);
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
  const T* v = static_cast<const T*>(p.v);
  T* out = static_cast<T*>(p.out);
  const size_t qrow = (size_t)p.H * hd, kvrow = (size_t)p.KV * hd;

  // Query rows of this block, turned at their positions.
  for (int idx = tid; idx < BQ * half; idx += blockDim.x) {
    const int r = idx / half, c = idx - r * half;
    const int i = q0 + r;
    float x = 0.f, y = 0.f;
    if (i < p.T) {
      const float2 e = Elem<T>::load2(q + ((size_t)b * p.T + i) * qrow + (size_t)h * hd + 2 * c);
      x = e.x;
      y = e.y;
      if (p.rope.on) {
        float cs, sn;
        rope_cos_sin(p.pos0 + i, p.rope.hi[c], p.rope.lo[c], cs, sn);
        rotate_pair(x, y, cs, sn);
      }
    }
    Qs[r * hd + 2 * c] = x;
    Qs[r * hd + 2 * c + 1] = y;
  }

  // Key range the block needs: [k_lo, k_hi] (inclusive).
  const int q_last = min(q0 + BQ, p.T) - 1;
  int k_hi = p.causal ? q_last : p.T - 1;
  int k_lo = (p.window > 0) ? max(0, q0 - p.window + 1) : 0;
  const float slope = p.alibi.on ? p.alibi.slope[h] : 0.f;

  float m[ROWS_PER_WARP], l[ROWS_PER_WARP], o[ROWS_PER_WARP][MAX_NT];
#pragma unroll
  for (int r = 0; r < ROWS_PER_WARP; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int t = 0; t < MAX_NT; ++t) o[r][t] = 0.f;
  }

  for (int kb = (k_lo / BK) * BK; kb <= k_hi; kb += BK) {
    __syncthreads();  // previous block's K/V fully consumed (and Qs written on entry)
    for (int idx = tid; idx < BK * half; idx += blockDim.x) {
      const int r = idx / half, c = idx - r * half;
      const int j = kb + r;
      float kx = 0.f, ky = 0.f, vx = 0.f, vy = 0.f;
      if (j < p.T) {
        const size_t off = ((size_t)b * p.T + j) * kvrow + (size_t)g * hd + 2 * c;
        const float2 ke = Elem<T>::load2(k + off);
        const float2 ve = Elem<T>::load2(v + off);
        kx = ke.x; ky = ke.y; vx = ve.x; vy = ve.y;
        if (p.rope.on && !p.k_rotated) {
          float cs, sn;
          rope_cos_sin(p.pos0 + j, p.rope.hi[c], p.rope.lo[c], cs, sn);
          rotate_pair(kx, ky, cs, sn);
        }
      }
      Ks[r * (hd + 1) + 2 * c] = kx;
      Ks[r * (hd + 1) + 2 * c + 1] = ky;
      Vs[r * hd + 2 * c] = vx;
      Vs[r * hd + 2 * c + 1] = vy;
    }
    __syncthreads();

#pragma unroll
    for (int rr = 0; rr < ROWS_PER_WARP; ++rr) {
      const int r = warp * ROWS_PER_WARP + rr;
      const int i = q0 + r;
      if (i >= p.T) continue;  // warp-uniform
      const int j = kb + lane;
      const bool ok = (j < p.T) && key_allowed(i, j, p.causal, p.window);
      float s = -INFINITY;
      if (ok) {
        const float* qr = Qs + r * hd;
        const float* kr = Ks + lane * (hd + 1);
        float acc = 0.f;
        for (int d = 0; d < hd; ++d) acc = fmaf(qr[d], kr[d], acc);
        s = acc * p.scale - slope * fabsf((float)(i - j));
      }
      const float m_new = fmaxf(m[rr], warp_max(s));
      if (m_new == -INFINITY) continue;  // nothing allowed yet for this row (warp-uniform)
      const float alpha = (m[rr] == -INFINITY) ? 0.f : expf(m[rr] - m_new);
      const float pj = ok ? expf(s - m_new) : 0.f;
      l[rr] = l[rr] * alpha + warp_sum(pj);
      m[rr] = m_new;
#pragma unroll
      for (int t = 0; t < MAX_NT; ++t) {
        const int d = lane + 32 * t;
        if (32 * t >= hd) break;
        float acc = o[rr][t] * alpha;
#pragma unroll 8
        for (int jj = 0; jj < BK; ++jj) {
          const float pw = __shfl_sync(0xffffffffu, pj, jj);
          if (d < hd) acc = fmaf(pw, Vs[jj * hd + d], acc);
        }
        o[rr][t] = acc;
      }
    }
  }

#pragma unroll
  for (int rr = 0; rr < ROWS_PER_WARP; ++rr) {
    const int i = q0 + warp * ROWS_PER_WARP + rr;
    if (i >= p.T) continue;
    const float inv = (l[rr] > 0.f) ? 1.f / l[rr] : 0.f;
    T* orow = out + ((size_t)b * p.T + i) * qrow + (size_t)h * hd;
#pragma unroll
    for (int t = 0; t < MAX_NT; ++t) {
      const int d = lane + 32 * t;
      if (32 * t >= hd) break;
      if (d < hd) Elem<T>::store(orow + d, o[rr][t] * inv);
    }
    if (p.lse && lane == 0)
      p.lse[((size_t)b * p.H + h) * p.T + i] = (l[rr] > 0.f) ? m[rr] + logf(l[rr]) : -INFINITY;
  }
}

template <typename T>
cudaError_t launch_t(const PrefillParams& p, cudaStream_t s) {
  const size_t smem = sizeof(float) * ((size_t)BQ * p.hd + (size_t)BK * (p.hd + 1) + (size_t)BK * p.hd);
  cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.T + BQ - 1) / BQ, p.H, p.B);
  prefill_simt_kernel<T><<<grid, 128, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillParams& p, int dtype, cudaStream_t s) {
  return dtype == 0 ? launch_t<float>(p, s) : launch_t<__nv_bfloat16>(p, s);
}

}  // namespace attn
