// KV-cache decode: one new query per sequence over its cache ("Building a Transformer
// from Scratch: Attention, Architecture, and Memory", Part 3 "KV caching"), split over
// the keys and merged with the log-sum-exp rule of the FlashAttention section's online
// softmax (m = max m_c, l = sum exp(m_c - m) l_c, O = sum exp(m_c - m) O_c / l).
//
// bf16 with hd 64 or 128 runs on the tensor cores (decode_tc.cu: its own work split and
// merge). Otherwise pass 1 is the CUDA-core kernel below, one CTA per (split, key/value head, sequence): the CTA
// reads its chunk of cache rows once, 16 bytes per lane per load, and serves every query
// head of the group from those rows. Each warp owns a stream of keys; a key row of hd bf16 is covered by
// hd/8 lanes, so one warp load instruction covers 32*8/hd rows. Per key the group's
// scores are reduced across the lanes of the row; weights are formed with a running
// maximum per warp and head, and each lane accumulates the group's outputs for its 8
// features. The warps' partial states are combined in shared memory at the end of the
// chunk and written to the workspace as (O unnormalised, m, l).
// Pass 2 merges the splits of each (sequence, head) and writes out and lse.
#include "kernels.h"
#include "merge.cuh"

namespace attn {
namespace {

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;

// Partial-state layout in the workspace for nsplit splits:
//   O [B][H][nsplit][hd] fp32, then m [B][H][nsplit], then l [B][H][nsplit].
struct Partials {
  float* O;
  float* m;
  float* l;
};

__host__ __device__ inline Partials partials(void* ws, int B, int H, int hd, int nsplit) {
  Partials P;
  P.O = static_cast<float*>(ws);
  P.m = P.O + (size_t)B * H * nsplit * hd;
  P.l = P.m + (size_t)B * H * nsplit;
  return P;
}

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
  // 8 bf16 = 16 bytes
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

// G: query heads per key/value head (compile time, 1..32). Lanes per key row: LPR = hd/8.
template <typename T, int G>
__global__ void __launch_bounds__(DEC_THREADS) decode_split_kernel(const DecodeParams p, int chunk,
                                                                    int nsplit, void* ws) {
  extern __shared__ float sm[];
  const int hd = p.hd;
  const int LPR = hd / 8;              // lanes per key row (8, 16 or 32)
  const int RPW = 32 / LPR;            // key rows per warp load
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPR;          // which row of the warp's group of RPW rows
  const int fl = lane % LPR;           // which 8 features of the row
  const Partials P = partials(ws, p.B, p.H, hd, nsplit);

  int L = p.seqlens[b];
  const int qp = p.qpos[b];
  if (L < 0 || L > p.Lmax || qp < 0 || qp >= (1 << 24)) {
    if (split == 0 && kvh == 0 && tid == 0) flag_error(p.status, DEV_BAD_ARG);
    L = 0;
  }
  int j0 = split * chunk;
  int j1 = min(L, j0 + chunk);
  if (p.window > 0) j0 = max(j0, qp - p.window + 1);

  // Group queries for this lane's 8 features, turned at qpos and pre-scaled.
  float qv[G][8];
  const T* q = static_cast<const T*>(p.q);
#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    const int h = kvh * G + gg;
    const T* qr = q + ((size_t)b * p.H + h) * hd + fl * 8;
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = Elem<T>::load(qr + e);
    if (p.rope.on) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = fl * 4 + e;
        float cs, sn;
        rope_cos_sin(qp, p.rope.hi[c], p.rope.lo[c], cs, sn);
        rotate_pair(x[2 * e], x[2 * e + 1], cs, sn);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[gg][e] = x[e] * p.scale;
  }
  float slope[G];
#pragma unroll
  for (int gg = 0; gg < G; ++gg) slope[gg] = p.alibi.on ? p.alibi.slope[kvh * G + gg] : 0.f;

  float m[G], l[G], o[G][8];
#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    m[gg] = -INFINITY;
    l[gg] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[gg][e] = 0.f;
  }

  const T* kc = static_cast<const T*>(p.kcache);
  const T* vc = static_cast<const T*>(p.vcache);
  const size_t row = (size_t)p.KV * hd;
  const size_t base = (size_t)b * p.Lmax * row + (size_t)kvh * hd + fl * 8;

  // Warp w takes rows j0 + (w*RPW + sub) + t*DEC_WARPS*RPW.
  const int stride = DEC_WARPS * RPW;
  for (int jb = j0 + warp * RPW; jb < j1; jb += stride) {
    const int j = jb + sub;
    const bool live = j < j1;
    float kx[8], vx[8];
    if (live) {
      Vec8<T>::load(kc + base + (size_t)j * row, kx);
      Vec8<T>::load(vc + base + (size_t)j * row, vx);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) { kx[e] = 0.f; vx[e] = 0.f; }
    }
    float s[G];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(qv[gg][e], kx[e], acc);
      s[gg] = acc;
    }
    // reduce across the LPR lanes of the row (xor over the low bits stays in the row)
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      for (int off = LPR / 2; off > 0; off >>= 1) s[gg] += __shfl_xor_sync(0xffffffffu, s[gg], off);
    }
    // online update; each row's lanes update with their own key (rows of a warp
    // are merged at the end, so every lane keeps its own (m, l, o) per head)
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const float sc = live ? s[gg] - slope[gg] * fabsf((float)(qp - j)) : -INFINITY;
      const float m_new = fmaxf(m[gg], sc);
      if (m_new == -INFINITY) continue;
      const float alpha = __expf(m[gg] - m_new);  // m = -inf gives 0
      const float pw = __expf(sc - m_new);
      l[gg] = l[gg] * alpha + pw;
      m[gg] = m_new;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[gg][e] = fmaf(pw, vx[e], o[gg][e] * alpha);
    }
  }

  // Combine the RPW rows of each warp (lanes with equal fl), then the warps, in smem.
#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    for (int off = LPR; off < 32; off <<= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[gg], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[gg], off);
      const float mn = fmaxf(m[gg], mo);
      const float a = (mn == -INFINITY) ? 0.f : __expf(m[gg] - mn);
      const float bb = (mn == -INFINITY) ? 0.f : __expf(mo - mn);
      l[gg] = l[gg] * a + lo * bb;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float oo = __shfl_xor_sync(0xffffffffu, o[gg][e], off);
        o[gg][e] = o[gg][e] * a + oo * bb;
      }
      m[gg] = mn;
    }
  }
  // smem: per warp, per head: m, l, o[hd]
  float* sw = sm;  // [DEC_WARPS][G][hd + 2]
  if (sub == 0) {
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float* dst = sw + ((size_t)warp * G + gg) * (hd + 2);
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[2 + fl * 8 + e] = o[gg][e];
      if (fl == 0) { dst[0] = m[gg]; dst[1] = l[gg]; }
    }
  }
  __syncthreads();
  // Thread t merges (head, feature) pairs across warps.
  for (int idx = tid; idx < G * hd; idx += DEC_THREADS) {
    const int gg = idx / hd, d = idx - gg * hd;
    float M = -INFINITY;
    for (int w = 0; w < DEC_WARPS; ++w) M = fmaxf(M, sw[((size_t)w * G + gg) * (hd + 2)]);
    float acc = 0.f, den = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < DEC_WARPS; ++w) {
        const float* src = sw + ((size_t)w * G + gg) * (hd + 2);
        const float a = __expf(src[0] - M);
        acc += a * src[2 + d];
        den += a * src[1];
      }
    }
    const int h = kvh * G + gg;
    const size_t pi = ((size_t)b * p.H + h) * nsplit + split;
    P.O[pi * hd + d] = acc;
    if (d == 0) {
      P.m[pi] = M;
      P.l[pi] = den;
    }
  }
}

// One warp per (sequence, head): four heads of one sequence per CTA.
template <typename T>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p, int chunk, int nsplit, const void* ws) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * 4 + warp, b = blockIdx.y;
  if (h >= p.H) return;
  const int hd = p.hd;
  const Partials P = partials(const_cast<void*>(ws), p.B, p.H, hd, nsplit);
  int L = p.seqlens[b];
  if (L < 0 || L > p.Lmax || p.qpos[b] < 0 || p.qpos[b] >= (1 << 24)) L = 0;
  const int used = min(nsplit, (L + chunk - 1) / chunk);
  const size_t pi0 = ((size_t)b * p.H + h) * nsplit;
  float acc[ATTN_MAX_HD / 32], M, den;
  warp_merge(P.m + pi0, P.l + pi0, P.O + pi0 * hd, 1, hd, used, hd, lane, acc, M, den);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  T* out = static_cast<T*>(p.out) + ((size_t)b * p.H + h) * hd;
#pragma unroll
  for (int i = 0; i < ATTN_MAX_HD / 32; ++i)
    if (lane + 32 * i < hd) Elem<T>::store(out + lane + 32 * i, acc[i] * inv);
  if (p.lse && lane == 0) p.lse[(size_t)b * p.H + h] = den > 0.f ? M + logf(den) : -INFINITY;
}

template <typename T, int G>
cudaError_t launch_g(const DecodeParams& p, int chunk, int nsplit, void* ws, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)DEC_WARPS * G * (p.hd + 2);
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<T, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(nsplit, p.KV, p.B);
  decode_split_kernel<T, G><<<grid, DEC_THREADS, smem, s>>>(p, chunk, nsplit, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<T><<<dim3((p.H + 3) / 4, p.B), 128, 0, s>>>(p, chunk, nsplit, ws);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const DecodeParams& p, void* ws, cudaStream_t s) {
  if (decode_tc_supported(p, sizeof(T) == 2 ? 1 : 0)) return launch_decode_tc(p, ws, s);
  if (p.W_out) return cudaErrorInvalidValue;  // the up-projection is on the tensor-core path only
  const int chunk = decode_chunk(p.B, p.KV, p.Lmax);
  const int nsplit = (p.Lmax + chunk - 1) / chunk;
  switch (p.H / p.KV) {
    case 1: return launch_g<T, 1>(p, chunk, nsplit, ws, s);
    case 2: return launch_g<T, 2>(p, chunk, nsplit, ws, s);
    case 4: return launch_g<T, 4>(p, chunk, nsplit, ws, s);
    case 8: return launch_g<T, 8>(p, chunk, nsplit, ws, s);
    case 16: return launch_g<T, 16>(p, chunk, nsplit, ws, s);
    case 32: return launch_g<T, 32>(p, chunk, nsplit, ws, s);
    default: return cudaErrorInvalidValue;
  }
}

// Row t of sequence b (block (b, t)) goes to slot pos[b] + t, its key turned at that position.
template <typename T>
__global__ void kv_append_kernel(const AppendParams p) {
  const int b = blockIdx.x, t = blockIdx.y;
  const int pos = p.pos[b] + t;
  if (p.pos[b] < 0 || pos < 0 || pos >= p.Lmax) {
    if (threadIdx.x == 0) flag_error(p.status, DEV_BAD_ARG);
    return;
  }
  const int half = p.hd / 2;
  size_t row = (size_t)b * p.Lmax + pos;  // row of the cache viewed as [rows][KV][hd]
  if (p.block_table) {
    const int page = p.block_table[(size_t)b * p.max_blocks + pos / p.page_size];
    if (page < 0 || page >= p.num_pages) {
      if (threadIdx.x == 0) flag_error(p.status, DEV_BAD_ARG);
      return;
    }
    row = (size_t)page * p.page_size + pos % p.page_size;
  }
  const T* kn = static_cast<const T*>(p.k_new) + ((size_t)b * p.Tn + t) * p.KV * p.hd;
  const T* vn = static_cast<const T*>(p.v_new) + ((size_t)b * p.Tn + t) * p.KV * p.hd;
  T* kc = static_cast<T*>(p.kcache) + row * p.KV * p.hd;
  T* vc = static_cast<T*>(p.vcache) + row * p.KV * p.hd;
  for (int idx = threadIdx.x; idx < p.KV * half; idx += blockDim.x) {
    const int g = idx / half, c = idx - g * half;
    const size_t off = (size_t)g * p.hd + 2 * c;
    float2 kx = Elem<T>::load2(kn + off);
    if (p.rope.on) {
      float cs, sn;
      rope_cos_sin(pos, p.rope.hi[c], p.rope.lo[c], cs, sn);
      rotate_pair(kx.x, kx.y, cs, sn);
    }
    Elem<T>::store2(kc + off, kx.x, kx.y);
    const float2 vx = Elem<T>::load2(vn + off);
    Elem<T>::store2(vc + off, vx.x, vx.y);
  }
}

}  // namespace

int decode_chunk(int B, int KV, int Lmax) {
  // Keys per split: 2048 (a multiple of the 128-key tile) unless that leaves fewer than
  // about two CTAs per SM on 148 SMs when every cache is full; then smaller, down to 256.
  const long long units = (long long)B * KV;
  long long chunk = 2048;
  while (chunk > 256 && units * (((long long)Lmax + chunk - 1) / chunk) < 2LL * 148) chunk /= 2;
  return (int)chunk;
}

size_t decode_workspace_bytes(int B, int H, int KV, int hd, int Lmax) {
  const int chunk = decode_chunk(B, KV, Lmax);
  const size_t nsplit = ((size_t)Lmax + chunk - 1) / chunk;
  const size_t split = sizeof(float) * (size_t)B * H * nsplit * (hd + 2);
  const size_t tc = (hd == 64 || hd == 128) ? decode_tc_workspace_bytes(B, H, KV, hd) : 0;
  return split > tc ? split : tc;
}

cudaError_t launch_decode(const DecodeParams& p, int dtype, void* ws, cudaStream_t s) {
  return dtype == 0 ? launch_t<float>(p, ws, s) : launch_t<__nv_bfloat16>(p, ws, s);
}

cudaError_t launch_kv_append(const AppendParams& p, int dtype, cudaStream_t s) {
  const dim3 grid(p.B, p.Tn);
  if (dtype == 0)
    kv_append_kernel<float><<<grid, 128, 0, s>>>(p);
  else
    kv_append_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace attn
