// Pieces shared by the two tensor-core prefill kernels (prefill_tc.cu, prefill_pair.cu):
// the in-place rotary turn of a swizzled tile, a tree maximum, and the 4-D tensor maps of
// q/k/v (or a cache).
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "tc_common.cuh"

namespace attn {
namespace tc {

constexpr int PF_BM = 128;  // query rows per slot
constexpr int PF_BN = 128;  // keys per tile

// Maximum of 32 values as a tree (depth 4) rather than a chain of dependent steps.
__device__ __forceinline__ float max32(const float (&x)[32]) {
  float a[11];
#pragma unroll
  for (int k = 0; k < 10; ++k) a[k] = max3(x[3 * k], x[3 * k + 1], x[3 * k + 2]);
  a[10] = fmaxf(x[30], x[31]);
  const float b0 = max3(a[0], a[1], a[2]), b1 = max3(a[3], a[4], a[5]);
  const float b2 = max3(a[6], a[7], a[8]), b3 = fmaxf(a[9], a[10]);
  return fmaxf(max3(b0, b1, b2), b3);
}

// Rotation of a whole key (or query) tile by the 128 threads of the rotary warpgroup. Thread t owns
// one 16-byte chunk (4 pairs) of the row and the rows phase, phase + PH, phase + 2 PH ...
// Along those rows the angle of a pair grows by the fixed step PH * w, so the cosine and
// sine follow the angle-addition recurrence (c, s) <- (c C - s S, s C + c S) with (C, S)
// the step's cosine and sine, computed once per CTA. A query tile's start angle is computed
// accurately; consecutive key tiles take theirs from the previous one by the same recurrence
// with the step 128 w (rotate_next), so fp32 rounding builds up over the tiles of one CTA
// (a few hundred steps at most, far below bf16 resolution). Eight threads of a quarter warp
// cover the 8 chunks of one 128-byte row: shared-memory accesses are free of bank
// conflicts. Only FMA-pipe arithmetic runs per element.
template <int HD>
struct KRot {
  static constexpr int CH = HD / 8;       // 16-byte chunks per row
  static constexpr int PH = 128 / CH;     // row step between a thread's rows
  static constexpr int NR = PF_BN / PH;      // rows per thread
  int chunk, phase;
  float stepc[4], steps[4];
  f2x TC[2], TS[2];  // cosine and sine of the key-tile step 128 w (pairs 0-1, 2-3 of the chunk)
  f2x KC[2], KS[2];  // start angle of the next key tile
  __device__ __forceinline__ void init(int t, const RopeFreqs& rope) {
    chunk = t % CH;
    phase = t / CH;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int pc = chunk * 4 + e;
      rope_cos_sin(PH, rope.hi[pc], rope.lo[pc], stepc[e], steps[e]);
    }
  }
  // The key tiles that follow start at position pos_row0 (first tile), pos_row0 + 128, ...
  __device__ __forceinline__ void start_keys(int pos_row0, const RopeFreqs& rope) {
    float c[4], sn[4], tc[4], ts[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int pc = chunk * 4 + e;
      rope_cos_sin(pos_row0 + phase, rope.hi[pc], rope.lo[pc], c[e], sn[e]);
      rope_cos_sin(PF_BN, rope.hi[pc], rope.lo[pc], tc[e], ts[e]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      KC[h] = pk2(c[2 * h], c[2 * h + 1]);
      KS[h] = pk2(sn[2 * h], sn[2 * h + 1]);
      TC[h] = pk2(tc[2 * h], tc[2 * h + 1]);
      TS[h] = pk2(ts[2 * h], ts[2 * h + 1]);
    }
  }
  // Rotate the next key tile, then advance the start angle by 128 rows.
  __device__ __forceinline__ void rotate_next(uint8_t* tile) {
    rotate_from(tile, KC, KS);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const f2x Cn = fma2(neg2(KS[h]), TS[h], mul2(KC[h], TC[h]));
      KS[h] = fma2(KC[h], TS[h], mul2(KS[h], TC[h]));
      KC[h] = Cn;
    }
  }
  // Rotate a tile whose first row sits at position pos_row0 (start angle computed accurately).
  __device__ __forceinline__ void rotate(uint8_t* tile, int pos_row0, const RopeFreqs& rope) const {
    float c[4], sn[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int pc = chunk * 4 + e;
      rope_cos_sin(pos_row0 + phase, rope.hi[pc], rope.lo[pc], c[e], sn[e]);
    }
    const f2x C0[2] = {pk2(c[0], c[1]), pk2(c[2], c[3])};
    const f2x S0[2] = {pk2(sn[0], sn[1]), pk2(sn[2], sn[3])};
    rotate_from(tile, C0, S0);
  }
  __device__ __forceinline__ void rotate_from(uint8_t* tile, const f2x (&C0)[2], const f2x (&S0)[2]) const {
    // pairs (0, 1) and (2, 3) of the chunk are handled two at a time in packed f32x2 form
    f2x C[2], S[2], N[2], SC[2], SS[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      C[h] = C0[h];
      S[h] = S0[h];
      N[h] = neg2(S[h]);
      SC[h] = pk2(stepc[2 * h], stepc[2 * h + 1]);
      SS[h] = pk2(steps[2 * h], steps[2 * h + 1]);
    }
    const uint32_t base = smem_u32(tile);
#pragma unroll 4
    for (int k = 0; k < NR; ++k) {
      const int r = phase + PH * k;
      const uint32_t addr = base + sw128_offset(r, chunk * 8, PF_BN);
      const uint4 u = lds128(addr);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t wa = w[2 * h], wb = w[2 * h + 1];
        const f2x X = pk2(__uint_as_float(wa << 16), __uint_as_float(wb << 16));
        const f2x Y = pk2(__uint_as_float(wa & 0xffff0000u), __uint_as_float(wb & 0xffff0000u));
        const f2x Xr = fma2(Y, N[h], mul2(X, C[h]));   // x c - y s
        const f2x Yr = fma2(X, S[h], mul2(Y, C[h]));   // x s + y c
        float xa, xb, ya, yb;
        up2(Xr, xa, xb);
        up2(Yr, ya, yb);
        o[2 * h] = f2_to_bf2(xa, ya);
        o[2 * h + 1] = f2_to_bf2(xb, yb);
        // advance both angles by the step: (c, s) <- (c C - s S, s C + c S)
        const f2x Cn = fma2(N[h], SS[h], mul2(C[h], SC[h]));
        S[h] = fma2(C[h], SS[h], mul2(S[h], SC[h]));
        C[h] = Cn;
        N[h] = neg2(S[h]);
      }
      sts128(addr, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
};

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 4-D map over [B][T][heads][hd] bf16 with a box of 128 rows x 64 features of one head.
inline bool make_map(CUtensorMap* map, const void* base, int B, int T, int heads, int hd) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)hd * 2, (cuuint64_t)heads * hd * 2,
                                 (cuuint64_t)T * heads * hd * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace attn
