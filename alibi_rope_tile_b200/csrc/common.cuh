// Shared device helpers of the attention core (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define ATTN_MAX_HD 256
#define ATTN_MAX_PAIRS (ATTN_MAX_HD / 2)
#define ATTN_MAX_ALIBI_HEADS 256

namespace attn {

// Rotary frequencies of one call, in turns per position: w_c = base^(-2c/hd) / (2 pi),
// computed on the host in double and split into an fp32 (hi, lo) pair so that the
// angle of pair c at an integer position p can be reduced modulo one turn exactly.
struct RopeFreqs {
  int on;
  float hi[ATTN_MAX_PAIRS];
  float lo[ATTN_MAX_PAIRS];
};

struct Alibi {
  int on;
  float slope[ATTN_MAX_ALIBI_HEADS];
};

// Device-side error codes written into the per-device status word.
enum DevStatus { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BAD_ARG = 2 };

__device__ __forceinline__ void flag_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Angle of pair c at position p, in turns, reduced to about [-1/2, 1/2]:
// t = p * (hi + lo) - round(p * hi). p * hi is split exactly into prod + err with one
// FMA (p < 2^24 is exact in fp32), so the reduction loses nothing.
__device__ __forceinline__ float rope_turns(int p, float hi, float lo) {
  const float pf = (float)p;
  const float prod = __fmul_rn(pf, hi);
  const float err = fmaf(pf, hi, -prod);
  return (prod - rintf(prod)) + fmaf(pf, lo, err);
}

// Accurate cos/sin of pair c at position p (CUDA's sincospif on the reduced angle).
__device__ __forceinline__ void rope_cos_sin(int p, float hi, float lo, float& c, float& s) {
  const float t = rope_turns(p, hi, lo);
  sincospif(2.0f * t, &s, &c);
}

// Turn the pair (x, y) by the angle whose cosine and sine are c and s.
__device__ __forceinline__ void rotate_pair(float& x, float& y, float c, float s) {
  const float rx = x * c - y * s;
  const float ry = x * s + y * c;
  x = rx;
  y = ry;
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
  static __device__ __forceinline__ float2 load2(const float* p) {
    return *reinterpret_cast<const float2*>(p);
  }
  static __device__ __forceinline__ void store2(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
  }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
  static __device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
  }
  static __device__ __forceinline__ void store2(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
  }
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Key range [lo, hi] a query at position i may see (inclusive), before the T clamp.
__device__ __forceinline__ bool key_allowed(int i, int j, int causal, int window) {
  if (causal && j > i) return false;
  if (window > 0 && i - j >= window) return false;
  return true;
}

}  // namespace attn
