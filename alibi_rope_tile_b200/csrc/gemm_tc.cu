// Tensor-core GEMM for the block projections (sm_100a): C[M,N] = A[M,K] @ W[K,N], bf16 in,
// fp32 accumulation in TMEM, bf16 out. The block applies its weights as x @ W with W
// stored [in, out] ("Write attention from scratch", worked example: x @ Wq ... ctx @ Wo),
// so W is consumed as stored: as the B operand it is MN-major (N contiguous), which the
// UMMA shared-memory descriptor expresses directly; nothing is transposed.
//
// One CTA computes a 128 x 256 tile of C. K is staged by 64 through a 4-stage TMA ring
// (A: one 128 x 64 box; W: four 64 x 64 boxes, 128-byte swizzle). Warp 4 issues the TMA
// loads, warp 5 allocates TMEM and issues the M=128, N=256, K=16 MMAs (four per stage),
// warps 0-3 read the accumulator back (one TMEM lane = one row of C per thread) and store
// bf16. Rows and columns past M, N are zero-filled on load and not stored.
//
// Epilogues (GemmEpilogue): a plain store; the fused block's QKV scatter, which sends each
// 32-column chunk (within one head, since hd is 64 or 128 and tiles start at multiples of 256)
// to q, k or v, turns q and k pairwise by the (cos, sin) table of its row's position, and
// also writes k and v rows into a KV cache; or the output projection plus a residual.
#include <cudaTypedefs.h>

#include <cstring>

#include "kernels.h"
#include "tc_common.cuh"

namespace attn {
namespace tcgemm {
namespace {

using namespace attn::tc;

constexpr int BM = 128, BN = 256, BK = 64, NS = 4;
constexpr int THREADS = 192;
constexpr int A_BYTES = BM * BK * 2;       // 16 KB
constexpr int B_BYTES = BK * BN * 2;       // 32 KB
constexpr int STAGE = A_BYTES + B_BYTES;
constexpr int OFF_BAR = NS * STAGE;
constexpr int SMEM = OFF_BAR + (2 * NS + 2) * 8 + 16 + 1024;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, 0, 1);
constexpr uint64_t WAIT_LIMIT_NS = 4000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 100000000ull;

struct GemmArgs {
  __nv_bfloat16* C;
  int M, N, K;
  int* status;
  GemmEpilogue ep;
};

__device__ __forceinline__ void store32(__nv_bfloat16* dst, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(dst + 8 * q) =
        make_uint4(f2_to_bf2(v[8 * q], v[8 * q + 1]), f2_to_bf2(v[8 * q + 2], v[8 * q + 3]),
                   f2_to_bf2(v[8 * q + 4], v[8 * q + 5]), f2_to_bf2(v[8 * q + 6], v[8 * q + 7]));
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                   const __grid_constant__ GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + NS;
  uint64_t* acc_full = full + 2 * NS;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int nk = (g.K + BK - 1) / BK;

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch(&tmA);
      tma_prefetch(&tmW);
      int kb = 0;
      for (; kb < nk; ++kb) {
        const int st = kb % NS, n = kb / NS;
        if (!mbar_wait(empty + st, (n & 1) ^ 1, abort_flag, g.status, WAIT_LIMIT_NS)) break;
        uint8_t* sa = smem + st * STAGE;
        // W boxes that start past N are not loaded: those columns of C are not stored
        const int nbv = min(BN / 64, (g.N - n0 + 63) / 64);
        mbar_expect_tx(full + st, A_BYTES + nbv * (BK * 128));
        tma_load_2d(sa, &tmA, full + st, kb * BK, m0);
        for (int nb = 0; nb < nbv; ++nb)
          tma_load_2d(sa + A_BYTES + nb * (BK * 128), &tmW, full + st, n0 + nb * 64, kb * BK);
      }
      // the copies issued last land before the CTA exits
      for (int w = (kb > NS ? kb - NS : 0); w < kb; ++w) mbar_wait_drain(full + w % NS, (w / NS) & 1, DRAIN_LIMIT_NS);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint64_t dA = smem_desc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t dW = smem_desc_sw128(smem_u32(smem + A_BYTES), BK * 128, 1024);
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % NS, n = kb / NS;
        if (!mbar_wait(full + st, n & 1, abort_flag, g.status, WAIT_LIMIT_NS)) break;
        tc_fence_after();
        const uint64_t so = (uint64_t)((st * STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_ss(tmem, dA + so + (uint64_t)((kk * 32) >> 4), dW + so + (uint64_t)((kk * 16 * 128) >> 4),
                  IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
        umma_commit(empty + st);
      }
      umma_commit(acc_full);
      umma_commit(drain);
      mbar_wait_drain(drain, 0, DRAIN_LIMIT_NS);  // every MMA completes before TMEM is freed
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = rows m0 + 32*w .. of C
    if (mbar_wait(acc_full, 0, abort_flag, g.status, WAIT_LIMIT_NS)) {
      tc_fence_after();
      const int row = m0 + warp * 32 + lane;
      const uint32_t t = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        tmem_ld32(t + c0, v);
        tmem_wait_ld();
        if (row < g.M && g.ep.mode == 1) {
          const GemmEpilogue& e = g.ep;
          const int n = n0 + c0;
          if (n < g.N) {
            const int b = row / e.T, t = row - b * e.T;
            const int hh = n / e.hd, d = n - hh * e.hd;
            const int region = hh < e.H ? 0 : (hh < e.H + e.KV ? 1 : 2);
            const int head = region == 0 ? hh : (region == 1 ? hh - e.H : hh - e.H - e.KV);
            if (region < 2 && e.rope_cs) {
              const float2* cs = e.rope_cs + (size_t)t * (e.hd / 2) + d / 2;
#pragma unroll
              for (int p = 0; p < 16; ++p) {
                const float2 c = cs[p];
                const float x = v[2 * p], y = v[2 * p + 1];
                v[2 * p] = x * c.x - y * c.y;
                v[2 * p + 1] = x * c.y + y * c.x;
              }
            }
            const int nh = region == 0 ? e.H : e.KV;
            __nv_bfloat16* base = static_cast<__nv_bfloat16*>(region == 0 ? e.q : (region == 1 ? e.k : e.v));
            store32(base + (((size_t)b * e.T + t) * nh + head) * e.hd + d, v);
            if (region > 0 && e.kcache) {
              __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(region == 1 ? e.kcache : e.vcache);
              store32(cache + (((size_t)b * e.Lmax + e.pos0 + t) * e.KV + head) * e.hd + d, v);
            }
          }
        } else if (row < g.M) {
          __nv_bfloat16* dst = g.C + (size_t)row * g.N + n0 + c0;
          if (g.ep.mode == 2) {
            const __nv_bfloat16* res = static_cast<const __nv_bfloat16*>(g.ep.residual) + (size_t)row * g.N + n0 + c0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (n0 + c0 + 8 * q + 8 <= g.N) {
                const uint4 u = *reinterpret_cast<const uint4*>(res + 8 * q);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float2 f = bf2_to_f2(w[i]);
                  v[8 * q + 2 * i] += f.x;
                  v[8 * q + 2 * i + 1] += f.y;
                }
              }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (n0 + c0 + 8 * q + 8 <= g.N)
              *reinterpret_cast<uint4*>(dst + 8 * q) =
                  make_uint4(f2_to_bf2(v[8 * q], v[8 * q + 1]), f2_to_bf2(v[8 * q + 2], v[8 * q + 3]),
                             f2_to_bf2(v[8 * q + 4], v[8 * q + 5]), f2_to_bf2(v[8 * q + 6], v[8 * q + 7]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D map over a row-major [rows][cols] bf16 matrix with a box of box_rows x 64 columns.
bool make_map2d(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace tcgemm

bool gemm_tc_supported(int M, int N, int K, int dtype) {
  // 16-byte aligned rows for TMA (N, K multiples of 8) and whole 16-byte output groups
  return dtype == 1 && M >= 1 && N >= 8 && K >= 8 && N % 8 == 0 && K % 8 == 0 &&
         tcgemm::encode_fn() != nullptr;
}

cudaError_t launch_gemm_tc(const void* A, const void* W, void* C, int M, int N, int K, int* status,
                           cudaStream_t s, const GemmEpilogue* ep) {
  using namespace tcgemm;
  CUtensorMap ma, mw;
  if (!make_map2d(&ma, A, M, K, BM) || !make_map2d(&mw, W, K, N, BK)) return cudaErrorInvalidValue;
  GemmArgs g;
  g.C = static_cast<__nv_bfloat16*>(C);
  g.M = M;
  g.N = N;
  g.K = K;
  g.status = status;
  std::memset(&g.ep, 0, sizeof(g.ep));
  if (ep) g.ep = *ep;
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  gemm_tc_kernel<<<dim3((N + BN - 1) / BN, (M + BM - 1) / BM), THREADS, SMEM, s>>>(ma, mw, g);
  return cudaGetLastError();
}

}  // namespace attn
