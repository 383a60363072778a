// Tensor-core GEMM for the block projections (sm_100a): C[M,N] = A[M,K] @ W[K,N], bf16 in,
// fp32 accumulation in TMEM, bf16 out. The block applies its weights as x @ W with W
// stored [in, out] ("Write attention from scratch", worked example: x @ Wq ... ctx @ Wo),
// so W is consumed as stored: as the B operand it is MN-major (N contiguous), which the
// UMMA shared-memory descriptor expresses directly; nothing is transposed.
//
// The kernel is persistent. In its pair form (M > 128) a cluster of two CTAs on two SMs
// computes 256 x 256 tiles of C in turn with cta_group::2 MMAs (M=256, N=256, K=16): CTA r
// stages rows 128 r .. 128 r + 127 of A (one 128 x 64 box per 64-deep K stage) and columns
// 128 r .. 128 r + 127 of W (two 64 x 64 boxes), six stages deep, and CTA 0's thread issues the
// MMAs, which read each SM's half of W once for both halves of the rows. On one SM the same
// 128 x 256 tile would need all four W boxes in its own shared memory per stage: the MMA reads
// of A and W plus the TMA writes (96 KB per stage) exceed what shared memory delivers at the
// tensor rate, so one-SM tiles stall on it. The one-SM form (M <= 128) keeps four stages of A
// and four W boxes. When the last round of pair tiles would keep at most half of the pairs
// busy, its tiles are cut into two 128-column halves (M=256, N=128 MMAs) so that it takes about
// half as long. In both forms, warp 4 issues the TMA loads (the pair's both count on CTA 0's
// barrier), warp 5 allocates TMEM and issues the MMAs into one of two 256-column accumulators,
// and warps 0-3 read the other accumulator back (one TMEM lane = one row of C per thread) and
// store bf16: a tile's epilogue overlaps the next tile's MMAs. Rows and columns past M, N are
// zero-filled on load or not loaded, and not stored.
//
// The weights may come as up to three matrices side by side (the block's x @ Wq, x @ Wk, x @ Wv
// in one launch: a CTA's columns fall in one of them, whose tensor map and output it uses).
//
// Epilogues (GemmEpilogue): a store, optionally with each row scaled (the fused block's
// 1/RMS), one segment's heads turned pairwise by the (cos, sin) table of the row's position
// (the keys: a 32-column chunk lies in one head, since hd is 64 or 128 and tiles and half-width
// items start at multiples of 128), and segments copied into a KV cache; or C = A W plus a
// residual.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>

#include "kernels.h"
#include "tc_common.cuh"

namespace attn {
namespace tcgemm {
namespace {

using namespace attn::tc;

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int THREADS = 192;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB: a CTA's 128 rows of A for one K stage
constexpr uint64_t WAIT_LIMIT_NS = 4000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 100000000ull;

// PAIR: a (2,1,1) cluster computes 256 x 256 tiles with cta_group::2 MMAs (M = 256): CTA r
// stages rows 128 r .. of A and W columns 128 r .. of the tile, so each SM's shared memory
// feeds half of B per MMA instead of all of it (for a 128 x 256 tile on one SM the MMA reads
// 48 KB and TMA writes 48 KB per 64-deep K stage, more than the SM's shared-memory bandwidth
// sustains at the tensor rate). Otherwise one CTA computes 128 x 256 tiles alone.
template <bool PAIR>
struct GCfg {
  static constexpr int ROWS = PAIR ? 2 * BM : BM;    // tile rows (M of the MMA)
  static constexpr int B_COLS = PAIR ? BN / 2 : BN;  // W columns a CTA stages
  static constexpr int B_BYTES = BK * B_COLS * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int NS = PAIR ? 6 : 4;
  static constexpr int OFF_BAR = NS * STAGE;
  static constexpr int SMEM = OFF_BAR + (2 * NS + 5) * 8 + 16 + 1024;
  static constexpr uint32_t IDESC = idesc_bf16_f32(ROWS, BN, 0, 1);
  static constexpr uint32_t IDESC_HALF = idesc_bf16_f32(ROWS, BN / 2, 0, 1);  // a 128-column item
};
static_assert(GCfg<true>::SMEM <= 227 * 1024 && GCfg<false>::SMEM <= 227 * 1024, "shared memory");

// Up to three weight matrices side by side (x @ [W0 | W1 | W2] with separate outputs): segment
// i covers columns [seg_end[i-1], seg_end[i]) of the launch; every boundary but the last is a
// multiple of 64, so each 64-column W box and each 32-column output chunk lies in one segment.
struct GemmArgs {
  __nv_bfloat16* C[3];
  int seg_end[3];
  int nseg;
  int M, N, K;  // N: all segments' columns
  int* status;
  GemmEpilogue ep;
};

// The work of a launch: tiles in rounds over the CTAs (pairs). In the pair form, when the last
// round would keep at most half of the pairs busy, its tiles are cut into two 128-column halves
// (items), so that it ends in about half the time. Item idx: rows m0.., columns gn0.., width w.
struct Item {
  int m0, gn0, w;
};
__device__ __forceinline__ Item item_of(int idx, int F, int ntn, int rows) {
  const int tile = idx < F ? idx : F + (idx - F) / 2;
  const int half = idx < F ? 0 : ((idx - F) & 1) + 1;  // 0: whole tile, 1 or 2: its halves
  Item it;
  it.m0 = (tile / ntn) * rows;
  it.gn0 = (tile % ntn) * BN + (half == 2 ? BN / 2 : 0);
  it.w = half ? BN / 2 : BN;
  return it;
}

__device__ __forceinline__ void store32(__nv_bfloat16* dst, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(dst + 8 * q) =
        make_uint4(f2_to_bf2(v[8 * q], v[8 * q + 1]), f2_to_bf2(v[8 * q + 2], v[8 * q + 3]),
                   f2_to_bf2(v[8 * q + 4], v[8 * q + 5]), f2_to_bf2(v[8 * q + 6], v[8 * q + 7]));
}

template <bool PAIR>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW0,
                   const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                   const __grid_constant__ GemmArgs g) {
  using C = GCfg<PAIR>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // (PAIR: rank 0's count both CTAs' bytes)
  uint64_t* empty = full + NS;
  uint64_t* acc_full = full + 2 * NS;   // [accumulator]: a tile's MMAs completed
  uint64_t* acc_empty = acc_full + 2;   // [accumulator]: the epilogue read it (PAIR: rank 0's, both CTAs)
  uint64_t* drain = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  // persistent: this CTA (or pair) computes tiles cid, cid + ncta, ... in the order (row tile,
  // column tile) with the column tile fastest
  const int cid = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int ncta = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int ntn = (g.N + BN - 1) / BN, ntiles = ntn * ((g.M + C::ROWS - 1) / C::ROWS);
  const int rem = ntiles % ncta;
  const bool split = PAIR && rem > 0 && 2 * rem <= ncta;
  const int F = split ? ntiles - rem : ntiles;   // whole tiles
  const int nitems = split ? F + 2 * rem : ntiles;
  const int nk = (g.K + BK - 1) / BK;
  // the segment of a column of the launch
  auto seg_of = [&](int col) {
    return (g.nseg > 1 && col >= g.seg_end[0]) ? ((g.nseg > 2 && col >= g.seg_end[1]) ? 2 : 1) : 0;
  };

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, PAIR ? 8 : 4);  // one arrival per epilogue warp (of both CTAs)
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    // two 128 x 256 fp32 accumulators (PAIR: in each CTA, for its 128 rows of the tile)
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (PAIR)
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch(&tmA);
      tma_prefetch(&tmW0);
      if (g.nseg > 1) tma_prefetch(&tmW1);
      if (g.nseg > 2) tma_prefetch(&tmW2);
      int u = 0;  // ring uses so far
      for (int idx = cid; idx < nitems && !*abort_flag; idx += ncta) {
        const Item itm = item_of(idx, F, ntn, C::ROWS);
        const int gn0 = itm.gn0, m0 = itm.m0;
        // this CTA's rows of A and columns of W (half of the item's in the pair form); boxes
        // that start past M or N are not loaded (those rows and columns of C are not stored)
        const int cw = PAIR ? itm.w / 2 : itm.w;
        const int am0 = m0 + (int)rank * BM, bn0 = gn0 + (int)rank * cw;
        const bool a_in = am0 < g.M;
        const int nbv = max(0, min(cw / 64, (g.N - bn0 + 63) / 64));
        // the bytes the stage's barrier counts: this CTA's, or (PAIR, on rank 0) both CTAs'
        uint32_t bytes = (a_in ? A_BYTES : 0) + nbv * (BK * 128);
        if (PAIR) {
          const int pbv = max(0, min(cw / 64, (g.N - (gn0 + cw) + 63) / 64));
          bytes += (m0 + BM < g.M ? A_BYTES : 0) + pbv * (BK * 128);  // (used on rank 0 only)
        }
        // the item's W map, chosen once when this CTA's columns lie in one segment (choosing it
        // per box costs ~10% of the GEMM); per box only for columns across a narrow segment
        const int sgt = seg_of(bn0 < g.N ? bn0 : g.N - 1);
        const bool one_seg = sgt == seg_of(min(bn0 + cw, g.N) - 1);
        const CUtensorMap* tmWt = sgt == 0 ? &tmW0 : (sgt == 1 ? &tmW1 : &tmW2);
        const int lc0 = bn0 - (sgt == 0 ? 0 : g.seg_end[sgt - 1]);
        for (int kb = 0; kb < nk; ++kb, ++u) {
          const int st = u % NS, n = u / NS;
          if (!mbar_wait(empty + st, (n & 1) ^ 1, abort_flag, g.status, WAIT_LIMIT_NS)) break;
          uint8_t* sa = smem + st * C::STAGE;
          if (!PAIR || rank == 0) mbar_expect_tx(full + st, bytes);
          const uint32_t fb = PAIR ? cluster_addr(full + st, 0) : 0u;
          auto load = [&](void* dst, const CUtensorMap* m, int c0, int c1) {
            if (PAIR)
              tma_load_2d_pair(dst, m, fb, c0, c1);
            else
              tma_load_2d(dst, m, full + st, c0, c1);
          };
          if (a_in) load(sa, &tmA, kb * BK, am0);
          if (one_seg) {
            for (int nb = 0; nb < nbv; ++nb) load(sa + A_BYTES + nb * (BK * 128), tmWt, lc0 + nb * 64, kb * BK);
          } else {
            for (int nb = 0; nb < nbv; ++nb) {
              const int col = bn0 + nb * 64, sg = seg_of(col);
              load(sa + A_BYTES + nb * (BK * 128), sg == 0 ? &tmW0 : (sg == 1 ? &tmW1 : &tmW2),
                   col - (sg == 0 ? 0 : g.seg_end[sg - 1]), kb * BK);
            }
          }
        }
      }
      // the copies issued last land before the CTA exits (PAIR: rank 0's barriers count the
      // peer's copies too, and the peer stays until rank 0 passes the final cluster barrier)
      if (!PAIR || rank == 0)
        for (int w = (u > NS ? u - NS : 0); w < u; ++w) mbar_wait_drain(full + w % NS, (w / NS) & 1, DRAIN_LIMIT_NS);
    }
  } else if (warp == 5) {
    if (lane == 0 && (!PAIR || rank == 0)) {
      const uint64_t dA = smem_desc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t dW = smem_desc_sw128(smem_u32(smem + A_BYTES), BK * 128, 1024);
      int u = 0, i = 0;  // ring uses and tiles so far
      for (int idx = cid; idx < nitems; idx += ncta, ++i) {
        const uint32_t idesc = item_of(idx, F, ntn, C::ROWS).w == BN ? C::IDESC : C::IDESC_HALF;
        // accumulator i % 2, free once the epilogue (of both CTAs) has read the item two before
        const int ab = i & 1;
        if (!mbar_wait(acc_empty + ab, ((i >> 1) & 1) ^ 1, abort_flag, g.status, WAIT_LIMIT_NS)) break;
        tc_fence_after();
        const uint32_t acc = tmem + ab * BN;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++u) {
          const int st = u % NS, n = u / NS;
          if (!mbar_wait(full + st, n & 1, abort_flag, g.status, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t so = (uint64_t)((st * C::STAGE) >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t a = dA + so + (uint64_t)((kk * 32) >> 4), b = dW + so + (uint64_t)((kk * 16 * 128) >> 4);
            const uint32_t acc_in = (kb > 0 || kk > 0) ? 1u : 0u;
            if (PAIR)
              umma_ss_pair(acc, a, b, idesc, acc_in);
            else
              umma_ss(acc, a, b, idesc, acc_in);
          }
          if (PAIR)
            umma_commit_pair(empty + st, 0x3);  // the stage is free in both CTAs
          else
            umma_commit(empty + st);
        }
        if (!ok) break;
        if (PAIR)
          umma_commit_pair(acc_full + ab, 0x3);
        else
          umma_commit(acc_full + ab);
      }
      if (PAIR)
        umma_commit_pair(drain, 0x1);
      else
        umma_commit(drain);
      mbar_wait_drain(drain, 0, DRAIN_LIMIT_NS);  // every MMA completes before TMEM is freed
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = rows m0 (+ 128 rank) + 32*w .. of C,
    // tile after tile, while the MMAs of the next tile fill the other accumulator
    const uint32_t ae = PAIR ? cluster_addr(acc_empty, 0) : 0u;
    int it = 0;
    for (int idx = cid; idx < nitems; idx += ncta, ++it) {
      const Item itm = item_of(idx, F, ntn, C::ROWS);
      const int gn0 = itm.gn0, m0 = itm.m0 + (int)rank * BM;
      const int ab = it & 1;
      if (!mbar_wait(acc_full + ab, (it >> 1) & 1, abort_flag, g.status, WAIT_LIMIT_NS)) break;
      tc_fence_after();
      const int row = m0 + warp * 32 + lane;
      const uint32_t t = tmem + ab * BN + ((uint32_t)(warp * 32) << 16);
      const float rs = (g.ep.mode == 0 && g.ep.row_scale && row < g.M) ? g.ep.row_scale[row] : 1.f;
#pragma unroll 1
      for (int c0 = 0; c0 < itm.w; c0 += 32) {
        float v[32];
        tmem_ld32(t + c0, v);
        tmem_wait_ld();
        // this chunk's segment, its output and width, and the tile's first column in it
        const int seg = seg_of(gn0 + c0);
        const int seg0 = seg == 0 ? 0 : g.seg_end[seg - 1];
        const int Ns = g.seg_end[seg] - seg0, n0 = gn0 - seg0;
        __nv_bfloat16* const Cs = g.C[seg];
        if (row < g.M && g.ep.mode == 0) {
          const GemmEpilogue& e = g.ep;
          const int n = n0 + c0;
          if (n < Ns) {
            if (e.row_scale) {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= rs;
            }
            const int bb = e.T > 0 ? row / e.T : 0, tt = row - bb * e.T;  // sequence and position
            if (seg == e.rot_seg && e.rope_cs) {
              // turn each pair (2c, 2c+1) of the head by the angle of this row's position
              const int d = n % e.hd;
              const float2* cs = e.rope_cs + (size_t)tt * (e.hd / 2) + d / 2;
#pragma unroll
              for (int pp = 0; pp < 16; ++pp) {
                const float2 c = cs[pp];
                const float x = v[2 * pp], y = v[2 * pp + 1];
                v[2 * pp] = x * c.x - y * c.y;
                v[2 * pp + 1] = x * c.y + y * c.x;
              }
            }
            if (n + 32 <= Ns) {
              store32(Cs + (size_t)row * Ns + n, v);
              if (e.cache[seg])
                store32(static_cast<__nv_bfloat16*>(e.cache[seg]) + ((size_t)bb * e.Lmax + e.pos0 + tt) * Ns + n, v);
            } else {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if (n + 8 * q + 8 <= Ns)
                  *reinterpret_cast<uint4*>(Cs + (size_t)row * Ns + n + 8 * q) =
                      make_uint4(f2_to_bf2(v[8 * q], v[8 * q + 1]), f2_to_bf2(v[8 * q + 2], v[8 * q + 3]),
                                 f2_to_bf2(v[8 * q + 4], v[8 * q + 5]), f2_to_bf2(v[8 * q + 6], v[8 * q + 7]));
            }
          }
        } else if (row < g.M) {
          __nv_bfloat16* dst = Cs + (size_t)row * Ns + n0 + c0;
          {
            const __nv_bfloat16* res = static_cast<const __nv_bfloat16*>(g.ep.residual) + (size_t)row * Ns + n0 + c0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (n0 + c0 + 8 * q + 8 <= Ns) {
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
            if (n0 + c0 + 8 * q + 8 <= Ns)
              *reinterpret_cast<uint4*>(dst + 8 * q) =
                  make_uint4(f2_to_bf2(v[8 * q], v[8 * q + 1]), f2_to_bf2(v[8 * q + 2], v[8 * q + 3]),
                             f2_to_bf2(v[8 * q + 4], v[8 * q + 5]), f2_to_bf2(v[8 * q + 6], v[8 * q + 7]));
        }
      }
      // every TMEM load of this accumulator completed (each chunk waited for its own)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR)
          mbar_arrive_remote(ae + ab * 8);
        else
          mbar_arrive(acc_empty + ab);
      }
    }
  }
  tc_fence_before();
  if (PAIR)
    cluster_sync();  // rank 0's MMAs (which read the peer's shared memory) and both epilogues are done
  else
    __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
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

// 2-D map over a row-major [rows][cols] bf16 matrix (rows ld elements apart; 0: cols) with a
// box of box_rows x 64 columns.
bool make_map2d(CUtensorMap* map, const void* base, int rows, int cols, int box_rows, int ld = 0) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld > 0 ? ld : cols) * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of two CTAs of the pair kernel the device holds at once (its shared memory admits
// one CTA per SM), found once per device: 0 when it holds none, -1 on a CUDA error.
int max_pair_clusters(int dev) {
  static int cached[64];
  static bool known[64];
  if (dev >= 0 && dev < 64 && known[dev]) return cached[dev];
  if (cudaFuncSetAttribute(gemm_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, GCfg<true>::SMEM) !=
      cudaSuccess)
    return -1;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = GCfg<true>::SMEM;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<true>, &cfg) != cudaSuccess) {
    cudaGetLastError();  // not an error of the caller's work: fall back to one SM per tile
    n = 0;
  }
  if (dev >= 0 && dev < 64) {
    cached[dev] = n;
    known[dev] = true;
  }
  return n;
}

}  // namespace
}  // namespace tcgemm

bool gemm_tc_supported(int M, int N, int K, int dtype) {
  // 16-byte aligned rows for TMA (N, K multiples of 8) and whole 16-byte output groups
  return dtype == 1 && M >= 1 && N >= 8 && K >= 8 && N % 8 == 0 && K % 8 == 0 &&
         tcgemm::encode_fn() != nullptr;
}

bool gemm_tc_segments_fit(int nseg, const int* Ns) {
  for (int i = 0; i + 1 < nseg; ++i)
    if (Ns[i] % 64) return false;
  return true;
}

cudaError_t launch_gemm_tc_multi(const void* A, int nseg, const void* const* Ws, void* const* Cs, const int* Ns,
                                 int M, int K, int* status, cudaStream_t s, const GemmEpilogue* ep, int ldw) {
  using namespace tcgemm;
  if (nseg < 1 || nseg > 3 || !gemm_tc_segments_fit(nseg, Ns)) return cudaErrorInvalidValue;
  CUtensorMap ma, mw[3];
  if (!make_map2d(&ma, A, M, K, BM)) return cudaErrorInvalidValue;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  int end = 0;
  for (int i = 0; i < 3; ++i) {
    const int j = i < nseg ? i : nseg - 1;  // unused maps repeat the last segment's
    if (!make_map2d(&mw[i], Ws[j], K, Ns[j], BK, ldw)) return cudaErrorInvalidValue;
    if (i < nseg) {
      end += Ns[i];
      g.seg_end[i] = end;
      g.C[i] = static_cast<__nv_bfloat16*>(Cs[i]);
    }
  }
  g.nseg = nseg;
  g.M = M;
  g.N = end;
  g.K = K;
  g.status = status;
  if (ep) {
    g.ep = *ep;
  } else {
    g.ep.rot_seg = -1;
  }
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long ntn = (end + BN - 1) / BN;
  // CTA pairs when the tiles have two row halves and the device co-schedules such clusters;
  // ATTN_TEST_GEMM_SINGLE=1 (a test hook) keeps the one-SM form
  int pairs = 0;
  if (M > BM && !(std::getenv("ATTN_TEST_GEMM_SINGLE") && std::atoi(std::getenv("ATTN_TEST_GEMM_SINGLE")) == 1)) {
    pairs = max_pair_clusters(dev);
    if (pairs < 0) return cudaErrorUnknown;
  }
  if (pairs > 0) {
    const long long tiles = ntn * ((M + 2 * BM - 1) / (2 * BM));
    if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    int ncl = tiles < pairs ? (int)tiles : pairs;
    // Test hook: ATTN_TEST_GEMM_CLUSTERS (1..the device's count) fixes the number of pairs, so
    // that small problems also run several rounds and a last round cut into half-width items.
    if (const char* env = std::getenv("ATTN_TEST_GEMM_CLUSTERS")) {
      const int nc = std::atoi(env);
      if (nc >= 1 && nc <= pairs) ncl = (int)std::min<long long>(nc, tiles);
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * ncl);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = GCfg<true>::SMEM;
    cfg.stream = s;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<true>, ma, mw[0], mw[1], mw[2], g)) != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if ((e = cudaFuncSetAttribute(gemm_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GCfg<false>::SMEM)) != cudaSuccess)
    return e;
  // persistent: one CTA per SM (its shared memory admits one) over the tiles
  const long long tiles = ntn * ((M + BM - 1) / BM);
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int grid = tiles < sms ? (int)tiles : sms;
  gemm_tc_kernel<false><<<grid, THREADS, GCfg<false>::SMEM, s>>>(ma, mw[0], mw[1], mw[2], g);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const void* A, const void* W, void* C, int M, int N, int K, int* status,
                           cudaStream_t s, const GemmEpilogue* ep) {
  return launch_gemm_tc_multi(A, 1, &W, &C, &N, M, K, status, s, ep);
}

}  // namespace attn
