// Split-KV decode on the tensor cores (sm_100a): one new query per sequence attends to
// its KV cache ("Building a Transformer from Scratch: Attention, Architecture, and
// Memory", Part 3 "KV caching"); the splits are merged with the log-sum-exp rule of that
// page's FlashAttention equations by the merge kernel in decode.cu.
//
// One CTA = one (split of the cache rows, key/value head, sequence); splits are 2048 keys
// (fewer CTAs amortise the set-up; see decode_chunk). The H/KV query heads served by the
// key/value head sit in every 32-row quarter of a 128-row MMA tile (row 32k + i holds head i
// for i < H/KV, other rows are zero), so the scores S = Q K^T of a 128-key tile land in
// tensor memory once per TMEM lane quarter. Warp k, which addresses lane quarter k, does the
// softmax of keys 32k..32k+31 for every head (one head per lane): the four warps sit on the
// four SM sub-partitions and share a tile's exponentials, where one warp alone would work
// through all 128 keys. They agree on each head's running maximum through shared memory and
// write P (bf16) for their quarter of the keys, zeros for the rest, over the S columns of
// their lanes; the TS-form PV MMA then accumulates in quarter k the part of O that keys of
// quarter k contribute. The four parts share one reference maximum and are added when the
// split's partial state is written. The replicated and padded rows cost tensor-core time
// that decode does not miss: the kernel is bound by streaming K and V from HBM, which TMA
// does through a two-stage ring (two CTAs per SM keep four 32 KB tiles in flight per SM).
//
// Warps: 0-3 = softmax (quarter = warp), 4 = TMA producer, 5 = TMEM allocation and MMA
// issue; all six set up the query tile.
// The cached keys are already rotated at their slot positions; only q is rotated here,
// at qpos[b]. Keys at or beyond seqlens[b] and, with a window, keys j with
// qpos - j >= window get weight exactly 0.
#include <cudaTypedefs.h>

#include <cstdlib>

#include "kernels.h"
#include "tc_common.cuh"

namespace attn {
namespace tcdec {
namespace {

using namespace attn::tc;

constexpr int BN = 128;               // keys per tile
constexpr int BM = 128;               // MMA rows (query heads, zero padded)
constexpr int NS = 2;                 // ring stages (K, V alternate)
constexpr int THREADS = 192;          // 4 softmax warps, the TMA warp, the MMA warp
constexpr int TMA_WARP = 4, MMA_WARP = 5;
constexpr uint64_t WAIT_LIMIT_NS = 4000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 100000000ull;  // own copies/MMAs finish in microseconds
constexpr float LOG2E = 1.4426950408889634f;

template <int HD>
struct Cfg {
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int KV_BYTES = BN * HD * 2;
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
  // kv_full[NS], kv_empty[NS], s_full, p_full, o_done, never, drain, red_bar[2], fin_bar
  static constexpr int NBAR = 2 * NS + 8;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // the softmax warps' exchange: running maxima red[2][4][32], row-sum parts lpart[4][32]
  static constexpr int OFF_RED = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int RED_BYTES = (2 * 4 * 32 + 4 * 32) * 4;
  static constexpr int OFF_TAB = OFF_RED + RED_BYTES;
  static constexpr int SMEM = OFF_TAB + 1024;  // (two CTAs per SM stay within 200 KB)
  // paged cache only: the page index of every block of a split (a split holds at most
  // 2048 / page_size <= 256 pages), reserved only when a paged decode is launched
  static constexpr int MAX_TAB = 256;
  static constexpr int SMEM_PAGED = OFF_TAB + MAX_TAB * 4 + 1024;
  // the four O parts [4][HD][32] fp32 are added through the K/V ring once it is idle
  static_assert(4 * HD * 32 * 4 <= NS * KV_BYTES, "O parts do not fit the ring");
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, 0, 1);
};

struct DecArgs {
  DecodeParams p;
  int chunk;   // keys per split (multiple of 128)
  int nsplit;
  float scale_log2;
  void* ws;
  unsigned long long wait_ns;  // bound of every wait (4 s unless a test lowers it)
  int test_stall;              // test hook: the MMA warp waits on a barrier nothing signals
  int kv_same;                 // keys and values are one cache (latent attention): each tile is
                               // fetched once and serves as K in QK and as V in PV
};

template <int HD>
__global__ void __launch_bounds__(THREADS, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ DecArgs a) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::OFF_KV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + NS;
  uint64_t* s_full = bars + 2 * NS;
  uint64_t* p_full = s_full + 1;
  uint64_t* o_done = s_full + 2;
  uint64_t* never = s_full + 3;    // not signalled by anything (test hook)
  uint64_t* drain = s_full + 4;    // the MMA thread's final commit
  uint64_t* red_bar = s_full + 5;  // [2]: the four softmax warps posted a tile's maxima
  uint64_t* fin_bar = s_full + 7;  // the four O parts are in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][32]
  float* lpart = red + 2 * 4 * 32;                           // [4][32]

  const DecodeParams& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kvh = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
  const int G = p.H / p.KV;

  int L = p.seqlens[b];
  const int qp = p.qpos[b];
  if (L < 0 || L > p.Lmax || qp < 0 || qp >= (1 << 24)) {
    if (split == 0 && kvh == 0 && tid == 0) flag_error(p.status, DEV_BAD_ARG);
    L = 0;
  }
  int j0 = split * a.chunk;
  const int j1 = min(L, j0 + a.chunk);         // keys [j0, j1) of this split
  if (p.window > 0) j0 = max(j0, qp - p.window + 1);
  const int jt0 = j0 / BN, jt1 = (j1 - 1) / BN;  // tiles (empty when j0 >= j1)
  const bool empty = j0 >= j1;

  // partial-state layout: O [B][H][nsplit][hd], m [B][H][nsplit], l [B][H][nsplit]
  float* wsO = static_cast<float*>(a.ws);
  float* wsM = wsO + (size_t)p.B * p.H * a.nsplit * HD;
  float* wsL = wsM + (size_t)p.B * p.H * a.nsplit;

  if (empty) {
    for (int h = tid; h < G; h += THREADS) {
      const size_t pi = ((size_t)b * p.H + kvh * G + h) * a.nsplit + split;
      wsM[pi] = -INFINITY;
      wsL[pi] = 0.f;
    }
    return;
  }

  // ---- query tile: head i (turned at qpos) in rows i, 32 + i, 64 + i and 96 + i for i < G,
  // other rows zero. Work items are (head slot, 16-byte chunk) pairs spread over all threads.
  {
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q);
    for (int it = tid; it < 32 * (HD / 8); it += THREADS) {
      const int row = it / (HD / 8), c = it % (HD / 8);
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (row < G) {
        const uint4 u = *reinterpret_cast<const uint4*>(q + ((size_t)b * p.H + kvh * G + row) * HD + c * 8);
        const uint32_t in[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = bf2_to_f2(in[e]);
          if (p.rope.on) {
            float cs, sn;
            rope_cos_sin(qp, p.rope.hi[c * 4 + e], p.rope.lo[c * 4 + e], cs, sn);
            rotate_pair(f.x, f.y, cs, sn);
          }
          w[e] = f2_to_bf2(f.x, f.y);
        }
      }
      const uint4 v = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
      for (int k = 0; k < 4; ++k) sts128(smem_u32(sQ) + sw128_offset(32 * k + row, c * 8, BM), v);
    }
    fence_proxy_async();
  }
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(never, 1);
    mbar_init(drain, 1);
    mbar_init(red_bar, 128);
    mbar_init(red_bar + 1, 128);
    mbar_init(fin_bar, 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // S: columns 0..127 (P over 0..63), O: 128..128+HD-1

  if (warp == TMA_WARP) {
    // ------------------------------------------------------------ TMA producer
    int* tab = reinterpret_cast<int*>(smem + C::OFF_TAB);
    if (p.block_table) {
      // the split's page indices, fetched by the whole warp at once; a page past the
      // sequence (or an invalid table entry) becomes an out-of-range index, which reads zeros
      const int ppt = BN / p.page_size;
      const int n = min((jt1 - jt0 + 1) * ppt, C::MAX_TAB);
      for (int idx = lane; idx < n; idx += 32) {
        const int blk = jt0 * ppt + idx;
        int page = p.num_pages;
        if (blk * p.page_size < L) {
          const int e = p.block_table[(size_t)b * p.max_blocks + blk];
          if (e >= 0 && e < p.num_pages)
            page = e;
          else
            flag_error(p.status, DEV_BAD_ARG);
        }
        tab[idx] = page;
      }
      __syncwarp();
    }
    if (lane == 0) {
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      const int per = a.kv_same ? 1 : 2;      // ring uses per tile: K then V, or one for both
      const int total = per * (jt1 - jt0 + 1);
      int u = 0;
      for (; u < total; ++u) {
        const int st = u % NS, n = u / NS, j = jt0 + u / per;
        const bool isv = per == 2 && (u & 1);
        if (!mbar_wait(kv_empty + st, (n & 1) ^ 1, abort_flag, p.status, a.wait_ns)) break;
        mbar_expect_tx(kv_full + st, C::KV_BYTES);
        if (!p.block_table) {
          for (int kb = 0; kb < HD / 64; ++kb)
            tma_load_4d(sKV + st * C::KV_BYTES + kb * BN * 128, isv ? &tmV : &tmK, kv_full + st,
                        kb * 64, kvh, j * BN, b);
        } else {
          // one box per page of the tile
          const int ppt = BN / p.page_size;
          for (int i = 0; i < ppt; ++i) {
            const int ti = (j - jt0) * ppt + i;
            const int page = ti < C::MAX_TAB ? tab[ti] : p.num_pages;
            for (int kb = 0; kb < HD / 64; ++kb)
              tma_load_4d(sKV + st * C::KV_BYTES + kb * BN * 128 + i * p.page_size * 128, isv ? &tmV : &tmK,
                          kv_full + st, kb * 64, kvh, 0, page);
          }
        }
      }
      // The loads of the last NS uses land before the CTA exits (immediate when the MMA
      // warp consumed them; after an abort they may still be in flight).
      for (int w = (u > NS ? u - NS : 0); w < u; ++w)
        mbar_wait_drain(kv_full + w % NS, (w / NS) & 1, DRAIN_LIMIT_NS);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint64_t dQ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sKV), BN * 128, 1024);
      int u = 0, c = 0;
      if (a.test_stall && !mbar_wait(never, 0, abort_flag, p.status, a.wait_ns)) goto mma_drain;
      for (int j = jt0; j <= jt1; ++j, ++c) {
        // keys at ring use u; values at u + 1, or (one cache) the same use
        const int stK = u % NS, uV = a.kv_same ? u : u + 1, stV = uV % NS;
        if (!mbar_wait(kv_full + stK, (u / NS) & 1, abort_flag, p.status, a.wait_ns)) goto mma_drain;
        tc_fence_after();
        const uint64_t bk = dK + (uint64_t)((stK * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * (BN * 128) + (kk & 3) * 32) >> 4;
          umma_ss(tmem, dQ + off, bk + off, C::IDESC_QK, kk > 0);
        }
        umma_commit(s_full);
        if (!a.kv_same) umma_commit(kv_empty + stK);
        if (!mbar_wait(kv_full + stV, (uV / NS) & 1, abort_flag, p.status, a.wait_ns)) goto mma_drain;
        if (!mbar_wait(p_full, c & 1, abort_flag, p.status, a.wait_ns)) goto mma_drain;
        tc_fence_after();
        const uint64_t bv = dV + (uint64_t)((stV * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts(tmem + 128, tmem + kk * 8, bv + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV,
                  (kk > 0 || c > 0) ? 1u : 0u);
        umma_commit(o_done);
        umma_commit(kv_empty + stV);
        u = uV + 1;
      }
    mma_drain:
      // every MMA issued above completes before tensor memory is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // ------------------------------------------------ softmax (warp = lane quarter, lane = head)
    const int k = warp;
    const uint32_t lq = (uint32_t)(32 * k) << 16;  // this warp's TMEM lanes
    const int h = kvh * G + lane;
    const bool real = lane < G;
    const float slope = (p.alibi.on && real) ? p.alibi.slope[h] * LOG2E : 0.f;
    const float sc = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    int c = 0;
    for (int j = jt0; j <= jt1; ++j, ++c) {
      if (!mbar_wait(s_full, c & 1, abort_flag, p.status, a.wait_ns)) goto done;
      tc_fence_after();
      const int key0 = j * BN + 32 * k;  // this warp's 32 keys of the tile
      const bool need_mask = key0 < j0 || key0 + 32 > j1;
      float x[32];
      tmem_ld32(tmem + lq + 32 * k, x);
      tmem_wait_ld();
      float hx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int key = key0 + i;
        float v = p.alibi.on ? fmaf(x[i], sc, -slope * fabsf((float)(qp - key))) : x[i] * sc;
        if (need_mask) v = (key >= j0 && key < j1) ? v : -INFINITY;
        x[i] = v;
        hx = fmaxf(hx, v);
      }
      // the head's maximum over the whole tile, from the four quarters
      float* rt = red + (c & 1) * 128;
      rt[k * 32 + lane] = hx;
      mbar_arrive(red_bar + (c & 1));
      if (!mbar_wait(red_bar + (c & 1), (c >> 1) & 1, abort_flag, p.status, a.wait_ns)) goto done;
      hx = fmaxf(fmaxf(rt[lane], rt[32 + lane]), fmaxf(rt[64 + lane], rt[96 + lane]));
      // same lazy reference as the prefill: move it only by more than 8 (log2 units)
      const float m_exp = (hx > m_ref + 8.f) ? hx : m_ref;
      const float mu = (m_exp == -INFINITY) ? 0.f : m_exp;
      uint32_t pk[16];
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const float e0 = ex2(x[2 * i] - mu), e1 = ex2(x[2 * i + 1] - mu);
        const float e2 = ex2(x[2 * i + 2] - mu), e3 = ex2(x[2 * i + 3] - mu);
        rs0 += e0 + e1;
        rs1 += e2 + e3;
        pk[i] = f2_to_bf2(e0, e1);
        pk[i + 1] = f2_to_bf2(e2, e3);
      }
      // P over the S columns of this warp's lanes: its keys' weights, zeros for the others
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = qq == k ? pk[i] : 0u;
        tmem_st16u(tmem + lq + 16 * qq, v);
      }
      const float alpha = (m_exp == m_ref) ? 1.f : ex2(m_ref - m_exp);
      m_ref = m_exp;
      // rescale this quarter's part of O (the previous PV finished before this tile's QK,
      // which this tile waited for)
      if (c > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int q4 = 0; q4 < HD / 32; ++q4) {
          float o[32];
          tmem_ld32(tmem + lq + 128 + q4 * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tmem + lq + 128 + q4 * 32, o);
        }
      }
      l = l * alpha + (rs0 + rs1);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // add the four parts of O and of the row sum, and write this split's partial state
    if (!mbar_wait(o_done, (c - 1) & 1, abort_flag, p.status, a.wait_ns)) goto done;
    tc_fence_after();
    {
      // every copy into the ring was consumed by an MMA that o_done covers: the ring is idle
      float* part = reinterpret_cast<float*>(sKV);  // [4][HD][32]
#pragma unroll 1
      for (int q4 = 0; q4 < HD / 32; ++q4) {
        float o[32];
        tmem_ld32(tmem + lq + 128 + q4 * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) part[(k * HD + q4 * 32 + e) * 32 + lane] = o[e];
      }
      lpart[k * 32 + lane] = l;
      mbar_arrive(fin_bar);
      if (!mbar_wait(fin_bar, 0, abort_flag, p.status, a.wait_ns)) goto done;
      if (real) {
        const size_t pi = ((size_t)b * p.H + h) * a.nsplit + split;
        constexpr int DQ = HD / 4;  // features of O this warp adds up and writes
        float4* dst = reinterpret_cast<float4*>(wsO + pi * HD + k * DQ);
#pragma unroll 1
        for (int v4 = 0; v4 < DQ / 4; ++v4) {
          float r[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int d = k * DQ + v4 * 4 + e;
            r[e] = part[d * 32 + lane] + part[(HD + d) * 32 + lane] + part[(2 * HD + d) * 32 + lane] +
                   part[(3 * HD + d) * 32 + lane];
          }
          dst[v4] = make_float4(r[0], r[1], r[2], r[3]);
        }
        if (k == 0) {
          // the merge kernel works in natural-log units
          wsM[pi] = m_ref == -INFINITY ? -INFINITY : m_ref * 0.6931471805599453f;
          wsL[pi] = lpart[lane] + lpart[32 + lane] + lpart[64 + lane] + lpart[96 + lane];
        }
      }
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
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

// 4-D map over the cache [B][Lmax][KV][hd] with a box of 128 slots x 64 features of one head.
bool make_cache_map(CUtensorMap* map, const void* base, int B, int Lmax, int KV, int hd) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)KV, (cuuint64_t)Lmax, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)hd * 2, (cuuint64_t)KV * hd * 2, (cuuint64_t)Lmax * KV * hd * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D map over a page pool [num_pages][page_size][KV][hd] with a box of one page x 64 features.
bool make_page_map(CUtensorMap* map, const void* base, int num_pages, int page_size, int KV, int hd) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)KV, (cuuint64_t)page_size, (cuuint64_t)num_pages};
  const cuuint64_t strides[3] = {(cuuint64_t)hd * 2, (cuuint64_t)KV * hd * 2,
                                 (cuuint64_t)page_size * KV * hd * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)page_size, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD>
cudaError_t launch_hd(const DecodeParams& p, int chunk, int nsplit, void* ws, cudaStream_t s) {
  CUtensorMap mk, mv;
  const bool ok = p.block_table
                      ? make_page_map(&mk, p.kcache, p.num_pages, p.page_size, p.KV, HD) &&
                            make_page_map(&mv, p.vcache, p.num_pages, p.page_size, p.KV, HD)
                      : make_cache_map(&mk, p.kcache, p.B, p.Lmax, p.KV, HD) &&
                            make_cache_map(&mv, p.vcache, p.B, p.Lmax, p.KV, HD);
  if (!ok) return cudaErrorInvalidValue;
  DecArgs a;
  a.p = p;
  a.chunk = chunk;
  a.nsplit = nsplit;
  a.scale_log2 = p.scale * LOG2E;
  a.ws = ws;
  // Test hook (failure detection without a GPU fault): with ATTN_TEST_DECODE_STALL_NS set
  // to a positive number of nanoseconds, every wait of this kernel is bounded by it and
  // the MMA warp first waits on a barrier that nothing signals, so each CTA gives up,
  // records ATTN_ERR_TIMEOUT in the device status word, drains its own copies and exits.
  a.wait_ns = WAIT_LIMIT_NS;
  a.test_stall = 0;
  a.kv_same = p.kcache == p.vcache;
  if (const char* e = std::getenv("ATTN_TEST_DECODE_STALL_NS")) {
    const long long ns = std::atoll(e);
    if (ns > 0) {
      a.wait_ns = (unsigned long long)ns;
      a.test_stall = 1;
    }
  }
  const int smem = p.block_table ? Cfg<HD>::SMEM_PAGED : Cfg<HD>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<HD>::SMEM_PAGED);
  if (e != cudaSuccess) return e;
  // split is the slowest grid dimension: the full leading splits of every sequence are
  // scheduled before the (shorter, often empty) trailing ones
  decode_tc_kernel<HD><<<dim3(p.KV, p.B, nsplit), THREADS, smem, s>>>(mk, mv, a);
  return cudaGetLastError();
}

}  // namespace
}  // namespace tcdec

bool decode_tc_supported(const DecodeParams& p, int dtype) {
  const int G = p.H / p.KV;
  return dtype == 1 && (p.hd == 64 || p.hd == 128) && G >= 1 && G <= 32 && tcdec::encode_fn() != nullptr;
}

cudaError_t launch_decode_tc(const DecodeParams& p, int chunk, int nsplit, void* ws, cudaStream_t s) {
  return p.hd == 128 ? tcdec::launch_hd<128>(p, chunk, nsplit, ws, s)
                     : tcdec::launch_hd<64>(p, chunk, nsplit, ws, s);
}

}  // namespace attn
