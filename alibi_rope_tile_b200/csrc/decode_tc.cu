// Decode on the tensor cores (sm_100a): one new query per sequence attends to its KV cache
// ("Building a Transformer from Scratch: Attention, Architecture, and Memory", Part 3 "KV
// caching"); partial results are combined with the log-sum-exp rule of that page's
// FlashAttention equations (merge.cuh).
//
// Work split (stream-K). A unit is one (sequence, key/value head); its keys are the 128-key
// tiles that hold slots [j0, seqlens) (j0 = qpos - window + 1 with a window, else 0). Every
// unit's tile count and their running sum come first (each CTA computes them for up to
// PLAN_MAX units; beyond that a plan kernel writes them once). The decode kernel runs two
// CTAs per SM and gives CTA i the tiles [i T / n, (i+1) T / n) of the concatenated units (T
// tiles in all, n = min(grid, T) working CTAs), so every CTA streams the same amount of cache
// whatever the mix of lengths. A CTA's range covers pieces of one or more units; each piece
// leaves a partial state in slot (unit + CTA index), which is unique because both numbers
// only grow along the concatenation. The merge kernel finds the CTAs that cover a unit from
// the same running sum and combines their partials.
//
// Inside a piece the H/KV query heads served by the key/value head sit in every 32-row
// quarter of a 128-row MMA tile (row 32k + i holds head i for i < H/KV, other rows are
// zero), so the scores S = Q K^T of a 128-key tile land in tensor memory once per TMEM lane
// quarter. Warp k, which addresses lane quarter k, does the softmax of keys 32k..32k+31 for
// every head (one head per lane): the four warps sit on the four SM sub-partitions and share
// a tile's exponentials. They agree on each head's running maximum through shared memory and
// write P (bf16) for their quarter of the keys, zeros for the rest, over the S columns of
// their lanes; the TS-form PV MMA then accumulates in quarter k the part of O that the keys
// of quarter k contribute. The four parts share one reference maximum and are added, through
// the query tile's shared memory, when a piece's partial state is written. The replicated
// and padded rows cost tensor-core time that decode does not miss: the kernel is bound by
// streaming K and V from HBM, which TMA does through a two-stage ring.
//
// Warps: 0-3 = softmax and query set-up (quarter = warp), 4 = TMA producer, 5 = TMEM
// allocation and MMA issue. The cached keys are already rotated at their slot positions;
// only q is rotated here, at qpos[b]. Keys at or beyond seqlens[b] and, with a window, keys
// j with qpos - j >= window get weight exactly 0.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>

#include "kernels.h"
#include "merge.cuh"
#include "tc_common.cuh"

namespace attn {
namespace tcdec {
namespace {

using namespace attn::tc;

constexpr int BN = 128;               // keys per tile
constexpr int BM = 128;               // MMA rows (query heads, replicated and zero padded)
constexpr int NS = 2;                 // ring stages (K, V alternate)
constexpr int THREADS = 192;          // 4 softmax warps, the TMA warp, the MMA warp
constexpr int TMA_WARP = 4, MMA_WARP = 5;
constexpr int CTAS_PER_SM = 2;
constexpr int PLAN_MAX = 1024;        // units up to which each CTA counts the tiles itself
constexpr uint64_t WAIT_LIMIT_NS = 4000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 100000000ull;  // own copies/MMAs finish in microseconds
constexpr float LOG2E = 1.4426950408889634f;

template <int HD>
struct Cfg {
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int KV_BYTES = BN * HD * 2;
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
  // kv_full[NS], kv_empty[NS], s_full, p_full, o_done, never, drain, red_bar[2], fin_bar, q_full
  static constexpr int NBAR = 2 * NS + 9;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // the softmax warps' exchange: running maxima red[2][4][32], row-sum parts lpart[4][32]
  static constexpr int OFF_RED = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int RED_BYTES = (2 * 4 * 32 + 4 * 32) * 4;
  // the running tile counts of up to PLAN_MAX units, when every CTA plans for itself (int)
  static constexpr int OFF_PREF = OFF_RED + RED_BYTES;
  static constexpr int SMEM = OFF_PREF + (PLAN_MAX + 1) * 4 + 1024;  // (two CTAs per SM: < 210 KB)
  // a piece's four O parts are added through the query tile's memory in rounds of RC columns:
  // [4 warps][RC][32 lanes] fp32
  static constexpr int RC = Q_BYTES / (4 * 32 * 4);
  static_assert(HD % RC == 0 && RC % 16 == 0, "O reduction rounds");
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, 0, 1);
};

struct DecArgs {
  DecodeParams p;
  float scale_log2;
  float* partO;              // [slots][G][hd]
  float* partM;              // [slots][G] (natural-log units)
  float* partL;              // [slots][G]
  long long* prefix;         // [U + 1]: tiles of the units before u; prefix[U] = all tiles
  int plan_in_cta;           // U <= PLAN_MAX: each CTA computes the counts (CTA 0 also writes
                             // prefix for the merge); otherwise the plan kernel wrote prefix
  int U;                     // units: B * KV
  int nctas;                 // grid size
  unsigned long long wait_ns;  // bound of every wait (4 s unless a test lowers it)
  int test_stall;              // test hook: the MMA warp waits on a barrier nothing signals
  int kv_same;                 // keys and values are one cache (latent attention): each tile is
                               // fetched once and serves as K in QK and as V in PV
};

// The key range of unit u = (sequence b, key/value head kvh).
struct Unit {
  int b, kvh, qp, j0, j1, jt0;
};
__device__ __forceinline__ bool bad_sequence(const DecodeParams& p, int L, int qp) {
  return L < 0 || L > p.Lmax || qp < 0 || qp >= (1 << 24);
}
__device__ __forceinline__ Unit unit_of(const DecodeParams& p, int u) {
  Unit x;
  x.b = u / p.KV;
  x.kvh = u - x.b * p.KV;
  int L = p.seqlens[x.b];
  x.qp = p.qpos[x.b];
  if (bad_sequence(p, L, x.qp)) L = 0;
  x.j0 = p.window > 0 ? max(0, x.qp - p.window + 1) : 0;
  x.j1 = L;
  x.jt0 = x.j0 / BN;
  return x;
}
__device__ __forceinline__ int unit_tiles(const Unit& x) { return x.j0 >= x.j1 ? 0 : (x.j1 - 1) / BN - x.jt0 + 1; }

// The CTA whose tile range holds global tile t (the last i with floor(i T / n) <= t), for
// n = min(grid, T) working CTAs: each of them then holds at least one tile.
__host__ __device__ __forceinline__ int cta_of(long long t, long long T, int grid) {
  const long long n = T < grid ? T : grid;
  return (int)(((t + 1) * n - 1) / T);
}

// One CTA: prefix[u] = tiles of units 0..u-1, prefix[U] = all tiles. A sequence whose length
// or position is out of range counts as empty and is recorded as DEV_BAD_ARG.
__global__ void __launch_bounds__(1024) decode_plan_kernel(const DecodeParams p, long long* prefix, int U) {
  __shared__ long long wsum[32];
  __shared__ long long carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < U; base += 1024) {
    const int u = base + tid;
    long long n = 0;
    if (u < U) {
      const Unit x = unit_of(p, u);
      n = unit_tiles(x);
      if (x.kvh == 0 && bad_sequence(p, p.seqlens[x.b], x.qp)) flag_error(p.status, DEV_BAD_ARG);
    }
    long long v = n;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
      long long w = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      wsum[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const long long before = carry + (warp > 0 ? wsum[warp - 1] : 0) + v - n;
    if (u < U) prefix[u] = before;
    __syncthreads();
    if (tid == 0) carry += wsum[31];
    __syncthreads();
  }
  if (tid == 0) prefix[U] = carry;
}

template <int HD>
__global__ void __launch_bounds__(THREADS, CTAS_PER_SM)
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
  uint64_t* fin_bar = s_full + 7;  // a round of the O-part reduction
  uint64_t* q_full = s_full + 8;   // a piece's query tile is in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* first_unit = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][32]
  float* lpart = red + 2 * 4 * 32;                           // [4][32]

  const DecodeParams& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.H / p.KV;
  launch_dependents();  // the merge may start its independent set-up
  int* spref = reinterpret_cast<int*>(smem + C::OFF_PREF);
  if (a.plan_in_cta) {
    // Tiles of every unit and their running sum, as the plan kernel computes them: thread tid
    // counts a run of up to PER consecutive units, one block scan adds the runs up.
    constexpr int PER = (PLAN_MAX + THREADS - 1) / THREADS;
    __shared__ int wsum[THREADS / 32];
    const int per = (a.U + THREADS - 1) / THREADS, u0 = tid * per;
    int n[PER], run = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      n[i] = 0;
      const int u = u0 + i;
      if (i < per && u < a.U) {
        const Unit x = unit_of(p, u);
        n[i] = unit_tiles(x);
        if (blockIdx.x == 0 && x.kvh == 0 && bad_sequence(p, p.seqlens[x.b], x.qp)) flag_error(p.status, DEV_BAD_ARG);
      }
      run += n[i];
    }
    int v = run;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    int before = v - run;
    for (int w = 0; w < warp; ++w) before += wsum[w];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (i < per && u0 + i < a.U) spref[u0 + i] = before;
      before += n[i];
    }
    if (tid == THREADS - 1) spref[a.U] = before;
    __syncthreads();
    if (blockIdx.x == 0)
      for (int u = tid; u <= a.U; u += THREADS) a.prefix[u] = spref[u];  // for the merge
  }
  auto pref = [&](int u) -> long long { return a.plan_in_cta ? (long long)spref[u] : a.prefix[u]; };
  // With fewer tiles than CTAs only the first T CTAs work, so that every working CTA has at
  // least one tile (the merge relies on it).
  const long long T = pref(a.U);
  const int nw = (int)(T < a.nctas ? T : a.nctas);
  if ((int)blockIdx.x >= nw) return;
  const long long t0 = T * blockIdx.x / nw, t1 = T * (blockIdx.x + 1) / nw;

  if (warp == 0) {
    // the unit holding tile t0: prefix[lo] <= t0 < prefix[hi], narrowed 32-fold per step
    int lo = 0, hi = a.U;
    while (hi - lo > 1) {
      const int step = (hi - lo + 31) / 32;
      const int idx = lo + lane * step;
      const unsigned le = __ballot_sync(0xffffffffu, idx < hi && pref(idx) <= t0);
      const int nlo = lo + (31 - __clz(le)) * step;  // lane 0 always qualifies
      hi = min(hi, nlo + step);
      lo = nlo;
    }
    if (lane == 0) *first_unit = lo;
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
    mbar_init(q_full, 128);
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
  const int u_first = *first_unit;

  // Every role walks the same pieces: unit u from tile t to pe (exclusive), which are the
  // unit's tiles jb .. jb + nt - 1.
#define FOR_EACH_PIECE(pc)                                                    \
  int u = u_first;                                                            \
  long long t = t0;                                                           \
  for (int pc = 0; t < t1; ++pc)
#define PIECE_BOUNDS                                                          \
  const long long ub = pref(u), ue = pref(u + 1);                             \
  const long long pe = ue < t1 ? ue : t1;                                     \
  const Unit x = unit_of(p, u);                                               \
  const int jb = x.jt0 + (int)(t - ub);                                       \
  const int nt = (int)(pe - t);
#define NEXT_PIECE                                                            \
  t = pe;                                                                     \
  ++u;                                                                        \
  while (t < t1 && pref(u + 1) <= t) ++u;

  if (warp == TMA_WARP) {
    // ------------------------------------------------------------ TMA producer (whole warp;
    // lane 0 issues, the lanes fetch a paged tile's block-table entries)
    if (lane == 0) {
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
    }
    const int per = a.kv_same ? 1 : 2;  // ring uses per tile: K then V, or one for both
    int use = 0;
    bool ok = true;
    // a paged tile's page indices, one per lane (the first BN / page_size lanes); fetched a
    // tile ahead so that the table read overlaps the waits for ring slots
    auto pages_of = [&](const Unit& x, int j) {
      int page = p.num_pages;  // out of range: the box reads zeros
      const int ppt = BN / p.page_size;
      const int blk = j * ppt + lane;
      if (lane < ppt && blk * p.page_size < x.j1) {
        const int e = p.block_table[(size_t)x.b * p.max_blocks + blk];
        if (e >= 0 && e < p.num_pages)
          page = e;
        else
          flag_error(p.status, DEV_BAD_ARG);
      }
      return page;
    };
    FOR_EACH_PIECE(pc) {
      PIECE_BOUNDS
      int page_next = p.block_table ? pages_of(x, jb) : 0;
      for (int k = 0; k < nt && ok; ++k) {
        const int j = jb + k;
        const int page = page_next;
        if (p.block_table && k + 1 < nt) page_next = pages_of(x, j + 1);
        for (int r = 0; r < per; ++r) {
          const int st = use % NS, n = use / NS;
          bool w = lane == 0 ? mbar_wait(kv_empty + st, (n & 1) ^ 1, abort_flag, p.status, a.wait_ns) : true;
          w = __shfl_sync(0xffffffffu, w, 0);
          if (!w) {
            ok = false;
            break;
          }
          const CUtensorMap* m = r ? &tmV : &tmK;
          uint8_t* dst = sKV + st * C::KV_BYTES;
          if (lane == 0) mbar_expect_tx(kv_full + st, C::KV_BYTES);
          if (!p.block_table) {
            if (lane == 0)
              for (int kb = 0; kb < HD / 64; ++kb)
                tma_load_4d(dst + kb * BN * 128, m, kv_full + st, kb * 64, x.kvh, j * BN, x.b);
          } else {
            // one box per page, each lane issuing its own page's boxes (the expected bytes
            // were posted by lane 0 first)
            __syncwarp();
            const int ppt = BN / p.page_size;
            if (lane < ppt)
              for (int kb = 0; kb < HD / 64; ++kb)
                tma_load_4d(dst + kb * BN * 128 + lane * p.page_size * 128, m, kv_full + st, kb * 64, x.kvh, 0,
                            page);
          }
          ++use;
        }
      }
      if (!ok) break;
      NEXT_PIECE
    }
    // The loads of the last NS uses land before the CTA exits (immediate when the MMA warp
    // consumed them; after an abort they may still be in flight).
    if (lane == 0)
      for (int w = (use > NS ? use - NS : 0); w < use; ++w) mbar_wait_drain(kv_full + w % NS, (w / NS) & 1, DRAIN_LIMIT_NS);
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint64_t dQ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sKV), BN * 128, 1024);
      int use = 0, c = 0;
      if (a.test_stall && !mbar_wait(never, 0, abort_flag, p.status, a.wait_ns)) goto mma_drain;
      {
        FOR_EACH_PIECE(pc) {
          PIECE_BOUNDS
          (void)jb;
          if (!mbar_wait(q_full, pc & 1, abort_flag, p.status, a.wait_ns)) goto mma_drain;
          tc_fence_after();
          for (int k = 0; k < nt; ++k, ++c) {
            // keys at ring use `use`; values at use + 1, or (one cache) the same use
            const int stK = use % NS, uV = a.kv_same ? use : use + 1, stV = uV % NS;
            if (!mbar_wait_poll(kv_full + stK, (use / NS) & 1, abort_flag, p.status, a.wait_ns)) goto mma_drain;
            tc_fence_after();
            const uint64_t bk = dK + (uint64_t)((stK * C::KV_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * (BN * 128) + (kk & 3) * 32) >> 4;
              umma_ss(tmem, dQ + off, bk + off, C::IDESC_QK, kk > 0);
            }
            umma_commit(s_full);
            if (!a.kv_same) umma_commit(kv_empty + stK);
            if (!mbar_wait_poll(kv_full + stV, (uV / NS) & 1, abort_flag, p.status, a.wait_ns)) goto mma_drain;
            if (!mbar_wait_poll(p_full, c & 1, abort_flag, p.status, a.wait_ns)) goto mma_drain;
            tc_fence_after();
            const uint64_t bv = dV + (uint64_t)((stV * C::KV_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              umma_ts(tmem + 128, tmem + kk * 8, bv + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV,
                      (kk > 0 || k > 0) ? 1u : 0u);
            umma_commit(o_done);
            umma_commit(kv_empty + stV);
            use = uV + 1;
          }
          NEXT_PIECE
        }
      }
    mma_drain:
      // every MMA issued above completes before tensor memory is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // ---------------------------------- softmax and query set-up (warp = lane quarter, lane = head)
    const int k4 = warp;
    const uint32_t lq = (uint32_t)(32 * k4) << 16;  // this warp's TMEM lanes
    // q may be the previous kernel's output (the latent fold, launched ahead of this one)
    grid_dependency_wait();
    const float sc = a.scale_log2;
    float* part = reinterpret_cast<float*>(sQ);  // [4][RC][32] while no query tile is needed
    int c = 0, fc = 0;
    FOR_EACH_PIECE(pc) {
      PIECE_BOUNDS
      const int h = x.kvh * G + lane;
      const bool real = lane < G;
      const float slope = (p.alibi.on && real) ? p.alibi.slope[h] * LOG2E : 0.f;
      {
        // The piece's query tile: head i (turned at qpos) in rows i, 32 + i, 64 + i and 96 + i
        // for i < G, other rows zero. Thread tid keeps one 16-byte chunk of every row it
        // writes, so it turns the chunk's four pairs by one set of angles.
        constexpr int CH = HD / 8;
        const int cc = tid % CH;
        float cs[4] = {1.f, 1.f, 1.f, 1.f}, sn[4] = {0.f, 0.f, 0.f, 0.f};
        if (p.rope.on)
#pragma unroll
          for (int e = 0; e < 4; ++e) rope_cos_sin(x.qp, p.rope.hi[cc * 4 + e], p.rope.lo[cc * 4 + e], cs[e], sn[e]);
        const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q);
        // the thread's rows tid/CH, +RSTEP, ...: all their loads are issued before any is used
        constexpr int RSTEP = 128 / CH, NROW = 32 / RSTEP;
        uint4 u4[NROW];
#pragma unroll
        for (int k = 0; k < NROW; ++k) {
          const int row = tid / CH + k * RSTEP;
          u4[k] = row < G ? *reinterpret_cast<const uint4*>(q + ((size_t)x.b * p.H + x.kvh * G + row) * HD + cc * 8)
                          : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < NROW; ++k) {
          const int row = tid / CH + k * RSTEP;
          uint32_t w[4] = {0u, 0u, 0u, 0u};
          if (row < G) {
            const uint32_t in[4] = {u4[k].x, u4[k].y, u4[k].z, u4[k].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float2 f = bf2_to_f2(in[e]);
              if (p.rope.on) rotate_pair(f.x, f.y, cs[e], sn[e]);
              w[e] = f2_to_bf2(f.x, f.y);
            }
          }
          const uint4 v = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) sts128(smem_u32(sQ) + sw128_offset(32 * kk + row, cc * 8, BM), v);
        }
        fence_proxy_async();
        tc_fence_before();  // the previous piece's O reads are complete before this arrive
        mbar_arrive(q_full);
      }
      float m_ref = -INFINITY, l = 0.f;
      for (int kt = 0; kt < nt; ++kt, ++c) {
        const int j = jb + kt;
        if (!mbar_wait_poll(s_full, c & 1, abort_flag, p.status, a.wait_ns)) goto done;
        tc_fence_after();
        const int key0 = j * BN + 32 * k4;  // this warp's 32 keys of the tile
        const bool need_mask = key0 < x.j0 || key0 + 32 > x.j1;
        float xs[32];
        tmem_ld32(tmem + lq + 32 * k4, xs);
        tmem_wait_ld();
        // plain tiles (no bias, no mask) keep the raw scores: the maximum is taken first and
        // scaled once (a positive scale keeps the order), the scale goes into the ex2 FMA
        const bool plain = !p.alibi.on && !need_mask;
        float hx = -INFINITY;
        if (plain) {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int i = 0; i < 32; i += 4)
#pragma unroll
            for (int t = 0; t < 4; ++t) m4[t] = fmaxf(m4[t], xs[i + t]);
          hx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sc;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int key = key0 + i;
            float v = p.alibi.on ? fmaf(xs[i], sc, -slope * fabsf((float)(x.qp - key))) : xs[i] * sc;
            if (need_mask) v = (key >= x.j0 && key < x.j1) ? v : -INFINITY;
            xs[i] = v;
            hx = fmaxf(hx, v);
          }
        }
        // the head's maximum over the whole tile, from the four quarters
        float* rt = red + (c & 1) * 128;
        rt[k4 * 32 + lane] = hx;
        mbar_arrive(red_bar + (c & 1));
        if (!mbar_wait_poll(red_bar + (c & 1), (c >> 1) & 1, abort_flag, p.status, a.wait_ns)) goto done;
        hx = fmaxf(fmaxf(rt[lane], rt[32 + lane]), fmaxf(rt[64 + lane], rt[96 + lane]));
        // same lazy reference as the prefill: move it only by more than 8 (log2 units)
        const float m_exp = (hx > m_ref + 8.f) ? hx : m_ref;
        const float mu = (m_exp == -INFINITY) ? 0.f : m_exp;
        uint32_t pk[16];
        // ex2 arguments by packed FMA: x * s - mu with s = the scale (plain tiles) or 1
        const f2x SC = plain ? pk2(sc, sc) : pk2(1.f, 1.f), NM = pk2(-mu, -mu);
        f2x RS = pk2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          float a0, a1, b0, b1;
          up2(fma2(pk2(xs[2 * i], xs[2 * i + 1]), SC, NM), a0, a1);
          up2(fma2(pk2(xs[2 * i + 2], xs[2 * i + 3]), SC, NM), b0, b1);
          const float e0 = ex2(a0), e1 = ex2(a1), e2 = ex2(b0), e3 = ex2(b1);
          RS = add2(RS, add2(pk2(e0, e1), pk2(e2, e3)));
          pk[i] = f2_to_bf2(e0, e1);
          pk[i + 1] = f2_to_bf2(e2, e3);
        }
        float rs0, rs1;
        up2(RS, rs0, rs1);
        // P over the S columns of this warp's lanes: its keys' weights, zeros for the others
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          uint32_t v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = qq == k4 ? pk[i] : 0u;
          tmem_st16u(tmem + lq + 16 * qq, v);
        }
        const float alpha = (m_exp == m_ref) ? 1.f : ex2(m_ref - m_exp);
        m_ref = m_exp;
        // rescale this quarter's part of O (the previous PV finished before this tile's QK,
        // which this tile waited for); a piece's first PV overwrites O
        if (kt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
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
      // The piece's partial state, once its last PV (and with it every MMA that read the query
      // tile) has completed: the four quarters' O parts are added through that memory.
      if (!mbar_wait(o_done, (c - 1) & 1, abort_flag, p.status, a.wait_ns)) goto done;
      tc_fence_after();
      {
        const size_t prow = (size_t)(u + blockIdx.x) * G + lane;  // slot (unit + CTA), head lane
        lpart[k4 * 32 + lane] = l;
#pragma unroll 1
        for (int r = 0; r < HD / C::RC; ++r) {
#pragma unroll 1
          for (int q4 = 0; q4 < C::RC / 32; ++q4) {
            float o[32];
            tmem_ld32(tmem + lq + 128 + r * C::RC + q4 * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) part[(k4 * C::RC + q4 * 32 + e) * 32 + lane] = o[e];
          }
          mbar_arrive(fin_bar);
          if (!mbar_wait(fin_bar, fc & 1, abort_flag, p.status, a.wait_ns)) goto done;
          ++fc;
          if (real) {
            constexpr int DQ = C::RC / 4;  // columns of this round that this warp adds up
            float4* dst = reinterpret_cast<float4*>(a.partO + prow * HD + r * C::RC + k4 * DQ);
#pragma unroll
            for (int v4 = 0; v4 < DQ / 4; ++v4) {
              float s4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int col = k4 * DQ + v4 * 4 + e;
                s4[e] = part[col * 32 + lane] + part[(C::RC + col) * 32 + lane] +
                        part[(2 * C::RC + col) * 32 + lane] + part[(3 * C::RC + col) * 32 + lane];
              }
              dst[v4] = make_float4(s4[0], s4[1], s4[2], s4[3]);
            }
            if (r == 0 && k4 == 0) {
              // the merge works in natural-log units
              a.partM[prow] = m_ref == -INFINITY ? -INFINITY : m_ref * 0.6931471805599453f;
              a.partL[prow] = lpart[lane] + lpart[32 + lane] + lpart[64 + lane] + lpart[96 + lane];
            }
          }
          mbar_arrive(fin_bar);
          if (!mbar_wait(fin_bar, fc & 1, abort_flag, p.status, a.wait_ns)) goto done;
          ++fc;
        }
      }
      NEXT_PIECE
    }
  }
#undef FOR_EACH_PIECE
#undef PIECE_BOUNDS
#undef NEXT_PIECE
done:
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// The partial states of unit u: slots u + i for the CTAs i that cover its tiles.
struct UnitParts {
  size_t row0;  // partial row of the first slot (slot * G + g)
  int n;        // number of partials (0: the unit has no keys)
};
__device__ __forceinline__ UnitParts unit_parts(const long long* prefix, int U, int nctas, int u, int G, int g) {
  UnitParts r{0, 0};
  const long long s0 = prefix[u], s1 = prefix[u + 1], T = prefix[U];
  if (s1 > s0) {
    const int i0 = cta_of(s0, T, nctas), i1 = cta_of(s1 - 1, T, nctas);
    r.row0 = (size_t)(u + i0) * G + g;
    r.n = i1 - i0 + 1;
  }
  return r;
}

// One warp per (sequence, head): four heads of one sequence per CTA.
__global__ void __launch_bounds__(128) sk_merge_kernel(const DecodeParams p, const float* partO, const float* partM,
                                                       const float* partL, const long long* prefix, int nctas) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * 4 + warp, b = blockIdx.y;
  grid_dependency_wait();  // the decode's partials and counts
  if (h >= p.H) return;
  const int G = p.H / p.KV, hd = p.hd;
  const UnitParts up = unit_parts(prefix, p.B * p.KV, nctas, b * p.KV + h / G, G, h % G);
  float acc[4], M, den;  // hd <= 128
  warp_merge(partM + up.row0, partL + up.row0, partO + up.row0 * hd, G, (size_t)G * hd, up.n, hd, lane, acc, M,
             den);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + ((size_t)b * p.H + h) * hd;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (lane + 32 * i < hd) out[lane + 32 * i] = __float2bfloat16_rn(acc[i] * inv);
  if (p.lse && lane == 0) p.lse[(size_t)b * p.H + h] = den > 0.f ? M + logf(den) : -INFINITY;
}

// Latent attention's merge (one key/value unit per sequence): one CTA per (head, group of
// MERGE_SEQ sequences). Warp w merges the partials of sequence b0 + w into its latent output
// (dc = hd numbers, in shared memory); the value up-projection W_out[h] ([dc][hd_out] bf16,
// staged once per CTA by 16-byte copies) follows: thread (e, half) writes
// out[b, h, e] = sum_m olat[m] W_out[h][m][e] for the sequences of its half of the group.
constexpr int MERGE_SEQ = 8;
constexpr int MERGE_THREADS = 32 * MERGE_SEQ;
__global__ void __launch_bounds__(MERGE_THREADS) sk_merge_up_kernel(const DecodeParams p, const float* partO,
                                                          const float* partM, const float* partL,
                                                          const long long* prefix, int nctas) {
  extern __shared__ uint4 msh[];
  const int h = blockIdx.x, b0 = blockIdx.y * MERGE_SEQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dc = p.hd, ho = p.hd_out, G = p.H;  // KV = 1
  __nv_bfloat16* Ws = reinterpret_cast<__nv_bfloat16*>(msh);    // [dc][ho]
  float* olat = reinterpret_cast<float*>(Ws + (size_t)dc * ho);  // [MERGE_SEQ][dc]
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.W_out) + (size_t)h * dc * ho);
  const int nchunk = dc * ho / 8;
  for (int c0 = threadIdx.x; c0 < nchunk; c0 += 8 * MERGE_THREADS) {  // eight loads in flight per thread
    uint4 v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (c0 + r * MERGE_THREADS < nchunk) v[r] = __ldg(src + c0 + r * MERGE_THREADS);
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (c0 + r * MERGE_THREADS < nchunk) msh[c0 + r * MERGE_THREADS] = v[r];
  }
  grid_dependency_wait();  // the decode's partials and counts (the weights did not depend on it)
  const int b = b0 + warp;
  if (b < p.B) {
    const UnitParts up = unit_parts(prefix, p.B, nctas, b, G, h);
    float acc[4], M, den;  // dc <= 128
    warp_merge(partM + up.row0, partL + up.row0, partO + up.row0 * dc, G, (size_t)G * dc, up.n, dc, lane, acc, M,
               den);
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (lane + 32 * i < dc) olat[warp * dc + lane + 32 * i] = acc[i] * inv;
    if (p.lse && lane == 0) p.lse[(size_t)b * p.H + h] = den > 0.f ? M + logf(den) : -INFINITY;
  }
  __syncthreads();
  const int nb = min(MERGE_SEQ, p.B - b0);
  constexpr int HALF = MERGE_SEQ / 2;
  for (int idx = threadIdx.x; idx < 2 * ho; idx += blockDim.x) {
    const int e = idx % ho, s0 = (idx / ho) * HALF;  // output feature, first sequence of the half
    float acc[HALF];
#pragma unroll
    for (int sq = 0; sq < HALF; ++sq) acc[sq] = 0.f;
#pragma unroll 2
    for (int m = 0; m < dc; m += 4) {
      const float w0 = __bfloat162float(Ws[(size_t)m * ho + e]), w1 = __bfloat162float(Ws[(size_t)(m + 1) * ho + e]);
      const float w2 = __bfloat162float(Ws[(size_t)(m + 2) * ho + e]), w3 = __bfloat162float(Ws[(size_t)(m + 3) * ho + e]);
#pragma unroll
      for (int sq = 0; sq < HALF; ++sq) {
        if (s0 + sq >= nb) break;
        const float4 o = *reinterpret_cast<const float4*>(olat + (s0 + sq) * dc + m);
        acc[sq] = fmaf(o.x, w0, fmaf(o.y, w1, fmaf(o.z, w2, fmaf(o.w, w3, acc[sq]))));
      }
    }
#pragma unroll
    for (int sq = 0; sq < HALF; ++sq)
      if (s0 + sq < nb)
        static_cast<__nv_bfloat16*>(p.out)[((size_t)(b0 + s0 + sq) * p.H + h) * ho + e] = __float2bfloat16_rn(acc[sq]);
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

constexpr int MAX_CTAS = 2 * 148;  // grid bound (two CTAs per SM of a 148-SM part): partial slots

size_t r256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Layout {
  long long* prefix;
  float *O, *M, *L;
};
Layout layout(void* ws, int B, int H, int KV, int hd) {
  const size_t U = (size_t)B * KV, rows = (U + MAX_CTAS) * (size_t)(H / KV);
  char* base = static_cast<char*>(ws);
  Layout l;
  l.prefix = reinterpret_cast<long long*>(base);
  l.O = reinterpret_cast<float*>(base + r256((U + 1) * sizeof(long long)));
  l.M = l.O + rows * hd;
  l.L = l.M + rows;
  return l;
}

template <int HD>
cudaError_t launch_hd(const DecodeParams& p, void* ws, cudaStream_t s) {
  CUtensorMap mk, mv;
  const bool ok = p.block_table
                      ? make_page_map(&mk, p.kcache, p.num_pages, p.page_size, p.KV, HD) &&
                            make_page_map(&mv, p.vcache, p.num_pages, p.page_size, p.KV, HD)
                      : make_cache_map(&mk, p.kcache, p.B, p.Lmax, p.KV, HD) &&
                            make_cache_map(&mv, p.vcache, p.B, p.Lmax, p.KV, HD);
  if (!ok) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  int nctas = std::max(1, std::min(CTAS_PER_SM * sms, MAX_CTAS));
  // Test hook: ATTN_TEST_DECODE_CTAS (1..MAX_CTAS) fixes the grid, so that small inputs also
  // run pieces of many tiles and CTAs that cross several units.
  if (const char* env = std::getenv("ATTN_TEST_DECODE_CTAS")) {
    const int n = std::atoi(env);
    if (n >= 1 && n <= MAX_CTAS) nctas = n;
  }
  const int U = p.B * p.KV;
  const Layout lay = layout(ws, p.B, p.H, p.KV, HD);

  if (U > PLAN_MAX) decode_plan_kernel<<<1, 1024, 0, s>>>(p, lay.prefix, U);

  DecArgs a;
  a.p = p;
  a.scale_log2 = p.scale * LOG2E;
  a.partO = lay.O;
  a.partM = lay.M;
  a.partL = lay.L;
  a.prefix = lay.prefix;
  a.plan_in_cta = U <= PLAN_MAX;
  a.U = U;
  a.nctas = nctas;
  // Test hook (failure detection without a GPU fault): with ATTN_TEST_DECODE_STALL_NS set
  // to a positive number of nanoseconds, every wait of this kernel is bounded by it and
  // the MMA warp first waits on a barrier that nothing signals, so each CTA gives up,
  // records ATTN_ERR_TIMEOUT in the device status word, drains its own copies and exits.
  a.wait_ns = WAIT_LIMIT_NS;
  a.test_stall = 0;
  a.kv_same = p.kcache == p.vcache;
  if (const char* env = std::getenv("ATTN_TEST_DECODE_STALL_NS")) {
    const long long ns = std::atoll(env);
    if (ns > 0) {
      a.wait_ns = (unsigned long long)ns;
      a.test_stall = 1;
    }
  }
  e = cudaFuncSetAttribute(decode_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<HD>::SMEM);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launches: the latent decode follows its fold, which writes only q'
  // (this kernel waits for it before reading q); the merges follow this kernel and wait for it
  // before reading the partials. The plain decode is launched normally: the kernel before it
  // may be writing the cache.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = Cfg<HD>::SMEM;
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = (p.W_out && U <= PLAN_MAX) ? 1 : 0;  // (a plan kernel writes what every role reads)
  if ((e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<HD>, mk, mv, a)) != cudaSuccess) return e;

  if (p.W_out) {
    const size_t smem = (size_t)p.hd * p.hd_out * 2 + (size_t)MERGE_SEQ * p.hd * sizeof(float);
    e = cudaFuncSetAttribute(sk_merge_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(p.H, (p.B + MERGE_SEQ - 1) / MERGE_SEQ);
    cfg.blockDim = dim3(MERGE_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, sk_merge_up_kernel, p, (const float*)lay.O, (const float*)lay.M, (const float*)lay.L,
                           (const long long*)lay.prefix, nctas);
    if (e != cudaSuccess) return e;
  } else {
    cfg.gridDim = dim3((p.H + 3) / 4, p.B);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, sk_merge_kernel, p, (const float*)lay.O, (const float*)lay.M, (const float*)lay.L,
                           (const long long*)lay.prefix, nctas);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace
}  // namespace tcdec

bool decode_tc_supported(const DecodeParams& p, int dtype) {
  const int G = p.H / p.KV;
  return dtype == 1 && (p.hd == 64 || p.hd == 128) && G >= 1 && G <= 32 && tcdec::encode_fn() != nullptr;
}

size_t decode_tc_workspace_bytes(int B, int H, int KV, int hd) {
  const size_t U = (size_t)B * KV, rows = (U + tcdec::MAX_CTAS) * (size_t)(H / KV);
  return tcdec::r256((U + 1) * sizeof(long long)) + sizeof(float) * rows * (hd + 2);
}

// The tensor-core decode: plan, decode (two CTAs per SM over all key tiles) and merge; with
// p.W_out the merge also applies the value up-projection (latent attention).
cudaError_t launch_decode_tc(const DecodeParams& p, void* ws, cudaStream_t s) {
  return p.hd == 128 ? tcdec::launch_hd<128>(p, ws, s) : tcdec::launch_hd<64>(p, ws, s);
}

}  // namespace attn
