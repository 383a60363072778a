// Persistent tensor-core flash prefill for sm_100a, the form for keys that need no turn inside
// the kernel (turned by the key rotation pass or a block's key projection, read from a cache
// that holds them turned, or no rotary embedding at all). One CTA per SM walks a list of work
// units; its roles run on from one unit to the next, so a unit's set-up (the query tile's
// load, turn and move into tensor memory) and its epilogue (normalising and storing the
// output rows) overlap the key tiles of its neighbours instead of idling the tensor core
// between CTAs.
//
// What it computes is the attention core of "Write attention from scratch" (worked
// example): per query row i, softmax over allowed keys j of
//   (R(P_i) q_i . k'_j) / sqrt(hd) - slope_h |P_i - j|,  k'_j = R(j) k_j (turned already)
// with P_i = pos0 + i (key j at position pos0 + j) or, in chunk mode, P_i = qpos0[b] + i over
// cache slots j, weighting the value rows, reached through the key-block recurrences of "Building
// grouped-query attention with RoPE and Flash Attention from scratch" (Step 3): a running
// maximum, a running denominator and a rescaled output accumulator.
//
// Work unit: 128 query rows of one head. Units are ranked longest-first (causal rows near the
// end see the most keys), the heads of one key/value group adjacent so that their reads of a
// K/V tile meet in L2. CTA c of G takes, in round r, the unit of rank r*G + c (r even) or
// r*G + G-1-c (r odd): a snake order that evens out the rounds' long and short units.
//
// Operands (as in the single-slot kernel): Q in tensor memory, S = Q K^T and O += P V as
// TS-form MMAs at N = 128 over whole 128-key tiles, P (bf16) over the S columns it came
// from, S double-buffered. Tensor memory (512 columns): O (hd) | Q0, Q1 (hd/2 each, bf16
// pairs, alternate units) | S0 (128) | S1 (128) from column 256.
// Issue order over the CTA's tiles t (all units in sequence): QK(0); then per tile t:
// QK(t+1) (after a unit's last tile: the next unit's first, if it has keys), PV(t). The
// first PV of a unit waits until the previous unit's output has been read out of O.
//
// Warp roles (22 warps):
//   warps 0-15  softmax: warp w owns TMEM lanes 32*(w%4).. (32 query rows) and keys
//               32*(w/4) .. +31 of every tile; at the end of a unit they leave each row's
//               running maximum and sum in shared memory
//   warps 16-19 query and epilogue: turn the next unit's query tile and move it into its
//               tensor-memory buffer, then write the finished unit's rows (O / l, lse)
//   warp 20     TMA producer (query tiles, K/V tiles through a ring of NS stages)
//   warp 21     TMEM allocation and UMMA issue
// Every wait on a barrier that serves several units names a phase that cannot be two
// phases behind the barrier (where a parity wait would pass early or hang): per-buffer
// barriers for the alternating query buffers and statistics, one-phase-per-unit barriers
// only where the waiter is at most one unit behind.
//
// Masking: a pair outside the causal/window/length limits gets -inf before the row max, so
// its weight is exactly 0; tiles outside a unit's key range are skipped entirely. In chunk
// mode (queries that continue sequences held in a cache) a unit may attend no key at all:
// it has no tiles and writes zero rows with lse = -inf.
#include <algorithm>

#include "prefill_common.cuh"

namespace attn {
namespace tc {
namespace {

constexpr int BM = PF_BM;  // query rows per unit
constexpr int BN = PF_BN;  // keys per tile
constexpr int NUM_WARPS = 22;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int WARP_QE0 = 16;
constexpr int WARP_TMA = 20;
constexpr int WARP_MMA = 21;
constexpr int QE_BARRIER = 1;  // named barrier of the four query/epilogue warps
constexpr uint64_t WAIT_LIMIT_NS = 4000000000ull;  // a wait that lasts 4 s has failed
constexpr uint64_t DRAIN_LIMIT_NS = 100000000ull;  // own copies/MMAs finish in microseconds
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

template <int HD>
struct Cfg {
  static constexpr int NS = HD == 128 ? 5 : 12;  // key/value ring stages
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int KV_BYTES = BN * HD * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
  static constexpr int NBAR = 2 * NS + 24;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // row-max exchange [tile parity][key quarter][128], row sums [unit parity][key quarter][128],
  // row maxima [unit parity][128]
  static constexpr int OFF_RED = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int RED_FLOATS = 2 * 4 * 128 + 2 * 4 * 128 + 2 * 128;
  static constexpr int SMEM = OFF_RED + RED_FLOATS * 4 + 1024;  // + slack to align the base
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static constexpr int COL_O = 0;
  static constexpr int COL_Q = HD;  // two buffers of HD/2 columns
  static constexpr int COL_S = 256;
  static_assert(COL_Q + HD <= COL_S && COL_S + 2 * BN <= 512, "tensor memory layout");
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, 0, 1);
};

struct PsArgs {
  PrefillParams p;
  int nqb;     // query blocks of 128 rows per (sequence, head)
  int nunits;  // B * H * nqb
  float scale_log2;
};

// A unit's rows and key range. Keys are indexed by position in k/v (a prefill: key j is row
// j) or by cache slot (chunk mode); qoff is the key index of query row 0, Tk the number of
// keys, qrope0 the position of row 0; the nt tiles from jt0 on hold the unit's keys.
struct Unit {
  int b, h, g, qs, qoff, Tk, qrope0, jt0, nt;
  bool bad;  // chunk mode: the sequence's cache position or length is out of range
};

// Rank of the n-th unit of this CTA (>= nunits: none; ranks grow with n).
__device__ __forceinline__ int unit_rank(int n) {
  const int G = gridDim.x, c = blockIdx.x;
  return n * G + ((n & 1) ? G - 1 - c : c);
}

// The unit of a rank: longest rows first, heads of one key/value group adjacent.
template <bool CHUNK>
__device__ __forceinline__ Unit unit_at(const PrefillParams& p, int nqb, int rank) {
  Unit x;
  const int per_qb = p.B * p.H;
  const int qb = nqb - 1 - rank / per_qb;
  const int rest = rank % per_qb;
  x.h = rest % p.H;
  x.b = rest / p.H;
  x.g = x.h / (p.H / p.KV);
  x.qs = qb * BM;
  x.qoff = 0;
  x.Tk = p.T;
  x.qrope0 = p.pos0;
  x.bad = false;
  if constexpr (CHUNK) {
    x.qoff = p.qpos0[x.b];
    x.Tk = p.seqlens[x.b];
    x.qrope0 = x.qoff;
    if (x.qoff < 0 || x.qoff > (1 << 24) - p.T || x.Tk < 0 || x.Tk > p.Lk) {
      x.bad = true;
      x.qoff = 0;
      x.Tk = 0;  // nothing is attended: zero rows
    }
  }
  // keys lo..hi (in a prefill lo <= qs <= hi: every unit has a tile)
  const int lo = p.window > 0 ? max(0, x.qoff + x.qs - p.window + 1) : 0;
  const int hi = p.causal ? min(x.Tk - 1, x.qoff + x.qs + BM - 1) : x.Tk - 1;
  x.jt0 = lo <= hi ? lo / BN : 0;
  x.nt = lo <= hi ? hi / BN - x.jt0 + 1 : 0;
  return x;
}

__device__ __forceinline__ void qe_sync() { asm volatile("bar.sync %0, 128;" ::"n"(QE_BARRIER) : "memory"); }

template <int HD, bool CHUNK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_ps_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ PsArgs a) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;               // [stage]: a K or V tile landed
  uint64_t* kv_empty = bars + C::NS;      // [stage]: the MMAs that read it completed
  uint64_t* q_full = bars + 2 * C::NS;    // a unit's query tile landed (one phase per unit)
  uint64_t* q_rot = q_full + 1;           // [query buffer]: a unit's query tile is in TMEM
  uint64_t* s_full = q_full + 3;          // [S buffer]: a QK completed
  uint64_t* p_full = q_full + 5;          // [S buffer]: P written (and O rescaled)
  uint64_t* o_done = q_full + 7;          // [S buffer]: the PV of a tile in it completed
  uint64_t* red_bar = q_full + 9;         // [tile parity][lane quarter]: row maxima written
  uint64_t* stats = q_full + 17;          // [unit parity]: row maxima and sums of a unit written
  uint64_t* stats_free = q_full + 19;     // [unit parity]: the epilogue read them
  uint64_t* unit_done = q_full + 21;      // every MMA of a unit completed (one phase per unit)
  uint64_t* o_free = q_full + 22;         // the epilogue read a unit's O (one phase per unit)
  uint64_t* drain = q_full + 23;          // the MMA thread's final commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [tile parity][kq][128] row maxima
  float* lsum = red + 2 * 4 * 128;                            // [unit parity][kq][128] row sums
  float* mrow = lsum + 2 * 4 * 128;                           // [unit parity][128] row maxima

  const PrefillParams& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto has_unit = [&](int n) { return unit_rank(n) < a.nunits; };
  auto unit = [&](int n) { return unit_at<CHUNK>(p, a.nqb, unit_rank(n)); };

  // ---- set-up: barriers, tensor memory
  if (tid == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_rot + s, 128);
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 16);  // one arrival per softmax warp
      mbar_init(o_done + s, 1);
      for (int qq = 0; qq < 4; ++qq) mbar_init(red_bar + 4 * s + qq, 4);
      mbar_init(stats + s, 16);
      mbar_init(stats_free + s, 128);
    }
    mbar_init(unit_done, 1);
    mbar_init(o_free, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch(&tmQ);
      tma_prefetch(&tmK);
      tma_prefetch(&tmV);
      int nq = 0, u = 0;  // query tiles and ring uses issued
      auto issue_q = [&](int n) {
        const Unit x = unit(n);
        mbar_expect_tx(q_full, C::Q_BYTES);
        for (int kb = 0; kb < HD / 64; ++kb)
          tma_load_4d(sQ + kb * BM * 128, &tmQ, q_full, kb * 64, x.h, x.qs, x.b);
        ++nq;
      };
      bool ok = true;
      if (has_unit(0)) issue_q(0);
      // after the key rotation pass (programmatic dependent launch), keys are read only once
      // that grid has completed; without a dependency this returns at once
      grid_dependency_wait();
      for (int n = 0; ok && has_unit(n); ++n) {
        const Unit x = unit(n);
        if (x.bad) flag_error(p.status, DEV_BAD_ARG);
        // The next unit's query tile goes into the one query buffer as soon as this unit's
        // tile has moved into tensor memory (q_rot of unit n; it cannot be a phase ahead,
        // as unit n+2's tile needs the load issued here).
        bool q_next = !has_unit(n + 1);
        const int total = 2 * x.nt;  // K and V of every tile
        for (int k = 0; k < total; ++k, ++u) {
          if (!q_next && mbar_test_wait(q_rot + (n & 1), (n >> 1) & 1)) {
            issue_q(n + 1);
            q_next = true;
          }
          const int st = u % C::NS, m = u / C::NS, j = x.jt0 + k / 2, kv = k & 1;
          if (!mbar_wait(kv_empty + st, (m & 1) ^ 1, abort_flag, p.status, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          mbar_expect_tx(kv_full + st, C::KV_BYTES);
          for (int kb = 0; kb < HD / 64; ++kb)
            tma_load_4d(sKV + st * C::KV_BYTES + kb * BN * 128, kv ? &tmV : &tmK, kv_full + st,
                        kb * 64, x.g, j * BN, x.b);
        }
        if (ok && !q_next) {
          if (!mbar_wait(q_rot + (n & 1), (n >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) break;
          issue_q(n + 1);
        }
      }
      // The copies issued last land before the CTA exits (immediate when they were
      // consumed; after an abort they may still be in flight).
      if (nq > 0) mbar_wait_drain(q_full, (nq - 1) & 1, DRAIN_LIMIT_NS);
      for (int w = (u > C::NS ? u - C::NS : 0); w < u; ++w)
        mbar_wait_drain(kv_full + w % C::NS, (w / C::NS) & 1, DRAIN_LIMIT_NS);
    }
  } else if (warp >= WARP_QE0 && warp < WARP_QE0 + 4) {
    // ------------------------------------------------------------ query and epilogue
    const int r = tid - WARP_QE0 * 32;  // row of a unit this thread moves in and writes out
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    KRot<HD> krot;
    if (p.rope.on) krot.init(r, p.rope);
    // Unit n's query: turn the tile in place (thread = 16-byte chunk, rows by the angle
    // recurrence), then each thread moves one row into query buffer n&1 of tensor memory
    // (column c: features 2c, 2c+1, one rotary pair). That buffer was last read by the QKs
    // of unit n-2, which had completed when the epilogue of unit n-2 began.
    auto prep = [&](int n) -> bool {
      const Unit x = unit(n);
      if (!mbar_wait(q_full, n & 1, abort_flag, p.status, WAIT_LIMIT_NS)) return false;
      if (p.rope.on) krot.rotate(sQ, x.qrope0 + x.qs, p.rope);
      qe_sync();
      const uint32_t base = smem_u32(sQ);
      const uint32_t colq = C::COL_Q + (uint32_t)(n & 1) * (HD / 2);
#pragma unroll
      for (int hb = 0; hb < HD / 64; ++hb) {
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = lds128(base + sw128_offset(r, hb * 64 + c * 8, BM));
          w[4 * c] = v.x;
          w[4 * c + 1] = v.y;
          w[4 * c + 2] = v.z;
          w[4 * c + 3] = v.w;
        }
        tmem_st32u(tmem + lane_off + colq + hb * 32, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(q_rot + (n & 1));
      return true;
    };
    // Unit n's output: out = O / l (bf16), lse = (m + log2 l) ln 2, once every MMA of the
    // unit completed and the softmax warps left the rows' statistics.
    auto epilogue = [&](int n) -> bool {
      const Unit x = unit(n);
      if (!mbar_wait(unit_done, n & 1, abort_flag, p.status, WAIT_LIMIT_NS)) return false;
      tc_fence_after();
      const int sb = n & 1;
      if (!mbar_wait(stats + sb, (n >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) return false;
      const float* ls = lsum + sb * 512;
      const float lt = (ls[r] + ls[128 + r]) + (ls[256 + r] + ls[384 + r]);
      const float m = mrow[sb * 128 + r];
      mbar_arrive(stats_free + sb);
      const int i = x.qs + r;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                            (((size_t)x.b * p.T + i) * p.H + x.h) * HD);
      if (x.nt == 0) {
        // no key attended (chunk mode): zero rows; O belongs to another unit and is not read
        if (i < p.T)
          for (int v4 = 0; v4 < HD / 8; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
      } else {
#pragma unroll
      for (int hb = 0; hb < HD / 32; ++hb) {
        float o[32];
        tmem_ld32(tmem + lane_off + C::COL_O + hb * 32, o);
        tmem_wait_ld();
        if (i < p.T) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[hb * 4 + v4] = make_uint4(f2_to_bf2(o[8 * v4] * inv, o[8 * v4 + 1] * inv),
                                          f2_to_bf2(o[8 * v4 + 2] * inv, o[8 * v4 + 3] * inv),
                                          f2_to_bf2(o[8 * v4 + 4] * inv, o[8 * v4 + 5] * inv),
                                          f2_to_bf2(o[8 * v4 + 6] * inv, o[8 * v4 + 7] * inv));
        }
      }
      }
      tc_fence_before();
      mbar_arrive(o_free);
      if (p.lse && i < p.T)
        p.lse[((size_t)x.b * p.H + x.h) * p.T + i] = lt > 0.f ? (m + __log2f(lt)) * LN2 : -INFINITY;
      return true;
    };
    if (has_unit(0) && !prep(0)) goto done;
    for (int n = 0; has_unit(n); ++n) {
      if (has_unit(n + 1) && !prep(n + 1)) goto done;
      if (!epilogue(n)) goto done;
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ UMMA issue
    if (lane == 0) {
      // Descriptors are built once; the start-address field (bits 0-13, in 16-byte units)
      // is then advanced by plain additions that stay below 2^14.
      const uint64_t dK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sKV), BN * 128, 1024);
      auto issue_qk = [&](int buf, int st, int qbuf) {
        const uint32_t d = tmem + C::COL_S + buf * BN;
        const uint32_t aq = tmem + C::COL_Q + qbuf * (HD / 2);
        const uint64_t b0 = dK + (uint64_t)((st * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * (BN * 128) + (kk & 3) * 32) >> 4;
          umma_ts(d, aq + kk * 8, b0 + off, C::IDESC_QK, kk > 0);
        }
      };
      auto issue_pv = [&](int buf, int st, bool acc) {
        const uint32_t d = tmem + C::COL_O;
        const uint32_t aP = tmem + C::COL_S + buf * BN;  // P: 64 columns of bf16 pairs over S
        const uint64_t b0 = dV + (uint64_t)((st * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts(d, aP + kk * 8, b0 + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV,
                  (kk > 0 || acc) ? 1u : 0u);
      };
      // tile t of the CTA (all units in sequence): keys at ring use 2t, values at 2t + 1
      auto wait_kv = [&](int u) -> bool {
        return mbar_wait(kv_full + u % C::NS, (u / C::NS) & 1, abort_flag, p.status, WAIT_LIMIT_NS);
      };
      int t = 0;
      // QK of a unit's first tile: issued ahead, during the previous unit's last tile, when
      // that unit had tiles; otherwise (the CTA's first unit, or one after a unit without
      // keys) at the unit's start. Its query buffer's q_rot cannot be a phase ahead: unit
      // n+2's query waits for the epilogue of unit n, which waits for unit n's MMAs.
      bool first_qk_issued = false;
      for (int n = 0; has_unit(n); ++n) {
        const Unit x = unit(n);
        const int nt = x.nt;
        if (nt > 0 && !first_qk_issued) {
          if (!mbar_wait(q_rot + (n & 1), (n >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
          if (!wait_kv(2 * t)) goto mma_drain;
          tc_fence_after();
          issue_qk(t & 1, (2 * t) % C::NS, n & 1);
          umma_commit(s_full + (t & 1));
          umma_commit(kv_empty + (2 * t) % C::NS);
        }
        first_qk_issued = false;
        const bool next_has_tiles = has_unit(n + 1) && unit(n + 1).nt > 0;
        for (int i = 0; i < nt; ++i, ++t) {
          // QK of the CTA's next tile: this unit's next one, or the next unit's first
          if (i + 1 < nt || next_has_tiles) {
            const int nq = i + 1 < nt ? n : n + 1;
            if (nq != n) {
              if (!mbar_wait(q_rot + (nq & 1), (nq >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
                goto mma_drain;
              first_qk_issued = true;
            }
            const int uK = 2 * (t + 1);
            if (!wait_kv(uK)) goto mma_drain;
            tc_fence_after();
            issue_qk((t + 1) & 1, uK % C::NS, nq & 1);
            umma_commit(s_full + ((t + 1) & 1));
            umma_commit(kv_empty + uK % C::NS);
          }
          const int uV = 2 * t + 1;
          if (!wait_kv(uV)) goto mma_drain;
          if (!mbar_wait(p_full + (t & 1), (t >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
          // the unit's first PV overwrites O: the previous unit's rows must have been read
          if (i == 0 && n > 0 && !mbar_wait(o_free, (n - 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
            goto mma_drain;
          tc_fence_after();
          issue_pv(t & 1, uV % C::NS, i > 0);
          umma_commit(o_done + (t & 1));
          umma_commit(kv_empty + uV % C::NS);
        }
        // Every MMA of the unit completed. A unit without keys has no PV to wait for the
        // previous unit's epilogue; it waits here, so that unit_done never runs two phases
        // ahead of the epilogue warps that wait on it.
        if (nt == 0 && n > 0 && !mbar_wait(o_free, (n - 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
          goto mma_drain;
        umma_commit(unit_done);
      }
    mma_drain:
      // every MMA issued above completes before tensor memory is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-15)
    // Warp w owns TMEM lanes 32*(w%4).. (32 query rows) and keys kq*32 .. kq*32+31 of every
    // tile, kq = w/4. The four warps of a row exchange their maxima through shared memory,
    // all derive the same row reference, and each writes the P (bf16) of its 32 keys to TMEM
    // columns kq*16 .. kq*16+15 of the tile's S buffer (every S column of those rows was read
    // before the exchange). O is rescaled (rarely) by column quarter, once the previous
    // tile's PV has completed; never at a unit's first tile, whose PV overwrites O.
    const int kq = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float sc = a.scale_log2;
    int t = 0;  // tile count over the CTA's units
    for (int n = 0; has_unit(n); ++n) {
      const Unit x = unit(n);
      const int Tk = x.Tk;
      const int q0 = x.qoff + x.qs;  // key index of the unit's first query row
      const int ip = q0 + r;         // the query's key index
      const float slope = p.alibi.on ? p.alibi.slope[x.h] * LOG2E : 0.f;
      // Row state in the log2 domain: m_ref is the reference the weights are taken against
      // (-inf until the row has seen an allowed key), l the running sum of this warp's share
      // of the weights. The reference moves only when a tile's maximum exceeds it by more than
      // 8 (a factor 256), so O is rescaled rarely; weights stay below 2^8.
      float m_ref = -INFINITY, l = 0.f;
#pragma unroll 1
      for (int j = x.jt0; j < x.jt0 + x.nt; ++j, ++t) {
        const int buf = t & 1;
        if (!mbar_wait(s_full + buf, (t >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + C::COL_S + buf * BN;
        const int key0 = j * BN + kq * 32;  // first of my 32 keys
        // does any row of this tile need per-element masking in my keys? (uniform per warp)
        const bool need_mask = (key0 + 32 > Tk) || (p.causal && key0 + 31 > q0) ||
                               (p.window > 0 && q0 + BM - 1 - key0 >= p.window);
        float xv[32];
        tmem_ld32(tS + kq * 32, xv);
        tmem_wait_ld();
        if (p.alibi.on) {
          // -slope |i - j| is, with the causal mask, slope (j - i) on every allowed pair: an
          // affine function c0 + slope k of the key
          const float c0 = slope * (float)(key0 - ip);
#pragma unroll
          for (int k = 0; k < 32; ++k)
            xv[k] = p.causal ? fmaf(xv[k], sc, fmaf(slope, (float)k, c0))
                             : fmaf(xv[k], sc, -slope * fabsf((float)(ip - key0 - k)));
        }
        if (need_mask) {
          // my keys allowed for this row: kmin <= k < kmax
          int kmax = Tk - key0;
          if (p.causal) kmax = min(kmax, ip - key0 + 1);
          const int kmin = p.window > 0 ? ip - p.window + 1 - key0 : 0;
#pragma unroll
          for (int k = 0; k < 32; ++k) xv[k] = (k >= kmin && k < kmax) ? xv[k] : -INFINITY;
        }
        // without ALiBi the scores are still unscaled: a positive scale keeps the order
        const float hx = p.alibi.on ? max32(xv) : max32(xv) * sc;
        float* rb = red + buf * 512;
        rb[kq * 128 + r] = hx;
        __syncwarp();
        if (lane == 0) mbar_arrive(red_bar + 4 * buf + (warp & 3));
        if (!mbar_wait(red_bar + 4 * buf + (warp & 3), (t >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
          goto done;
        const float mt = fmaxf(fmaxf(rb[r], rb[128 + r]), fmaxf(rb[256 + r], rb[384 + r]));
        const float m_new = (mt > m_ref + 8.f) ? mt : m_ref;  // takes mt when m_ref = -inf
        const float alpha = (m_new == m_ref) ? 1.f : ex2(m_ref - m_new);
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        m_ref = m_new;
        f2x RS = pk2(0.f, 0.f);
        uint32_t pk[16];  // column k: keys 2k, 2k+1 of my 32 (low half = even key)
        const f2x SC = p.alibi.on ? pk2(1.f, 1.f) : pk2(sc, sc), NM = pk2(-mu, -mu);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float a0, a1, b0, b1;
          up2(fma2(pk2(xv[4 * k], xv[4 * k + 1]), SC, NM), a0, a1);
          up2(fma2(pk2(xv[4 * k + 2], xv[4 * k + 3]), SC, NM), b0, b1);
          const float e0 = ex2(a0), e1 = ex2(a1), e2 = ex2(b0), e3 = ex2(b1);
          RS = add2(RS, add2(pk2(e0, e1), pk2(e2, e3)));
          pk[2 * k] = f2_to_bf2(e0, e1);
          pk[2 * k + 1] = f2_to_bf2(e2, e3);
        }
        tmem_st16u(tS + kq * 16, pk);
        // O is rescaled before this tile's PV is issued, once the previous PV has completed
        if (j > x.jt0 && kq * 32 < HD && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!mbar_wait(o_done + ((t - 1) & 1), ((t - 1) >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
            goto done;
          tc_fence_after();
          const uint32_t tO = tmem + lane_off + C::COL_O + kq * 32;
          float o[32];
          tmem_ld32(tO, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tO, o);
        }
        {
          float r0, r1;
          up2(RS, r0, r1);
          l = l * alpha + (r0 + r1);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + buf);
      }
      // the unit's row statistics for the epilogue warps: buffer n&1 is free once they read
      // those of unit n-2 (stats_free cannot be a phase ahead: unit n's are not written yet)
      const int sb = n & 1;
      if (n >= 2 && !mbar_wait(stats_free + sb, ((n - 2) >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
        goto done;
      lsum[sb * 512 + kq * 128 + r] = l;
      if (kq == 0) mrow[sb * 128 + r] = m_ref;
      __syncwarp();
      if (lane == 0) mbar_arrive(stats + sb);
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
template <int HD>
cudaError_t launch_ps(const PrefillParams& p, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const int Lk = p.seqlens ? p.Lk : p.T;  // rows of k and v
  if (!make_map(&mq, p.q, p.B, p.T, p.H, HD) || !make_map(&mk, p.k, p.B, Lk, p.KV, HD) ||
      !make_map(&mv, p.v, p.B, Lk, p.KV, HD))
    return cudaErrorInvalidValue;
  PsArgs a;
  a.p = p;
  a.nqb = (p.T + BM - 1) / BM;
  a.scale_log2 = p.scale * LOG2E;
  const long long units = (long long)p.B * p.H * a.nqb;
  if (units > 0x3fffffffLL) return cudaErrorInvalidValue;
  a.nunits = (int)units;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::min<long long>(units, (long long)sms);
  auto kern = p.seqlens ? prefill_ps_kernel<HD, true> : prefill_ps_kernel<HD, false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<HD>::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = Cfg<HD>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.after_key_pass ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, a);
}

}  // namespace
}  // namespace tc

bool prefill_ps_supported(const PrefillParams& p) {
  // chunk mode reads keys turned in the cache
  return (p.seqlens || p.k_rotated || !p.rope.on) && (p.hd == 64 || p.hd == 128);
}

cudaError_t launch_prefill_ps(const PrefillParams& p, cudaStream_t s) {
  if (!prefill_ps_supported(p)) return cudaErrorInvalidValue;
  return p.hd == 128 ? tc::launch_ps<128>(p, s) : tc::launch_ps<64>(p, s);
}

}  // namespace attn
