// Tensor-core flash prefill for sm_100a: TMA-staged tiles, tcgen05 MMAs accumulating in
// TMEM, warp-specialised online softmax, rotary embedding applied as tiles land. One CTA per
// 128-row unit; it serves attn_prefill without a workspace for hd = 64 with RoPE, where the keys
// are turned inside the kernel (hd = 128 takes the two-slot kernel of prefill_pair.cu; every
// prefill whose keys need no turn here, and every chunk, takes the persistent kernel of
// prefill_persist.cu).
//
// What it computes is the attention core of "Write attention from scratch" (worked
// example): per query row i, softmax over allowed keys j of
//   (R(pos0+i) q_i . R(pos0+j) k_j) / sqrt(hd) - slope_h |i - j|
// weighting the value rows, reached through the key-block recurrences of "Building
// grouped-query attention with RoPE and Flash Attention from scratch" (Step 3): a running
// maximum, a running denominator and a rescaled output accumulator.
//
// Work unit (one CTA): 128 query rows of one head. CTAs are numbered longest-first (causal
// rows near the end see the most keys) so the block scheduler packs them like an LPT
// schedule, and the heads of one key/value group are adjacent, so the four reads of each
// K/V tile of a GQA group meet in L2.
//
// Operands. The query tile is turned once and moved into tensor memory, so S = Q K^T is a
// TS-form MMA whose only shared-memory operand is the key tile; O += P V is a TS-form MMA
// that reads P (bf16) from tensor memory. Both run at N = 128 over whole 128-key tiles,
// which K/V tiles reach through a TMA ring of NS stages (keys turned in place as they
// land). S is double-buffered in tensor memory: the tensor core computes the scores of key
// tile j+1 while the softmax works on tile j. Tensor memory (512 columns): O (hd) | Q
// (hd/2: bf16 pairs) | ... | S0 (128) | S1 (128) from column 256.
// Issue order: QK(0); then per tile j: QK(j+1), PV(j). QK(j+1) overwrites the S/P buffer of
// tile j-1 only after PV(j-1) (the tensor core executes one CTA's MMAs in issue order).
//
// Warp roles (22 warps):
//   warps 0-15  softmax: warp w owns TMEM lanes 32*(w%4).. (32 query rows) and keys
//               32*(w/4) .. +31 of every tile
//   warps 16-19 rotary embedding: turns the Q tile in place and moves it into tensor memory,
//               then turns every K tile in place in its 128-byte-swizzled layout
//   warp 20     TMA producer (the Q tile, then K/V tiles through the ring)
//   warp 21     TMEM allocation and UMMA issue
//
// Masking: a pair outside the causal/window/length limits gets -inf before the row max,
// so its weight is exactly 0, and the sums' order depends only on the tile structure;
// a row's output never depends on the keys it may not see. Tiles outside the key range
// are skipped entirely.
#include "prefill_common.cuh"

namespace attn {
namespace tc {
namespace {

constexpr int BM = PF_BM;  // query rows per CTA
constexpr int BN = PF_BN;  // keys per tile
constexpr int NUM_WARPS = 22;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int WARP_ROPE0 = 16;
constexpr int WARP_TMA = 20;
constexpr int WARP_MMA = 21;
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
  static constexpr int NBAR = 3 * NS + 19;
  // the MMA thread waits for tile j+1's keys before issuing tile j's PV: the ring must hold
  // more than two tiles so that those keys never wait for a stage only that PV frees
  static_assert(NS >= 5, "ring depth");
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // row-max exchange [parity][key quarter][128] and row-sum exchange [key quarter][128]
  static constexpr int OFF_RED = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int RED_FLOATS = 2 * 4 * 128 + 4 * 128;
  static constexpr int SMEM = OFF_RED + RED_FLOATS * 4 + 1024;  // + slack to align the base
  // tensor-memory columns
  static constexpr int COL_O = 0;
  static constexpr int COL_Q = HD;
  static constexpr int COL_S = 256;
  static_assert(COL_Q + HD / 2 <= COL_S && COL_S + 2 * BN <= 512, "tensor memory layout");
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, 0, 1);
};

struct TcArgs {
  PrefillParams p;
  int nqb;         // query blocks of 128 rows per (sequence, head)
  float scale_log2;
};

template <int HD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ TcArgs a) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sKV = smem + C::OFF_KV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + C::NS;
  uint64_t* k_rot = bars + 2 * C::NS;
  uint64_t* q_full = bars + 3 * C::NS;
  uint64_t* q_turned = q_full + 1;  // all rotary threads turned their query chunks in place
  uint64_t* q_rot = q_full + 2;     // the query tile is in tensor memory
  uint64_t* s_full = q_full + 3;    // [S buffer]: a QK completed
  uint64_t* p_full = q_full + 5;    // [S buffer]: P written (and O rescaled)
  // [S buffer]: the PV of a tile in that buffer (and every MMA before it) completed. One per
  // buffer: with QK a tile ahead of PV, a single barrier can be two phases behind its waiter
  // at the last tile, where a parity wait would pass early.
  uint64_t* o_done = q_full + 7;
  uint64_t* red_bar = q_full + 9;   // [parity of the tile count][lane quarter]: the four warps of
                                    // those rows wrote their maxima
  uint64_t* lsum_bar = q_full + 17; // all warps' row sums written
  uint64_t* drain = q_full + 18;    // the MMA thread's final commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const PrefillParams& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work unit: longest rows first; the heads of a key/value group adjacent
  const int per_qb = p.B * p.H;
  const int qb = a.nqb - 1 - (int)(blockIdx.x / per_qb);
  const int rest = blockIdx.x % per_qb;
  const int h = rest % p.H;
  const int b = rest / p.H;
  const int g = h / (p.H / p.KV);
  const int qs = qb * BM;
  // Key j is row j of k/v: qoff is the key index of query row 0, Tk the number of keys.
  const int qoff = 0, Tk = p.T, qrope0 = p.pos0;
  const int lo = p.window > 0 ? max(0, qoff + qs - p.window + 1) : 0;
  const int hi = p.causal ? min(Tk - 1, qoff + qs + BM - 1) : Tk - 1;
  const bool has = lo <= hi;  // the tile attends at least one key
  const int jt0 = has ? lo / BN : 1, jt1 = has ? hi / BN : 0;

  // ---- set-up: barriers, tensor memory
  if (tid == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
      mbar_init(k_rot + i, 128);
    }
    mbar_init(q_full, 1);
    mbar_init(q_turned, 128);
    mbar_init(q_rot, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 16);   // one arrival per softmax warp
      for (int qq = 0; qq < 4; ++qq) mbar_init(red_bar + 4 * s + qq, 4);
    }
    mbar_init(o_done, 1);
    mbar_init(o_done + 1, 1);
    mbar_init(lsum_bar, 16);
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
      mbar_expect_tx(q_full, C::Q_BYTES);
      for (int kb = 0; kb < HD / 64; ++kb)
        tma_load_4d(sQ + kb * BM * 128, &tmQ, q_full, kb * 64, h, qs, b);
      const int total = 2 * (jt1 - jt0 + 1);  // K and V of every tile
      int u = 0;
      for (; u < total; ++u) {
        const int st = u % C::NS, n = u / C::NS, j = jt0 + u / 2, kv = u & 1;
        if (!mbar_wait(kv_empty + st, (n & 1) ^ 1, abort_flag, p.status, WAIT_LIMIT_NS)) break;
        mbar_expect_tx(kv_full + st, C::KV_BYTES);
        for (int kb = 0; kb < HD / 64; ++kb)
          tma_load_4d(sKV + st * C::KV_BYTES + kb * BN * 128, kv ? &tmV : &tmK, kv_full + st,
                      kb * 64, g, j * BN, b);
      }
      // The copies issued last land before the CTA exits (immediate when they were
      // consumed; after an abort they may still be in flight).
      mbar_wait_drain(q_full, 0, DRAIN_LIMIT_NS);
      for (int w = (u > C::NS ? u - C::NS : 0); w < u; ++w)
        mbar_wait_drain(kv_full + w % C::NS, (w / C::NS) & 1, DRAIN_LIMIT_NS);
    }
  } else if (warp >= WARP_ROPE0 && warp < WARP_ROPE0 + 4) {
    // ------------------------------------------------------------ rotary embedding
    const int r = tid - WARP_ROPE0 * 32;  // row of the query tile this thread moves to TMEM
    KRot<HD> krot;
    if (p.rope.on) krot.init(r, p.rope);
    if (!mbar_wait(q_full, 0, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
    // Turn the query tile in place (thread = 16-byte chunk, rows by the angle recurrence),
    // then each thread moves one row into the Q columns of tensor memory, where the QK MMAs
    // read it as their A operand: column c holds features 2c (low half) and 2c + 1, one
    // rotary pair.
    if (p.rope.on) krot.rotate(sQ, qrope0 + qs, p.rope);
    mbar_arrive(q_turned);
    if (!mbar_wait(q_turned, 0, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
    {
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t base = smem_u32(sQ);
#pragma unroll
      for (int hb = 0; hb < HD / 64; ++hb) {
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 u = lds128(base + sw128_offset(r, hb * 64 + c * 8, BM));
          w[4 * c] = u.x;
          w[4 * c + 1] = u.y;
          w[4 * c + 2] = u.z;
          w[4 * c + 3] = u.w;
        }
        tmem_st32u(tmem + lane_off + C::COL_Q + hb * 32, w);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(q_rot);
    // hd = 128: key-tile start angles by recurrence; hd = 64 (half the rotation work per
    // tile) computes each accurately
    if constexpr (HD == 128)
      if (p.rope.on && !p.k_rotated) krot.start_keys(p.pos0 + jt0 * BN, p.rope);
    int u = 0;
    for (int j = jt0; j <= jt1; ++j) {
      for (int kv = 0; kv < 2; ++kv, ++u) {
        const int st = u % C::NS, n = u / C::NS;
        if (!mbar_wait(kv_full + st, n & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
        if (kv == 0 && p.rope.on && !p.k_rotated) {  // keys that arrive turned are not turned again
          if constexpr (HD == 128)
            krot.rotate_next(sKV + st * C::KV_BYTES);
          else
            krot.rotate(sKV + st * C::KV_BYTES, p.pos0 + j * BN, p.rope);
        }
        fence_proxy_async();
        mbar_arrive(k_rot + st);
      }
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ UMMA issue
    if (lane == 0) {
      // Descriptors are built once; the start-address field (bits 0-13, in 16-byte units)
      // is then advanced by plain additions that stay below 2^14.
      const uint64_t dK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sKV), BN * 128, 1024);
      auto issue_qk = [&](int buf, int st) {
        const uint32_t d = tmem + C::COL_S + buf * BN;
        const uint32_t aq = tmem + C::COL_Q;
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
      // ring use u of tile j: keys at u = 2 (j - jt0), values at u + 1
      auto wait_rot = [&](int u) -> bool {
        return mbar_wait(k_rot + u % C::NS, (u / C::NS) & 1, abort_flag, p.status, WAIT_LIMIT_NS);
      };
      if (!mbar_wait(q_rot, 0, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
      if (!has) goto mma_drain;  // no key at all
      if (!wait_rot(0)) goto mma_drain;
      tc_fence_after();
      issue_qk(0, 0);
      umma_commit(s_full);
      umma_commit(kv_empty);
      for (int i = 0; i <= jt1 - jt0; ++i) {
        if (i < jt1 - jt0) {
          const int uK = 2 * (i + 1);
          if (!wait_rot(uK)) goto mma_drain;  // keys of the next tile, turned
          tc_fence_after();
          issue_qk((i + 1) & 1, uK % C::NS);
          umma_commit(s_full + ((i + 1) & 1));
          umma_commit(kv_empty + uK % C::NS);
        }
        const int uV = 2 * i + 1;
        if (!wait_rot(uV)) goto mma_drain;
        if (!mbar_wait(p_full + (i & 1), (i >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
        tc_fence_after();
        issue_pv(i & 1, uV % C::NS, i > 0);
        umma_commit(o_done + (i & 1));
        umma_commit(kv_empty + uV % C::NS);
      }
    mma_drain:
      // every MMA issued above completes before tensor memory is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-15)
    // Warp w owns TMEM lanes 32*(w%4).. (32 query rows) and keys kq*32 .. kq*32+31 of every
    // tile, kq = w/4: one 32-column TMEM load per thread and tile. The four warps of a row
    // exchange their maxima through shared memory (an mbarrier per parity of the tile count
    // and lane quarter), all derive the same row reference, and each writes the P (bf16) of
    // its 32 keys to TMEM columns kq*16 .. kq*16+15 of the tile's S buffer; every S column of
    // those rows was read before the exchange, so P may overwrite any of them. O is rescaled (rarely) by column
    // quarter, once the previous tile's PV has completed.
    const int kq = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [parity][kq][128] row maxima
    float* lsum = red + 2 * 4 * 128;                            // [kq][128] row sums
    const float sc = a.scale_log2;
    const int i = qs + r;     // query row
    const int ip = qoff + i;  // the query's key index
    const float slope = p.alibi.on ? p.alibi.slope[h] * LOG2E : 0.f;
    // Row state in the log2 domain: m_ref is the reference the weights are taken against
    // (-inf until the row has seen an allowed key), l the running sum of this warp's share
    // of the weights. The reference moves only when a tile's maximum exceeds it by more than
    // 8 (a factor 256), so O is rescaled rarely; weights stay below 2^8.
    float m_ref = -INFINITY, l = 0.f;
    int c = 0;
    if (has) {
#pragma unroll 1
      for (int j = jt0; j <= jt1; ++j, ++c) {
        const int buf = c & 1;
        if (!mbar_wait(s_full + buf, (c >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + C::COL_S + buf * BN;
        const int key0 = j * BN + kq * 32;  // first of my 32 keys
        // does any row of this tile need per-element masking in my keys? (uniform per warp)
        const bool need_mask = (key0 + 32 > Tk) || (p.causal && key0 + 31 > qoff + qs) ||
                               (p.window > 0 && qoff + qs + BM - 1 - key0 >= p.window);
        float x[32];
        tmem_ld32(tS + kq * 32, x);
        tmem_wait_ld();
        if (p.alibi.on) {
          // -slope |i - j| is, with the causal mask, slope (j - i) on every allowed pair: an
          // affine function c0 + slope k of the key
          const float c0 = slope * (float)(key0 - ip);
#pragma unroll
          for (int k = 0; k < 32; ++k)
            x[k] = p.causal ? fmaf(x[k], sc, fmaf(slope, (float)k, c0))
                            : fmaf(x[k], sc, -slope * fabsf((float)(ip - key0 - k)));
        }
        if (need_mask) {
          // my keys allowed for this row: kmin <= k < kmax
          int kmax = Tk - key0;
          if (p.causal) kmax = min(kmax, ip - key0 + 1);
          const int kmin = p.window > 0 ? ip - p.window + 1 - key0 : 0;
#pragma unroll
          for (int k = 0; k < 32; ++k) x[k] = (k >= kmin && k < kmax) ? x[k] : -INFINITY;
        }
        // without ALiBi the scores are still unscaled: a positive scale keeps the order
        const float hx = p.alibi.on ? max32(x) : max32(x) * sc;
        float* rb = red + buf * 512;
        rb[kq * 128 + r] = hx;
        __syncwarp();
        if (lane == 0) mbar_arrive(red_bar + 4 * buf + (warp & 3));
        if (!mbar_wait(red_bar + 4 * buf + (warp & 3), (c >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
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
          up2(fma2(pk2(x[4 * k], x[4 * k + 1]), SC, NM), a0, a1);
          up2(fma2(pk2(x[4 * k + 2], x[4 * k + 3]), SC, NM), b0, b1);
          const float e0 = ex2(a0), e1 = ex2(a1), e2 = ex2(b0), e3 = ex2(b1);
          RS = add2(RS, add2(pk2(e0, e1), pk2(e2, e3)));
          pk[2 * k] = f2_to_bf2(e0, e1);
          pk[2 * k + 1] = f2_to_bf2(e2, e3);
        }
        tmem_st16u(tS + kq * 16, pk);
        // O is rescaled before this tile's PV is issued, once the previous PV has completed
        // (the tile before the previous one completed before this tile's QK)
        if (c > 0 && kq * 32 < HD && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!mbar_wait(o_done + ((c - 1) & 1), ((c - 1) >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
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
    }
    // ---- epilogue: out = O / l (bf16), lse = (m + log2 l) ln 2
    if (c == 0) {
      // a tile that attends no key at all (not a prefill's rows, which see their own key):
      // zero rows, lse -inf
      if (i < p.T) {
        if (kq * 32 < HD) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                (((size_t)b * p.T + i) * p.H + h) * HD + kq * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (p.lse && kq == 0) p.lse[((size_t)b * p.H + h) * p.T + i] = -INFINITY;
      }
    } else {
      // the row's total sum: the four warps' partial sums, exchanged through shared memory
      lsum[kq * 128 + r] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(lsum_bar);
      if (!mbar_wait(lsum_bar, 0, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
      const float lt = (lsum[r] + lsum[128 + r]) + (lsum[256 + r] + lsum[384 + r]);
      if (!mbar_wait(o_done + ((c - 1) & 1), ((c - 1) >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
      tc_fence_after();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      if (kq * 32 < HD) {
        float o[32];
        tmem_ld32(tmem + lane_off + C::COL_O + kq * 32, o);
        tmem_wait_ld();
        if (i < p.T) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                (((size_t)b * p.T + i) * p.H + h) * HD + kq * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(f2_to_bf2(o[8 * v4] * inv, o[8 * v4 + 1] * inv),
                                 f2_to_bf2(o[8 * v4 + 2] * inv, o[8 * v4 + 3] * inv),
                                 f2_to_bf2(o[8 * v4 + 4] * inv, o[8 * v4 + 5] * inv),
                                 f2_to_bf2(o[8 * v4 + 6] * inv, o[8 * v4 + 7] * inv));
        }
      }
      if (p.lse && i < p.T && kq == 0)
        p.lse[((size_t)b * p.H + h) * p.T + i] = lt > 0.f ? (m_ref + __log2f(lt)) * LN2 : -INFINITY;
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
cudaError_t launch_hd(const PrefillParams& p, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  if (p.seqlens) return cudaErrorInvalidValue;  // chunks run on the persistent kernel
  if (!make_map(&mq, p.q, p.B, p.T, p.H, HD) || !make_map(&mk, p.k, p.B, p.T, p.KV, HD) ||
      !make_map(&mv, p.v, p.B, p.T, p.KV, HD))
    return cudaErrorInvalidValue;
  TcArgs a;
  a.p = p;
  a.nqb = (p.T + BM - 1) / BM;
  a.scale_log2 = p.scale * LOG2E;
  const long long units = (long long)p.B * p.H * a.nqb;
  if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
  auto kern = prefill_tc_kernel<HD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<HD>::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)units, NUM_THREADS, Cfg<HD>::SMEM, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace
}  // namespace tc

bool prefill_tc_supported(const PrefillParams& p, int dtype) {
  return dtype == 1 && (p.hd == 64 || p.hd == 128) && tc::encode_fn() != nullptr;
}

cudaError_t launch_prefill_tc(const PrefillParams& p, cudaStream_t s) {
  // no key to turn in the kernel (keys turned before, no RoPE, or a chunk over the cache): the
  // persistent form, whose units' set-up and epilogues overlap their neighbours' key tiles
  if (prefill_ps_supported(p)) return launch_prefill_ps(p, s);
  // hd = 128 with the keys turned in the kernel: the two-slot kernel turns each key tile
  // once per 256 query rows instead of once per 128
  if (p.hd == 128 && p.rope.on && !p.seqlens && !p.k_rotated) return launch_prefill_pair(p, s);
  return p.hd == 128 ? tc::launch_hd<128>(p, s) : tc::launch_hd<64>(p, s);
}

}  // namespace attn
