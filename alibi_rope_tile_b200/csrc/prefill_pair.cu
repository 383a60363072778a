// Tensor-core flash prefill for sm_100a, the form for hd = 128 with keys turned in the
// kernel: two 128-row slots per CTA share every K/V tile, so each tile is fetched and turned
// once per 256 query rows (the single-slot kernel of prefill_tc.cu, which keeps Q in tensor
// memory, turns each tile once per 128 rows; when the keys arrive turned, or for hd = 64,
// that kernel is the faster one). TMA-staged tiles, tcgen05 MMAs accumulating in TMEM,
// warp-specialised online softmax, rotary embedding applied as tiles land.
//
// What it computes is the attention core of "Write attention from scratch" (worked
// example): per query row i, softmax over allowed keys j of
//   (R(pos0+i) q_i . R(pos0+j) k_j) / sqrt(hd) - slope_h |i - j|
// weighting the value rows, reached through the key-block recurrences of "Building
// grouped-query attention with RoPE and Flash Attention from scratch" (Step 3): a running
// maximum, a running denominator and a rescaled output accumulator.
//
// Work unit (one CTA): two "slots" of 128 query rows that read the same key/value head:
//   * H/KV even: two query heads of one group at the same rows (GQA sharing);
//   * H/KV odd (MHA included): one head, two consecutive 128-row tiles.
// Both slots consume every key/value tile the CTA loads, so each tile is fetched and
// rotated once per 256 query rows. CTAs are numbered longest-first (causal rows near the
// end see the most keys) so the block scheduler packs them like an LPT schedule.
//
// Warp roles (22 warps):
//   warps 0-15  softmax, one slot at a time (slot 0, then slot 1, for every key tile):
//               warp w owns 32 query rows (TMEM lanes 32*(w%4)..) and 32 keys of the tile
//               (keys 32*(w/4)..)
//   warps 16-19 rotary embedding: turns the two Q tiles once, then every K tile in place
//               in its 128-byte-swizzled shared-memory layout (RoPE on load)
//   warp 20     TMA producer (Q tiles, then K/V tiles through a ring of NS stages)
//   warp 21     TMEM allocation and UMMA issue
// Tensor memory (512 columns): S0 | S1 (128 fp32 columns each) | O0 | O1 (hd each).
// P (bf16, two per 32-bit column) goes over the first 64 columns of the slot's S region
// once every softmax warp has read its S columns (keys 2c, 2c+1 -> column c), and PV takes
// P straight from tensor memory (the A operand of the TS-form MMA): P never touches shared
// memory, which the SS-form QK MMAs, the TMA writes and the in-place key rotation already
// share (an M=128, N=128 SS MMA reads 8 KB of operands from shared memory). The next
// QK of a slot overwrites that slot's S/P columns; it is issued after the slot's PV, and
// the tensor core executes one CTA's MMAs in issue order, so P is read before it is
// overwritten. Issue order per key tile j: PV0(j), QK0(j+1), PV1(j), QK1(j+1): the tensor
// core works on one slot while the softmax warps work on the other.
//
// Masking: a pair outside the causal/window/length limits gets -inf before the row max,
// so its weight is exactly 0, and the sums' order depends only on the tile structure;
// a row's output never depends on the keys it may not see. Tiles outside a slot's key
// range are skipped entirely.
#include "prefill_common.cuh"

namespace attn {
namespace tc {
namespace pair {

constexpr int BM = PF_BM;
constexpr int BN = PF_BN;
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
  static constexpr int NS = HD == 128 ? 4 : 10;  // key/value ring stages
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int KV_BYTES = BN * HD * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
  static constexpr int NBAR = 3 * NS + 19;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // row-max exchange [parity][key quarter][128] and row-sum exchange [slot][key quarter][128]
  static constexpr int OFF_RED = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int RED_FLOATS = 2 * 4 * 128 + 2 * 4 * 128;
  static constexpr int SMEM = OFF_RED + RED_FLOATS * 4 + 1024;  // + slack to align the base
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, 0, 1);
};

struct TcArgs {
  PrefillParams p;
  int group;       // H / KV
  int two_heads;   // 1: slots are two heads at the same rows; 0: one head, two row tiles
  int npairs;      // slot pairs per key/value head
  int nqb;         // query blocks per (sequence, pair)
  float scale_log2;
};

template <int HD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
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
  uint64_t* q_rot = q_full + 1;
  uint64_t* s_full = q_full + 2;
  uint64_t* p_full = q_full + 4;
  uint64_t* o_done = q_full + 6;
  uint64_t* drain = q_full + 8;  // the MMA thread's final commit
  uint64_t* red_bar = q_full + 9;    // [parity of the slot-tile count][lane quarter]: the four
                                     // warps of those rows wrote their maxima
  uint64_t* lsum_bar = q_full + 17;  // [slot]: all warps' row sums written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const PrefillParams& p = a.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work unit: longest rows first
  const int per_qb = p.B * p.KV * a.npairs;
  const int qb = a.nqb - 1 - (int)(blockIdx.x / per_qb);
  int rest = blockIdx.x % per_qb;
  const int pair = rest % a.npairs;
  rest /= a.npairs;
  const int g = rest % p.KV;
  const int b = rest / p.KV;
  int head[2], qs[2];
  if (a.two_heads) {
    head[0] = g * a.group + 2 * pair;
    head[1] = head[0] + 1;
    qs[0] = qs[1] = qb * BM;
  } else {
    head[0] = head[1] = g * a.group + pair;
    qs[0] = qb * 2 * BM;
    qs[1] = qs[0] + BM;
  }
  // Key j is row j of k/v: qoff is the key index of query row 0, Tk the number of keys.
  const int qoff = 0, Tk = p.T, qrope0 = p.pos0;
  int t0[2], t1[2];
  bool valid[2], has[2];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    valid[s] = qs[s] < p.T;
    const int lo = p.window > 0 ? max(0, qoff + qs[s] - p.window + 1) : 0;
    const int hi = p.causal ? min(Tk - 1, qoff + qs[s] + BM - 1) : Tk - 1;
    has[s] = valid[s] && lo <= hi;  // the slot attends at least one key
    t0[s] = has[s] ? lo / BN : 1;
    t1[s] = has[s] ? hi / BN : 0;
  }
  const int jt0 = has[0] ? (has[1] ? min(t0[0], t0[1]) : t0[0]) : t0[1];
  const int jt1 = has[0] ? (has[1] ? max(t1[0], t1[1]) : t1[0]) : t1[1];
  auto active = [&](int s, int j) { return has[s] && j >= t0[s] && j <= t1[s]; };

  // ---- set-up: barriers, tensor memory
  if (tid == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
      mbar_init(k_rot + i, 128);
    }
    mbar_init(q_full, 1);
    mbar_init(q_rot, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_full + s, 16);  // one arrival per softmax warp
      for (int qq = 0; qq < 4; ++qq) mbar_init(red_bar + 4 * s + qq, 4);
      mbar_init(lsum_bar + s, 16);
      mbar_init(o_done + s, 1);
    }
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
      const uint32_t qbytes = (valid[0] ? C::Q_BYTES : 0) + (valid[1] ? C::Q_BYTES : 0);
      mbar_expect_tx(q_full, qbytes);
      for (int s = 0; s < 2; ++s)
        if (valid[s])
          for (int kb = 0; kb < HD / 64; ++kb)
            tma_load_4d(sQ + s * C::Q_BYTES + kb * BM * 128, &tmQ, q_full, kb * 64, head[s], qs[s], b);
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
    const int r = tid - WARP_ROPE0 * 32;  // row of a query tile this thread turns
    KRot<HD> krot;
    if (p.rope.on) krot.init(r, p.rope);
    if (!mbar_wait(q_full, 0, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
    if (p.rope.on)
      for (int s = 0; s < 2; ++s)
        if (valid[s]) krot.rotate(sQ + s * C::Q_BYTES, qrope0 + qs[s], p.rope);
    fence_proxy_async();
    mbar_arrive(q_rot);
    // hd = 128: key-tile start angles by recurrence; hd = 64 (half the rotation work per
    // tile, and registers are tighter) computes each accurately
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
      // Descriptors are built once; the start-address field (bits 0-13, in 16-byte
      // units) is then advanced by plain additions that stay below 2^14.
      const uint64_t dQ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sKV), BN * 128, 1024);
      auto issue_qk = [&](int s, int st) {
        const uint32_t d = tmem + s * BN;
        const uint64_t a0 = dQ + (uint64_t)((s * C::Q_BYTES) >> 4);
        const uint64_t b0 = dK + (uint64_t)((st * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4;
          umma_ss(d, a0 + off, b0 + off, C::IDESC_QK, kk > 0);
        }
      };
      auto issue_pv = [&](int s, int st, bool acc) {
        const uint32_t d = tmem + 2 * BN + s * HD;
        const uint32_t aP = tmem + s * BN;  // P: 64 columns of bf16 pairs over the first half of S
        const uint64_t b0 = dV + (uint64_t)((st * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          umma_ts(d, aP + kk * 8, b0 + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV,
                  (kk > 0 || acc) ? 1u : 0u);
        }
      };
      int cnt[2] = {0, 0};
      if (!mbar_wait(q_rot, 0, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
      if (jt1 < jt0) goto mma_drain;  // no key tile at all
      // K of the first tile
      if (!mbar_wait(k_rot + 0, 0, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
      tc_fence_after();
      for (int s = 0; s < 2; ++s)
        if (active(s, jt0)) {
          issue_qk(s, 0);
          umma_commit(s_full + s);
        }
      umma_commit(kv_empty + 0);
      for (int j = jt0; j <= jt1; ++j) {
        const int uV = 2 * (j - jt0) + 1, stV = uV % C::NS;
        const int uK = uV + 1, stK = uK % C::NS;
        const bool next = j < jt1;
        if (!mbar_wait(k_rot + stV, (uV / C::NS) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
        for (int s = 0; s < 2; ++s) {
          if (active(s, j)) {
            if (!mbar_wait(p_full + s, cnt[s] & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
            tc_fence_after();
            issue_pv(s, stV, cnt[s] > 0);
            umma_commit(o_done + s);
            ++cnt[s];
          }
          if (next && s == 0) {
            if (!mbar_wait(k_rot + stK, (uK / C::NS) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto mma_drain;
            tc_fence_after();
          }
          if (next && active(s, j + 1)) {
            issue_qk(s, stK);
            umma_commit(s_full + s);
          }
        }
        umma_commit(kv_empty + stV);
        if (next) umma_commit(kv_empty + stK);
      }
    mma_drain:
      // every MMA issued above completes before tensor memory is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-15)
    // All sixteen warps work on one slot at a time, slot 0 then slot 1 for every key tile, so
    // the tensor core runs one slot's PV and next QK while the other slot's weights are
    // formed. Warp w owns TMEM lanes 32*(w%4).. (32 query rows) and keys kq*32 .. kq*32+31 of
    // the tile, kq = w/4: one 32-column TMEM load per thread per slot and tile. The four
    // warps of a row exchange their maxima through shared memory (an mbarrier per parity of
    // the slot-tile count and lane quarter), all derive the same row reference, and each writes the P (bf16)
    // of its 32 keys to TMEM columns kq*16 .. kq*16+15 of the slot's S region; every S column
    // was read before the exchange, so P may overwrite any of them. O is rescaled (rarely)
    // by column quarter.
    const int kq = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [parity][kq][128] row maxima
    float* lsum = red + 2 * 4 * 128;                            // [slot][kq][128] row sums
    const float sc = a.scale_log2;
    // Row state per slot in the log2 domain: m_ref is the reference the weights are taken
    // against (-inf until the row has seen an allowed key), l the running sum of this warp's
    // share of the weights. The reference moves only when a tile's maximum exceeds it by
    // more than 8 (a factor 256), so O is rescaled rarely; weights stay below 2^8.
    float m_ref0 = -INFINITY, m_ref1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    int cs0 = 0, cs1 = 0, t = 0;
#pragma unroll 1
    for (int j = jt0; j <= jt1; ++j) {
#pragma unroll 1
      for (int s = 0; s < 2; ++s) {
        if (!active(s, j)) continue;
        // this slot's row state (scalars selected by slot: no indexed local arrays)
        const int c = s ? cs1 : cs0;
        float m_ref = s ? m_ref1 : m_ref0;
        if (!mbar_wait(s_full + s, c & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
        tc_fence_after();
        const int q0s = qs[s];  // first query row of the slot
        const int hs = head[s];
        const int i = q0s + r;
        const int ip = qoff + i;  // the query's key index
        const uint32_t tS = tmem + lane_off + s * BN;
        const int key0 = j * BN + kq * 32;  // first of my 32 keys
        const float slope = p.alibi.on ? p.alibi.slope[hs] * LOG2E : 0.f;
        // does any row of this slot need per-element masking in my keys of this tile?
        const bool need_mask = (key0 + 32 > Tk) || (p.causal && key0 + 31 > qoff + q0s) ||
                               (p.window > 0 && qoff + q0s + BM - 1 - key0 >= p.window);
        const bool plain = !need_mask && !p.alibi.on;
        float x[32];
        tmem_ld32(tS + kq * 32, x);
        tmem_wait_ld();
        float hx = -INFINITY;
        if (plain) {
          hx = max32(x) * sc;  // a positive scale keeps the order: max then scale is exact
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int jk = key0 + k;
            float v = p.alibi.on ? fmaf(x[k], sc, -slope * fabsf((float)(ip - jk))) : x[k] * sc;
            if (need_mask) {
              const bool ok = jk < Tk && (!p.causal || jk <= ip) && (p.window <= 0 || ip - jk < p.window);
              v = ok ? v : -INFINITY;
            }
            x[k] = v;
          }
          hx = max32(x);
        }
        float* rb = red + (t & 1) * 512;
        rb[kq * 128 + r] = hx;
        __syncwarp();
        if (lane == 0) mbar_arrive(red_bar + 4 * (t & 1) + (warp & 3));
        if (!mbar_wait(red_bar + 4 * (t & 1) + (warp & 3), (t >> 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS))
          goto done;
        const float mt = fmaxf(fmaxf(rb[r], rb[128 + r]), fmaxf(rb[256 + r], rb[384 + r]));
        const float m_new = (mt > m_ref + 8.f) ? mt : m_ref;  // takes mt when m_ref = -inf
        const float alpha = (m_new == m_ref) ? 1.f : ex2(m_ref - m_new);
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        m_ref = m_new;
        f2x RS = pk2(0.f, 0.f);
        uint32_t pk[16];  // column k: keys 2k, 2k+1 of my 32 (low half = even key)
        if (plain) {
          const f2x SC = pk2(sc, sc), NM = pk2(-mu, -mu);
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
        } else {
          const f2x NM = pk2(-mu, -mu);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float a0, a1, b0, b1;
            up2(add2(pk2(x[4 * k], x[4 * k + 1]), NM), a0, a1);
            up2(add2(pk2(x[4 * k + 2], x[4 * k + 3]), NM), b0, b1);
            const float e0 = ex2(a0), e1 = ex2(a1), e2 = ex2(b0), e3 = ex2(b1);
            RS = add2(RS, add2(pk2(e0, e1), pk2(e2, e3)));
            pk[2 * k] = f2_to_bf2(e0, e1);
            pk[2 * k + 1] = f2_to_bf2(e2, e3);
          }
        }
        tmem_st16u(tS + kq * 16, pk);
        float rs;
        {
          float r0, r1;
          up2(RS, r0, r1);
          rs = r0 + r1;
        }
        // O is rescaled before this tile's PV is issued. The previous PV of this slot has
        // completed: it was issued before the QK whose completion this tile waited for.
        if (c > 0 && kq * 32 < HD && __any_sync(0xffffffffu, alpha != 1.f)) {
          const uint32_t tO = tmem + lane_off + 2 * BN + s * HD + kq * 32;
          float o[32];
          tmem_ld32(tO, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tO, o);
        }
        if (s) {
          l1 = l1 * alpha + rs;
          m_ref1 = m_ref;
          cs1 = c + 1;
        } else {
          l0 = l0 * alpha + rs;
          m_ref0 = m_ref;
          cs0 = c + 1;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + s);
        ++t;
      }
    }
#pragma unroll 1
    for (int s = 0; s < 2; ++s) {
      const int c = s ? cs1 : cs0;
      if (c == 0) {
        // a slot that attends no key at all (not a prefill's rows, which see their own key):
        // zero rows, lse -inf
        const int i = qs[s] + r;
        if (valid[s] && i < p.T) {
          if (kq * 32 < HD) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                  (((size_t)b * p.T + i) * p.H + head[s]) * HD + kq * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
          }
          if (p.lse && kq == 0) p.lse[((size_t)b * p.H + head[s]) * p.T + i] = -INFINITY;
        }
        continue;
      }
      const float m_ref = s ? m_ref1 : m_ref0;
      // the row's total sum: the four warps' partial sums, exchanged through shared memory
      lsum[(s * 4 + kq) * 128 + r] = s ? l1 : l0;
      __syncwarp();
      if (lane == 0) mbar_arrive(lsum_bar + s);
      if (!mbar_wait(lsum_bar + s, 0, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
      const float* ls = lsum + s * 4 * 128 + r;
      const float lt = (ls[0] + ls[128]) + (ls[256] + ls[384]);
      if (!mbar_wait(o_done + s, (c - 1) & 1, abort_flag, p.status, WAIT_LIMIT_NS)) goto done;
      tc_fence_after();
      const int hs = head[s];
      const int i = qs[s] + r;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      if (kq * 32 < HD) {
        float o[32];
        tmem_ld32(tmem + lane_off + 2 * BN + s * HD + kq * 32, o);
        tmem_wait_ld();
        if (i < p.T) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                (((size_t)b * p.T + i) * p.H + hs) * HD + kq * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(f2_to_bf2(o[8 * v4] * inv, o[8 * v4 + 1] * inv),
                                 f2_to_bf2(o[8 * v4 + 2] * inv, o[8 * v4 + 3] * inv),
                                 f2_to_bf2(o[8 * v4 + 4] * inv, o[8 * v4 + 5] * inv),
                                 f2_to_bf2(o[8 * v4 + 6] * inv, o[8 * v4 + 7] * inv));
        }
      }
      if (p.lse && i < p.T && kq == 0)
        p.lse[((size_t)b * p.H + hs) * p.T + i] = lt > 0.f ? (m_ref + __log2f(lt)) * LN2 : -INFINITY;
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
  if (!make_map(&mq, p.q, p.B, p.T, p.H, HD) || !make_map(&mk, p.k, p.B, p.T, p.KV, HD) ||
      !make_map(&mv, p.v, p.B, p.T, p.KV, HD))
    return cudaErrorInvalidValue;
  TcArgs a;
  a.p = p;
  a.group = p.H / p.KV;
  a.two_heads = (a.group % 2 == 0) ? 1 : 0;
  a.npairs = a.two_heads ? a.group / 2 : a.group;
  const int rows = a.two_heads ? BM : 2 * BM;
  a.nqb = (p.T + rows - 1) / rows;
  a.scale_log2 = p.scale * LOG2E;
  const long long units = (long long)p.B * p.KV * a.npairs * a.nqb;
  if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
  auto kern = prefill_pair_kernel<HD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<HD>::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)units, NUM_THREADS, Cfg<HD>::SMEM, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace pair
}  // namespace tc

cudaError_t launch_prefill_pair(const PrefillParams& p, cudaStream_t s) {
  if (p.hd != 128 || p.seqlens) return cudaErrorInvalidValue;  // not a case this form serves
  return tc::pair::launch_hd<128>(p, s);
}

}  // namespace attn
