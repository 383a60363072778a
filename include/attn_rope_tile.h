/*
 * attn_rope_tile.h -- C ABI of the B200 (sm_100a) attention core.
 *
 * The library computes the attention core of a decoder self-attention block,
 *     out = softmax(Q K^T / sqrt(hd) + bias, masked) V,
 * with grouped-query head sharing, interleaved rotary embeddings applied as the Q/K
 * tiles are loaded, a causal mask with an optional sliding window, an optional ALiBi
 * bias, a KV-cache decode step, and the projections of the surrounding block.
 *
 * Sources of the definitions (page title, then the place on the page):
 *   [LAB]   "Write attention from scratch" (Inside the Model, lab 2): the worked
 *           example (rope, softmax, attention), Properties 1 and 2, exercises 2-4.
 *   [ALIBI] "Building a Multi-Head Self-Attention Block with RoPE and ALiBi from
 *           Scratch": Step 1 (slopes), Step 3 "Implement ALiBi Bias", Step 4.
 *   [FLASH] "Building grouped-query attention with RoPE and Flash Attention from
 *           scratch": Step 3 (tiled online-softmax forward), roadmap (sliding window,
 *           causal mask with KV cache, bf16 inputs with fp32 statistics).
 *   [XF5]   "Building a Transformer from Scratch: Attention, Architecture, and Memory":
 *           Part 1 step 2 (causal mask), Part 3 "KV caching", "FlashAttention" equations.
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, contiguous, caller-owned DEVICE buffers unless a
 *     parameter says "host". The library never allocates device memory, frees or keeps a
 *     pointer after a call returns (attn_prefill_host keeps two copy streams per device).
 *   - Layouts: q and out [B, T, H, hd]; k and v [B, T, KV, hd]; decode q/out [B, H, hd];
 *     caches [B, Lmax, KV, hd]; lse (log-sum-exp of each softmax row, natural log, fp32)
 *     [B, H, T] for prefill and [B, H] for decode.
 *   - dtype selects the element type of q, k, v, out, caches, x and weights (all the
 *     same). Arithmetic is fp32 for either type; bf16 results are rounded to nearest
 *     even. Statistics (running max and sum) are always fp32.
 *   - Query head h reads key/value head h / (H / KV) ([LAB] np.repeat; [FLASH]).
 *   - RoPE: rope_base > 0 turns interleaved pairs (2i, 2i+1) of q and k by the angle
 *     p * rope_base^(-2i/hd) at position p ([LAB] rope). rope_base <= 0: no rotation.
 *     Prefill positions are pos0 .. pos0+T-1; pos0 + T must stay below 2^24.
 *   - Masks: causal keeps key j <= i ([LAB], [XF5]); window > 0 also requires
 *     i - j < window (a window of W keys including the query's own) ([FLASH] roadmap,
 *     [LAB] exercise 3). A masked pair has weight exactly zero.
 *   - ALiBi: alibi_slopes (HOST pointer to H floats, copied at launch) adds
 *     -slope_h * |i - j| to the scaled score ([ALIBI] Step 3); NULL turns it off.
 *     attn_alibi_slopes() fills the schedule 2^(-8(h+1)/H).
 *   - stream is a cudaStream_t (NULL: the legacy default stream). Calls are
 *     asynchronous; the return value covers argument checks and launch errors. Errors
 *     found on the device (an out-of-range cache position, a wait that gave up) are
 *     recorded in a per-device error word read by attn_sync_status().
 *   - Every call returns ATTN_OK (0) or a negative attn_status; attn_last_error() gives
 *     a one-line message for the calling thread's last failure. Nothing aborts.
 *   - Pointers must be 16-byte aligned; hd must be even and at most 256.
 */
#ifndef ATTN_ROPE_TILE_H
#define ATTN_ROPE_TILE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_F32 = 0,   /* IEEE fp32 elements */
  ATTN_BF16 = 1   /* bfloat16 elements */
} attn_dtype;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_ARG = -1,          /* a size, flag or pointer is invalid */
  ATTN_ERR_ALIGN = -2,        /* a pointer is not 16-byte aligned */
  ATTN_ERR_UNSUPPORTED = -3,  /* a valid request the library does not implement */
  ATTN_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed */
  ATTN_ERR_TIMEOUT = -5,      /* a device-side wait gave up (reported by attn_sync_status) */
  ATTN_ERR_WORKSPACE = -6,    /* workspace missing or smaller than the size query returned */
  ATTN_ERR_DEVICE_ARG = -7    /* a device-resident argument was out of range (attn_sync_status) */
} attn_status;

/*
 * attn_prefill -- causal (or full) attention of T query rows over the same T keys.
 *
 * Computes, for every batch b, query head h and row i, the softmax-weighted sum of the
 * value rows of head g = h / (H/KV) over the allowed keys j ([LAB] attention(); the
 * tiled online-softmax route of [FLASH] Step 3 reaches the same result):
 *   s_ij = (R(pos0+i) q_i) . (R(pos0+j) k_j) / sqrt(hd) - slope_h |i - j|
 *   out_i = sum_j softmax_j(s_ij) v_j,   lse_i = log sum_j exp(s_ij)
 * q, k, v: inputs (device, read only). out: [B,T,H,hd] (device, written).
 * lse: [B,H,T] fp32 (device, written) or NULL. B, T >= 1; H % KV == 0.
 * causal: 0 or 1. window: <= 0 none, else W >= 1 (requires causal).
 * bf16 with hd in {64, 128} runs the tensor-core (tcgen05/TMEM) kernel; other shapes
 * and fp32 run the CUDA-core kernel. Returns ATTN_OK or an attn_status.
 * The keys are turned inside the attention kernel as its tiles land (every CTA that reads
 * a key tile turns it); attn_prefill_ws turns them once in a pass of their own instead.
 */
int attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse,
                 int B, int T, int H, int KV, int hd, long long pos0, float rope_base,
                 int causal, int window, const float* alibi_slopes, int dtype, void* stream);

/*
 * attn_prefill_workspace_size -- bytes of device scratch attn_prefill_ws uses to hold the
 * turned keys: B*T*KV*hd*2 for bf16 with hd in {64, 128} and rope_base > 0 (where a
 * separate key rotation pass is faster than turning each key tile in every CTA that reads
 * it), else 0. Returns 0 on invalid sizes.
 */
size_t attn_prefill_workspace_size(int B, int T, int KV, int hd, float rope_base, int dtype);

/*
 * attn_prefill_ws -- attn_prefill with caller-owned scratch ([LAB] rope: turning a key
 * depends only on its own position, so it may be done once, before the attention).
 *
 * Arguments and results are those of attn_prefill, plus workspace: NULL (ws_bytes 0), or
 * 16-byte aligned device memory of at least attn_prefill_workspace_size(B,T,KV,hd,
 * rope_base,dtype) bytes, owned by the caller, contents on entry irrelevant. When that
 * size is non-zero and the workspace is given, two kernels run on stream: the rotation pass
 * writes k turned at positions pos0+j into the workspace (fp32 arithmetic, rounded once to
 * bf16), then the persistent attention kernel reads the keys from there (it may start while
 * the pass finishes, and reads no key before the pass has completed). Otherwise (size 0 or
 * workspace NULL) this is attn_prefill. A non-NULL workspace smaller than the size query
 * returns ATTN_ERR_WORKSPACE; a misaligned one ATTN_ERR_ALIGN.
 */
int attn_prefill_ws(const void* q, const void* k, const void* v, void* out, float* lse,
                    int B, int T, int H, int KV, int hd, long long pos0, float rope_base,
                    int causal, int window, const float* alibi_slopes, int dtype, void* workspace,
                    size_t ws_bytes, void* stream);

/*
 * attn_prefill_host_workspace_size -- bytes of device scratch attn_prefill_host needs: dense
 * device copies of q, k, v, out (and lse) cut into its slices, and the rotation pass's
 * scratch for one slice. Returns 0 on invalid sizes.
 */
size_t attn_prefill_host_workspace_size(int B, int T, int H, int KV, int hd, float rope_base, int dtype);

/*
 * attn_prefill_host -- attn_prefill_ws on q, k, v and results in HOST memory ([LAB]
 * attention(): every (sequence, query head) reads only its own key/value head, so the problem
 * splits into independent slices).
 *
 * q, k, v: [B,T,H,hd] / [B,T,KV,hd] host buffers (read); out: [B,T,H,hd] host buffer
 * (written); lse: [B,H,T] fp32 host buffer or NULL. Page-locked (pinned) host memory lets the
 * copies run asynchronously and overlap; pageable memory gives the same results without the
 * overlap. workspace: 256-byte aligned device memory of at least
 * attn_prefill_host_workspace_size(...) bytes, owned by the caller; it must not be in use by
 * work that the call does not follow on `stream`. The other arguments are attn_prefill's.
 * The call cuts the problem into slices: runs of whole sequences when B >= 4, else one
 * sequence and a group of key/value heads with their query heads; the last slice is cut
 * finer (halving groups of key/value heads), as its attention and copy back are what remains
 * once every slice's rows have landed. It copies each slice's rows
 * into the workspace on a copy stream of its own, runs the prefill of attn_prefill_ws on
 * `stream` as soon as the slice has landed, and copies the slice's results back on a second
 * copy stream, so copies in, attention and copies out of different slices overlap; every
 * output row is computed exactly as by attn_prefill_ws over the whole tensors on the device.
 * Asynchronous: work issued on `stream` after the call (a synchronisation included) sees out
 * and lse in host memory. The copy streams and their events are created on the first call on a
 * device and kept for the process. Returns ATTN_OK or an attn_status (ATTN_ERR_WORKSPACE for
 * a missing or short workspace, ATTN_ERR_ALIGN for a misaligned one).
 */
int attn_prefill_host(const void* q, const void* k, const void* v, void* out, float* lse,
                      int B, int T, int H, int KV, int hd, long long pos0, float rope_base,
                      int causal, int window, const float* alibi_slopes, int dtype, void* workspace,
                      size_t ws_bytes, void* stream);

/*
 * attn_prefill_chunk -- a chunk of Tq query rows that continues sequences held in a KV
 * cache ([XF5] "KV caching"; [LAB] exercise 2 with several new tokens at once): the step
 * between a prefill and a decode, for prompts processed in pieces.
 *
 * q: [B,Tq,H,hd] BEFORE rotation; row i of sequence b sits at position qpos0[b] + i and is
 * turned there. kcache, vcache: [B,Lmax,KV,hd]; slot j holds the key already rotated at
 * position j (attn_kv_write / attn_kv_append write it that way; write the chunk's own keys
 * first, so that it attends to itself). Row i attends slots j < seqlens[b] with, when
 * causal, j <= qpos0[b] + i and, with window W > 0, qpos0[b] + i - j < W; ALiBi adds
 * -slope_h |qpos0[b] + i - j|. seqlens, qpos0: [B] int32 (device). A row with no allowed
 * slot gets out = 0, lse = -inf. out: [B,Tq,H,hd] (device, written); lse: [B,H,Tq] or NULL.
 * seqlens[b] > Lmax, qpos0[b] < 0 or qpos0[b] + Tq > 2^24 is recorded as
 * ATTN_ERR_DEVICE_ARG (attn_sync_status) and that sequence's rows are zeroed.
 * Runs the tensor-core prefill kernel: bf16 with hd in {64, 128}; anything else returns
 * ATTN_ERR_UNSUPPORTED.
 */
int attn_prefill_chunk(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                       const int* qpos0, void* out, float* lse, int B, int Tq, int H, int KV, int hd,
                       int Lmax, float rope_base, int causal, int window, const float* alibi_slopes,
                       int dtype, void* stream);

/*
 * attn_decode_workspace_size -- bytes of device scratch attn_decode needs for these
 * sizes (partial outputs of runs of key tiles, their softmax statistics, the tile counts of
 * the (sequence, key/value head) units). Returns 0 on invalid sizes.
 */
size_t attn_decode_workspace_size(int B, int H, int KV, int hd, int Lmax);

/*
 * attn_decode -- one decode step per sequence over a KV cache ([XF5] "KV caching";
 * [LAB] exercise 2: token-by-token decode equals the full causal computation).
 *
 * q: [B,H,hd] new-token queries BEFORE rotation; the kernel turns query b at position
 * qpos[b]. kcache, vcache: [B,Lmax,KV,hd]; slot j holds the key already rotated at
 * position j (attn_kv_append writes it that way). seqlens: [B] int32 (device): the
 * query attends to slots 0..seqlens[b]-1; window > 0 also requires qpos - j < window.
 * qpos: [B] int32 (device). A sequence with seqlens[b] == 0 gets out = 0, lse = -inf.
 * out: [B,H,hd] (device, written). lse: [B,H] fp32 or NULL.
 * workspace: device scratch of at least attn_decode_workspace_size(B,H,KV,hd,Lmax)
 * bytes, owned by the caller; its contents on entry do not matter.
 * seqlens[b] > Lmax or qpos[b] < 0 is recorded as ATTN_ERR_DEVICE_ARG (read it with
 * attn_sync_status) and that sequence's output is zeroed.
 * Two kernels run on stream (bf16, hd 64 or 128, H/KV <= 32): the tensor-core pass, whose
 * CTAs (two per SM) take equal runs of all sequences' 128-key tiles and serve every query
 * head of a key/value head from each tile they read once, then a log-sum-exp merge of the
 * runs; with more than 1024 (sequence, key/value head) units a one-CTA kernel counts their
 * tiles first. Other types and head sizes: a CUDA-core split pass (16-byte loads, fixed
 * splits of 2048 keys) and the same merge rule.
 */
int attn_decode(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                const int* qpos, void* out, float* lse, int B, int H, int KV, int hd, int Lmax,
                float rope_base, int window, const float* alibi_slopes, int dtype,
                void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device memory.
 *
 * There is no counterpart to this entry point on the pages; it exists for callers that
 * must not call cudaMalloc (or any allocating library routine) and cannot hand over a
 * workspace: code running under an allocator or memory budget that it does not own (a
 * plugin inside another framework's memory pool), or a latency-critical step where an
 * allocation, which may synchronise the device, is not allowed.
 *
 * Arguments and results are those of attn_decode without workspace/ws_bytes. The
 * partials live in a fixed scratch array of ATTN_DECODE_NOALLOC_MAX_SCRATCH bytes that is
 * part of the library's device image: every GPU that loads the library holds it until the
 * process exits. Sizes whose attn_decode_workspace_size() exceeds that maximum are
 * rejected with ATTN_ERR_UNSUPPORTED and a message naming the limit; nothing is launched.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * once per device, with that device current); make that first call before any stream
 * capture. Every call on a device shares the one array and leaves its contents behind:
 * nothing in it needs to start at zero, but two calls that overlap on the GPU (different
 * streams without ordering between them) race on it and may return wrong results.
 * The entry point allocates nothing.
 */
#define ATTN_DECODE_NOALLOC_MAX_SCRATCH ((size_t)8 << 20)
int attn_decode_noalloc(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                        const int* qpos, void* out, float* lse, int B, int H, int KV, int hd,
                        int Lmax, float rope_base, int window, const float* alibi_slopes,
                        int dtype, void* stream);

/*
 * attn_kv_append -- write one new token per sequence into the cache ([XF5] "KV caching";
 * [FLASH] roadmap: preallocate the cache and write by position).
 * k_new, v_new: [B,KV,hd] (device). pos: [B] int32 (device) slot = position of the token.
 * The key is rotated at pos[b] (if rope_base > 0) before it is stored; the value is
 * stored as is. pos[b] outside [0, Lmax) is recorded as ATTN_ERR_DEVICE_ARG and skipped.
 */
int attn_kv_append(const void* k_new, const void* v_new, void* kcache, void* vcache,
                   const int* pos, int B, int KV, int hd, int Lmax, float rope_base, int dtype,
                   void* stream);

/*
 * attn_kv_write -- write a chunk of Tn tokens per sequence into the cache (the multi-token
 * form of attn_kv_append, for attn_prefill_chunk): row t of sequence b goes to slot
 * pos0[b] + t, its key rotated at that position (if rope_base > 0), its value as is.
 * k_new, v_new: [B,Tn,KV,hd] (device). pos0: [B] int32 (device). 1 <= Tn <= 65535.
 * A slot outside [0, Lmax) is recorded as ATTN_ERR_DEVICE_ARG and that row is skipped.
 */
int attn_kv_write(const void* k_new, const void* v_new, void* kcache, void* vcache, const int* pos0,
                  int B, int Tn, int KV, int hd, int Lmax, float rope_base, int dtype, void* stream);

/*
 * attn_decode_paged -- attn_decode over a paged KV cache (the block-table layout of the
 * PagedAttention the pages mention for serving): the caches are page pools
 * kpages, vpages [num_pages, page_size, KV, hd]; slot j of sequence b is row j % page_size
 * of page block_table[b * max_blocks + j / page_size] (block_table: [B, max_blocks] int32,
 * device). page_size in {8, 16, 32, 64, 128}; seqlens[b] <= max_blocks * page_size. Entries
 * the sequence does not reach are not read. A table entry outside [0, num_pages) is
 * recorded as ATTN_ERR_DEVICE_ARG and its page reads as zeros. Everything else (q rotated
 * at qpos[b], window, ALiBi, outputs, workspace = attn_decode_workspace_size(B, H, KV, hd,
 * max_blocks * page_size)) is as attn_decode. Runs the tensor-core pass: bf16, hd 64 or 128,
 * H/KV <= 32; anything else returns ATTN_ERR_UNSUPPORTED.
 */
int attn_decode_paged(const void* q, const void* kpages, const void* vpages, const int* block_table,
                      const int* seqlens, const int* qpos, void* out, float* lse, int B, int H, int KV,
                      int hd, int page_size, int num_pages, int max_blocks, float rope_base, int window,
                      const float* alibi_slopes, int dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_decode_latent -- one decode step of latent attention ([LAB] exercise 5): every cached
 * token holds a latent c_j of dc numbers, and query head h's key and value are c_j W_uk[h]
 * and c_j W_uv[h] (W_uk, W_uv: [H, dc, hd] bf16, device). The key up-projection is folded
 * into the query (q'_h = W_uk[h] q_h), the decode runs over the latents themselves as one
 * key/value head of dimension dc (score q'_h . c_j / sqrt(hd)), and the value up-projection
 * is applied once to the weighted latent sum: the result equals attention over the
 * up-projected keys and values. No rotary embedding on this path (a position rotation
 * between c and W_uk does not fold into the query); window and ALiBi as attn_decode.
 * q: [B,H,hd]; ccache: [B,Lmax,dc] (device); out: [B,H,hd]; lse: [B,H] or NULL.
 * workspace: attn_decode_latent_workspace_size(B,H,hd,dc,Lmax) bytes (device, caller-owned).
 * bf16 with dc in {64, 128}, H <= 32 and hd a multiple of 8; anything else returns
 * ATTN_ERR_UNSUPPORTED. Three launches: the fold, the tensor-core pass over the latent cache
 * (one fetch of each latent tile serves as both key and value), and the merge of its runs with
 * the value up-projection.
 */
size_t attn_decode_latent_workspace_size(int B, int H, int hd, int dc, int Lmax);
int attn_decode_latent(const void* q, const void* ccache, const void* W_uk, const void* W_uv,
                       const int* seqlens, const int* qpos, void* out, float* lse, int B, int H, int hd,
                       int dc, int Lmax, int window, const float* alibi_slopes, int dtype, void* workspace,
                       size_t ws_bytes, void* stream);

/*
 * attn_kv_write_paged -- attn_kv_write into page pools: row t of sequence b goes to slot
 * pos0[b] + t, i.e. row (pos0[b] + t) % page_size of page block_table[b * max_blocks +
 * (pos0[b] + t) / page_size], its key rotated at that position. A slot past
 * max_blocks * page_size or a table entry outside [0, num_pages) is recorded as
 * ATTN_ERR_DEVICE_ARG and that row is skipped.
 */
int attn_kv_write_paged(const void* k_new, const void* v_new, void* kpages, void* vpages,
                        const int* block_table, const int* pos0, int B, int Tn, int KV, int hd,
                        int page_size, int num_pages, int max_blocks, float rope_base, int dtype,
                        void* stream);

/*
 * attn_block_workspace_size -- bytes of device scratch attn_block needs (the q, k, v and
 * context activations). Returns 0 on invalid sizes.
 */
size_t attn_block_workspace_size(int B, int T, int d, int H, int KV, int hd, int dtype);

/*
 * attn_block -- the attention block of [LAB] attention(): q = x Wq, k = x Wk, v = x Wv
 * (weights [in, out], applied as x @ W; head h is columns h*hd..h*hd+hd-1), then
 * attn_prefill on them, then out = ctx Wo. No bias, residual or normalisation.
 * x: [B,T,d]; Wq: [d, H*hd]; Wk, Wv: [d, KV*hd]; Wo: [H*hd, d]; out: [B,T,d].
 * workspace: at least attn_block_workspace_size(...) bytes (device, caller-owned).
 * Intermediate activations are stored in dtype.
 */
int attn_block(const void* x, const void* Wq, const void* Wk, const void* Wv, const void* Wo,
               void* out, int B, int T, int d, int H, int KV, int hd, long long pos0,
               float rope_base, int causal, int window, const float* alibi_slopes, int dtype,
               void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_fold_rmsnorm_gamma -- Wg[k][n] = gamma[k] W[k][n] (bf16, rounded to nearest even): the
 * weights of a projection that follows RMSNorm with gamma folded in, since
 * (x / r * gamma) @ W = (x @ diag(gamma) W) / r ([XF5] "RMSNorm and Pre-LN residuals").
 * gamma: [d]; W, Wg: [d, N] (device, bf16; Wg caller-owned, may not alias W). N a multiple of
 * 8. One launch on stream; errors as the other entry points.
 */
int attn_fold_rmsnorm_gamma(const void* gamma, const void* W, void* Wg, int d, int N, void* stream);

/*
 * attn_block_fused -- the attention sub-layer of a pre-norm decoder block ([XF5] "RMSNorm and
 * Pre-LN residuals": x + attn(norm(x))), fused around the attention core:
 *   xn = x / sqrt(mean(x^2) + eps) * gamma                      (RMSNorm per row)
 *   [q | k | v] = xn @ Wqkv, Wqkv [d, (H + 2 KV) hd] ([in, out]; columns: q heads, k heads,
 *                 v heads); q and k are turned at positions pos0 + t in the GEMM's epilogue,
 *                 which also writes k (turned) and v to kcache, vcache slots pos0 + t
 *   out = x + attention(q, k, v) @ Wo                           (the residual in the epilogue)
 * x, out: [B,T,d]; gamma: [d]; Wo: [H*hd, d]; all bf16 (device). gamma may be NULL: Wqkv is then
 * taken as already carrying gamma in its rows (diag(gamma) Wqkv, from attn_fold_rmsnorm_gamma),
 * which saves re-folding static weights on every call. kcache, vcache: [B,Lmax,KV,hd]
 * or both NULL (no cache write); with caches, pos0 + T <= Lmax. Causal, window and ALiBi as
 * attn_prefill. workspace: attn_block_fused_workspace_size(...) bytes (device, caller-owned).
 * bf16, hd in {64, 128}, d and (H + 2 KV) hd multiples of 8; anything else returns
 * ATTN_ERR_UNSUPPORTED. Launches: RoPE table, 1/rms per row, gamma folding (with gamma only),
 * QKV GEMM (rows scaled by 1/rms in its epilogue), attention, Wo GEMM (+ residual).
 */
size_t attn_block_fused_workspace_size(int B, int T, int d, int H, int KV, int hd);
int attn_block_fused(const void* x, const void* gamma, const void* Wqkv, const void* Wo, void* out,
                     void* kcache, void* vcache, int Lmax, int B, int T, int d, int H, int KV, int hd,
                     long long pos0, float rope_base, int causal, int window, const float* alibi_slopes,
                     float eps, int dtype, void* workspace, size_t ws_bytes, void* stream);

/* attn_alibi_slopes -- host_out[h] = 2^(-8(h+1)/H) for h < H ([ALIBI] Step 1; the slope
 * schedule with exponent 8/H). host_out is a HOST buffer of H floats. */
void attn_alibi_slopes(int H, float* host_out);

/* attn_sync_status -- synchronise stream, then read and clear this device's error word.
 * Returns ATTN_OK, ATTN_ERR_TIMEOUT, ATTN_ERR_DEVICE_ARG or ATTN_ERR_CUDA. */
int attn_sync_status(void* stream);

/* attn_last_error -- copy the calling thread's last error message (NUL-terminated,
 * truncated to n bytes) into buf; returns the last status. */
int attn_last_error(char* buf, size_t n);

/* attn_version -- static version string of the library. */
const char* attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_ROPE_TILE_H */
