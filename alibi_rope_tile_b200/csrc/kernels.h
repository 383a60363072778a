// Host-side launchers of the attention-core kernels (internal; the C ABI is in
// include/attn_rope_tile.h). Every launcher is asynchronous on the given stream and
// returns the launch's cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace attn {

struct PrefillParams {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;       // [B,H,T] or nullptr
  int B, T, H, KV, hd;
  int pos0;         // position of row 0 (pos0 + T < 2^24)
  int causal, window;
  float scale;      // 1/sqrt(hd)
  int* status;      // device error word
  RopeFreqs rope;
  Alibi alibi;
  // Chunk mode (seqlens != nullptr): k and v are caches [B,Lk,KV,hd] whose keys are already
  // rotated; query row i of sequence b sits at position qpos0[b] + i (T = query rows) and
  // attends slots j < seqlens[b] under the same causal / window rule. Otherwise nullptr.
  const int* seqlens;
  const int* qpos0;
  int Lk;
  // Keys arrive turned at positions pos0 + j (a block's key projection turned them in its
  // epilogue): only the queries are turned here.
  int k_rotated;
  // The launch directly follows the key rotation pass, whose only output is k: the kernel may
  // start while the pass finishes (programmatic dependent launch) and waits for it only
  // before its first key/value load.
  int after_key_pass;
};

// CUDA-core flash prefill: fp32 or bf16 elements, any even hd <= 256.
cudaError_t launch_prefill_simt(const PrefillParams& p, int dtype, cudaStream_t s);

// Tensor-core (tcgen05 + TMEM + TMA) prefill: bf16, hd in {64, 128}. launch_prefill_tc picks
// the kernel; launch_prefill_pair is the two-slot form it uses for hd = 128 with rotation.
bool prefill_tc_supported(const PrefillParams& p, int dtype);
cudaError_t launch_prefill_tc(const PrefillParams& p, cudaStream_t s);
cudaError_t launch_prefill_pair(const PrefillParams& p, cudaStream_t s);
// Persistent form of the single-slot kernel (one CTA per SM over all work units) for a
// prefill whose keys need no turn in the kernel (k_rotated, a chunk over a cache, or no RoPE).
bool prefill_ps_supported(const PrefillParams& p);
cudaError_t launch_prefill_ps(const PrefillParams& p, cudaStream_t s);

struct DecodeParams {
  const void* q;        // [B,H,hd]
  const void* kcache;   // [B,Lmax,KV,hd]
  const void* vcache;
  const int* seqlens;   // [B]
  const int* qpos;      // [B]
  void* out;            // [B,H,hd]
  float* lse;           // [B,H] or nullptr
  int B, H, KV, hd, Lmax;
  int window;
  float scale;
  int* status;
  RopeFreqs rope;
  Alibi alibi;
  // Paged cache (block_table != nullptr): kcache, vcache are page pools
  // [num_pages][page_size][KV][hd]; slot j of sequence b is row j % page_size of page
  // block_table[b * max_blocks + j / page_size]; Lmax = max_blocks * page_size.
  const int* block_table;
  int page_size, num_pages, max_blocks;
  // Latent attention: the merge multiplies each head's merged output (hd numbers, the latent
  // width) by W_out[h] ([H][hd][hd_out], bf16) and writes out [B,H,hd_out]. Otherwise nullptr.
  const void* W_out;
  int hd_out;
};

// Split-KV geometry of the CUDA-core path: keys per split for these sizes.
int decode_chunk(int B, int KV, int Lmax);
// Workspace of either decode path (the larger of the two).
size_t decode_workspace_bytes(int B, int H, int KV, int hd, int Lmax);
cudaError_t launch_decode(const DecodeParams& p, int dtype, void* workspace, cudaStream_t s);
// Tensor-core decode (bf16, hd in {64, 128}, H/KV <= 32): plan, stream-K pass over all key
// tiles, merge (with the up-projection when W_out is set). Its own partial layout.
bool decode_tc_supported(const DecodeParams& p, int dtype);
size_t decode_tc_workspace_bytes(int B, int H, int KV, int hd);
cudaError_t launch_decode_tc(const DecodeParams& p, void* ws, cudaStream_t s);

struct AppendParams {
  const void* k_new;
  const void* v_new;
  void* kcache;
  void* vcache;
  const int* pos;   // [B]: slot of row 0 of sequence b
  int B, Tn, KV, hd, Lmax;  // Tn rows per sequence
  int* status;
  RopeFreqs rope;
  // paged cache, as in DecodeParams (block_table == nullptr: contiguous [B][Lmax][KV][hd])
  const int* block_table;
  int page_size, num_pages, max_blocks;
};
cudaError_t launch_kv_append(const AppendParams& p, int dtype, cudaStream_t s);

// Latent attention's key up-projection folded into the query (bf16): y[b,h,:] = W[h] x[b,h,:]
// (hd -> dc), W [H][dc][hd].
cudaError_t launch_latent_fold(const void* x, const void* W, void* y, int B, int H, int dc, int hd,
                               cudaStream_t s);

// C[M,N] = A[M,K] @ W[K,N], row-major, fp32 accumulation, output in the input dtype.
cudaError_t launch_gemm_simt(const void* A, const void* W, void* C, int M, int N, int K, int dtype,
                             cudaStream_t s);
// Tensor-core (tcgen05) version for bf16 when M, N, K fit its tiles.
// Epilogues of the tensor-core GEMM beyond a plain store of C (bf16).
struct GemmEpilogue {
  int mode;                // 0: C = A W with the options below; 2: C = A W + residual ([M,N])
  const float* row_scale;  // [M] or nullptr: row m of C scaled by row_scale[m]
  int rot_seg;             // segment whose heads are turned (-1: none): pairs (2c, 2c+1) of each
                           // hd-wide head by the (cos, sin) of the row's position, from rope_cs
                           // [T][hd/2] with t = m % T
  const float2* rope_cs;
  int T, hd;
  void* cache[3];          // per segment, or nullptr: also written into a cache [B][Lmax][Ns] at
                           // row slot pos0 + t (B = M / T)
  int Lmax, pos0;
  const void* residual;
};
bool gemm_tc_supported(int M, int N, int K, int dtype);
cudaError_t launch_gemm_tc(const void* A, const void* W, void* C, int M, int N, int K, int* status,
                           cudaStream_t s, const GemmEpilogue* ep = nullptr);
// One launch over nseg <= 3 weight matrices side by side: C_i [M, Ns[i]] = A @ W_i. Every
// segment but the last must be a multiple of 64 columns wide (gemm_tc_segments_fit).
bool gemm_tc_segments_fit(int nseg, const int* Ns);
// The weights W_i are [K, Ns[i]] with rows ldw elements apart (0: Ns[i]), so they may be column
// blocks of one matrix.
cudaError_t launch_gemm_tc_multi(const void* A, int nseg, const void* const* Ws, void* const* Cs, const int* Ns,
                                 int M, int K, int* status, cudaStream_t s, const GemmEpilogue* ep = nullptr,
                                 int ldw = 0);

// Pre-norm helpers of the fused block: the inverse root-mean-square of every row of x, 1 / sqrt(mean
// (x^2) + eps) (fp32), the weights with gamma folded into their rows, Wg[k][n] = gamma[k] W[k][n]
// (bf16), and the table of (cos, sin) of every (position pos0 + t, pair) an epilogue turns by.
cudaError_t launch_rms_inverse(const void* x, float* rinv, int M, int d, float eps, cudaStream_t s);
cudaError_t launch_fold_gamma(const void* W, const void* gamma, void* Wg, int d, int N, cudaStream_t s);
cudaError_t launch_rope_table(float2* cs, int T, int pos0, const RopeFreqs& rope, int hd, cudaStream_t s);

// Key rotation pass (bf16, hd % 8 == 0): kr [B,T,KV,hd] = k turned at positions pos0 + t.
// The prefill then runs with k_rotated set on kr.
cudaError_t launch_rope_keys(const void* k, void* kr, int B, int T, int KV, int hd, int pos0,
                             const RopeFreqs& rope, cudaStream_t s);

// Records a failure for attn_last_error() and returns ``code`` (used by entry points
// defined outside api.cu).
int record_error(int code, const char* message);

}  // namespace attn
