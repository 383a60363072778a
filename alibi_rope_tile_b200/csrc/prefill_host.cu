// attn_prefill_host: a prefill whose q, k, v and results live in host memory. The call cuts the
// problem into slices that are independent in the attention ("Write attention from scratch",
// worked example: each (sequence, query head) row set reads only its own key/value head), so
// the copies of one slice overlap the attention of another:
//   copy-in stream   H2D slice 0, H2D slice 1, ...            (2-D copies of strided heads)
//   caller's stream          attention slice 0, attention slice 1, ...
//   copy-out stream                  D2H slice 0, D2H slice 1, ...
// Each slice runs the device prefill (attn_prefill_ws) on a dense copy of its rows, so every
// output row is computed exactly as by one call over the whole device tensors.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "attn_rope_tile.h"
#include "kernels.h"

namespace {

constexpr int kMaxSlices = 16;
constexpr int kMaxDevices = 64;

// The copy streams and events of one device, created on first use and kept for the process
// (the library's only long-lived CUDA objects besides its status word and no-alloc scratch).
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t entry = nullptr, done = nullptr;
  cudaEvent_t landed[kMaxSlices] = {}, computed[kMaxSlices] = {};
  bool ready = false;
};
std::mutex g_pipe_mu;  // also serialises the enqueueing of calls that share a device's objects
HostPipe g_pipe[kMaxDevices];

cudaError_t make_pipe(HostPipe& p) {
  cudaError_t e;
  if ((e = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if ((e = cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if ((e = cudaEventCreateWithFlags(&p.entry, cudaEventDisableTiming)) != cudaSuccess) return e;
  if ((e = cudaEventCreateWithFlags(&p.done, cudaEventDisableTiming)) != cudaSuccess) return e;
  for (int s = 0; s < kMaxSlices; ++s) {
    if ((e = cudaEventCreateWithFlags(&p.landed[s], cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&p.computed[s], cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  p.ready = true;
  return cudaSuccess;
}

size_t r256(size_t n) { return (n + 255) & ~(size_t)255; }

// How the problem is cut: nbs sequences and ng key/value heads per slice. Four or more
// sequences: runs of whole sequences (contiguous rows), at most kMaxSlices of them; fewer: one
// sequence and the largest group of key/value heads that still gives four slices.
struct Plan {
  int nbs, ng, nslices;
};
Plan plan_of(int B, int KV) {
  Plan pl;
  if (B >= 4) {
    const int s = std::min(B, kMaxSlices);
    pl.nbs = (B + s - 1) / s;
    pl.ng = KV;
  } else {
    pl.nbs = 1;
    pl.ng = 1;
    for (int ng = KV; ng >= 1; --ng)
      if (KV % ng == 0 && B * (KV / ng) >= 4) {
        pl.ng = ng;
        break;
      }
  }
  pl.nslices = ((B + pl.nbs - 1) / pl.nbs) * (KV / pl.ng);
  return pl;
}

// Device bytes of one slice's dense q, k, v, out and lse, and the rotation pass's scratch.
struct SliceBytes {
  size_t q, kv, lse, rot;
};
SliceBytes slice_bytes(const Plan& pl, int T, int H, int KV, int hd, float rope_base, int dtype) {
  const size_t es = dtype == ATTN_F32 ? 4 : 2;
  const int G = H / KV;
  SliceBytes sb;
  sb.q = r256((size_t)pl.nbs * T * pl.ng * G * hd * es);
  sb.kv = r256((size_t)pl.nbs * T * pl.ng * hd * es);
  sb.lse = r256((size_t)pl.nbs * pl.ng * G * T * sizeof(float));
  sb.rot = r256(attn_prefill_workspace_size(pl.nbs, T, pl.ng, hd, rope_base, dtype));
  return sb;
}

}  // namespace

extern "C" {

size_t attn_prefill_host_workspace_size(int B, int T, int H, int KV, int hd, float rope_base, int dtype) {
  if (B < 1 || T < 1 || H < 1 || KV < 1 || H % KV || hd < 2 || hd > 256 || (hd & 1) ||
      (dtype != ATTN_F32 && dtype != ATTN_BF16))
    return 0;
  const Plan pl = plan_of(B, KV);
  const SliceBytes sb = slice_bytes(pl, T, H, KV, hd, rope_base, dtype);
  return (size_t)pl.nslices * (2 * sb.q + 2 * sb.kv + sb.lse) + sb.rot;
}

int attn_prefill_host(const void* q, const void* k, const void* v, void* out, float* lse, int B, int T,
                      int H, int KV, int hd, long long pos0, float rope_base, int causal, int window,
                      const float* alibi_slopes, int dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !out) return attn::record_error(ATTN_ERR_ARG, "q, k, v and out must not be NULL");
  if (B < 1 || T < 1 || H < 1 || KV < 1 || H % KV)
    return attn::record_error(ATTN_ERR_ARG, "B, T, H, KV must be >= 1 with H a multiple of KV");
  if (hd < 2 || hd > 256 || (hd & 1)) return attn::record_error(ATTN_ERR_ARG, "hd must be even and in [2, 256]");
  if (dtype != ATTN_F32 && dtype != ATTN_BF16) return attn::record_error(ATTN_ERR_ARG, "unknown dtype");
  const size_t need = attn_prefill_host_workspace_size(B, T, H, KV, hd, rope_base, dtype);
  if (!workspace || ws_bytes < need)
    return attn::record_error(ATTN_ERR_WORKSPACE, "attn_prefill_host needs its workspace size of device scratch");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return attn::record_error(ATTN_ERR_ALIGN, "the workspace must be 256-byte aligned");

  const Plan pl = plan_of(B, KV);
  const SliceBytes sb = slice_bytes(pl, T, H, KV, hd, rope_base, dtype);
  const size_t es = dtype == ATTN_F32 ? 4 : 2;
  const int G = H / KV;
  const int ngrp = KV / pl.ng;  // slices per run of sequences
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* rot = ws + (size_t)pl.nslices * (2 * sb.q + 2 * sb.kv + sb.lse);
  cudaStream_t user = static_cast<cudaStream_t>(stream);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return attn::record_error(ATTN_ERR_CUDA, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe& P = g_pipe[dev];
  if (!P.ready && (e = make_pipe(P)) != cudaSuccess)
    return attn::record_error(ATTN_ERR_CUDA, "attn_prefill_host: stream or event creation failed");
#define HP_TRY(call)                                                             \
  do {                                                                           \
    if ((e = (call)) != cudaSuccess)                                             \
      return attn::record_error(ATTN_ERR_CUDA, "attn_prefill_host: " #call);    \
  } while (0)
  // the copies in start after the caller's earlier work on its stream (which may still use a
  // workspace it shares with this call)
  HP_TRY(cudaEventRecord(P.entry, user));
  HP_TRY(cudaStreamWaitEvent(P.in, P.entry, 0));
  HP_TRY(cudaStreamWaitEvent(P.out, P.entry, 0));
  for (int s = 0; s < pl.nslices; ++s) {
    const int b0 = (s / ngrp) * pl.nbs, g0 = (s % ngrp) * pl.ng;
    const int nb = std::min(pl.nbs, B - b0);
    uint8_t* base = ws + (size_t)s * (2 * sb.q + 2 * sb.kv + sb.lse);
    uint8_t *dq = base, *dk = dq + sb.q, *dv = dk + sb.kv, *dout = dv + sb.kv, *dl = dout + sb.q;
    // rows of nb sequences; a row holds this slice's heads (width) out of all heads (pitch)
    const size_t qw = (size_t)pl.ng * G * hd * es, qp = (size_t)H * hd * es;
    const size_t kw = (size_t)pl.ng * hd * es, kp = (size_t)KV * hd * es;
    const size_t rows = (size_t)nb * T;
    const size_t qoff = (size_t)b0 * T * qp + (size_t)g0 * G * hd * es;
    const size_t koff = (size_t)b0 * T * kp + (size_t)g0 * hd * es;
    HP_TRY(cudaMemcpy2DAsync(dq, qw, static_cast<const uint8_t*>(q) + qoff, qp, qw, rows, cudaMemcpyHostToDevice, P.in));
    HP_TRY(cudaMemcpy2DAsync(dk, kw, static_cast<const uint8_t*>(k) + koff, kp, kw, rows, cudaMemcpyHostToDevice, P.in));
    HP_TRY(cudaMemcpy2DAsync(dv, kw, static_cast<const uint8_t*>(v) + koff, kp, kw, rows, cudaMemcpyHostToDevice, P.in));
    HP_TRY(cudaEventRecord(P.landed[s], P.in));
    HP_TRY(cudaStreamWaitEvent(user, P.landed[s], 0));
    const int st = attn_prefill_ws(dq, dk, dv, dout, lse ? reinterpret_cast<float*>(dl) : nullptr, nb, T,
                                   pl.ng * G, pl.ng, hd, pos0, rope_base, causal, window,
                                   alibi_slopes ? alibi_slopes + (size_t)g0 * G : nullptr, dtype,
                                   sb.rot ? rot : nullptr, sb.rot, user);
    if (st != ATTN_OK) return st;
    HP_TRY(cudaEventRecord(P.computed[s], user));
    HP_TRY(cudaStreamWaitEvent(P.out, P.computed[s], 0));
    HP_TRY(cudaMemcpy2DAsync(static_cast<uint8_t*>(out) + qoff, qp, dout, qw, qw, rows, cudaMemcpyDeviceToHost, P.out));
    if (lse) {
      // lse [B][H][T]: a slice's heads of a sequence are contiguous; its sequences are H*T apart
      const size_t lw = (size_t)pl.ng * G * T * sizeof(float);
      HP_TRY(cudaMemcpy2DAsync(lse + ((size_t)b0 * H + (size_t)g0 * G) * T, (size_t)H * T * sizeof(float), dl, lw,
                               lw, nb, cudaMemcpyDeviceToHost, P.out));
    }
  }
  // work queued on the caller's stream after this call sees the results in host memory
  HP_TRY(cudaEventRecord(P.done, P.out));
  HP_TRY(cudaStreamWaitEvent(user, P.done, 0));
#undef HP_TRY
  return ATTN_OK;
}

}  // extern "C"
