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

constexpr int kMaxSlices = 32;
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

// How the problem is cut. A slice is nb sequences from b0 with ng key/value heads from g0
// (and their query heads): either whole sequences (ng = KV) or part of one sequence (nb = 1).
// Four or more sequences: up to eight runs of whole sequences; fewer: one sequence and the
// largest group of key/value heads that still gives four slices (at most 16). At most
// 8 + 1 + 9 or 16 + 9 slices in all (KV <= 256), within kMaxSlices. Once the last slice's rows
// have landed, only its attention and its copy back remain, so the last slice is cut finer:
// its sequences but one become a slice of their own, and the heads of the last sequence are
// split in halves (for example 4 heads -> 2, 1, 1), each a slice.
struct Slice {
  int b0, nb, g0, ng;
};
int plan_of(int B, int KV, Slice* sl) {
  int n = 0;
  if (B >= 4) {
    const int runs = std::min(B, 8), nbs = (B + runs - 1) / runs;
    for (int b0 = 0; b0 < B; b0 += nbs) sl[n++] = Slice{b0, std::min(nbs, B - b0), 0, KV};
  } else {
    // at most 16 slices before the last is cut (a prime KV falls back to whole sequences)
    int ng = KV;
    for (int g = KV; g >= 1; --g)
      if (KV % g == 0 && B * (KV / g) >= 4) {
        if (B * (KV / g) <= 16) ng = g;
        break;
      }
    for (int b = 0; b < B; ++b)
      for (int g0 = 0; g0 < KV; g0 += ng) sl[n++] = Slice{b, 1, g0, ng};
  }
  Slice last = sl[--n];
  if (last.nb > 1) {
    sl[n++] = Slice{last.b0, last.nb - 1, 0, KV};
    last = Slice{last.b0 + last.nb - 1, 1, 0, KV};
  }
  int g0 = last.g0, rem = last.ng;
  while (rem > 1) {
    const int part = (rem + 1) / 2;
    sl[n++] = Slice{last.b0, 1, g0, part};
    g0 += part;
    rem -= part;
  }
  if (rem == 1) sl[n++] = Slice{last.b0, 1, g0, 1};
  return n;
}

// Device bytes of a slice's dense q, k, v, out and lse.
struct SliceBytes {
  size_t q, kv, lse;
};
SliceBytes slice_bytes(const Slice& sl, int T, int H, int KV, int hd, int dtype) {
  const size_t es = dtype == ATTN_F32 ? 4 : 2;
  const int G = H / KV;
  SliceBytes sb;
  sb.q = r256((size_t)sl.nb * T * sl.ng * G * hd * es);
  sb.kv = r256((size_t)sl.nb * T * sl.ng * hd * es);
  sb.lse = r256((size_t)sl.nb * sl.ng * G * T * sizeof(float));
  return sb;
}
size_t slice_total(const SliceBytes& sb) { return 2 * sb.q + 2 * sb.kv + sb.lse; }

// The rotation pass's scratch of the largest slice (slices run one after another).
size_t rot_bytes(const Slice* sl, int n, int T, int hd, float rope_base, int dtype) {
  size_t m = 0;
  for (int i = 0; i < n; ++i)
    m = std::max(m, attn_prefill_workspace_size(sl[i].nb, T, sl[i].ng, hd, rope_base, dtype));
  return r256(m);
}

}  // namespace

extern "C" {

size_t attn_prefill_host_workspace_size(int B, int T, int H, int KV, int hd, float rope_base, int dtype) {
  if (B < 1 || T < 1 || H < 1 || KV < 1 || H % KV || hd < 2 || hd > 256 || (hd & 1) ||
      (dtype != ATTN_F32 && dtype != ATTN_BF16))
    return 0;
  Slice sl[kMaxSlices];
  const int n = plan_of(B, KV, sl);
  size_t total = 0;
  for (int i = 0; i < n; ++i) total += slice_total(slice_bytes(sl[i], T, H, KV, hd, dtype));
  return total + rot_bytes(sl, n, T, hd, rope_base, dtype);
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

  Slice sl[kMaxSlices];
  const int nsl = plan_of(B, KV, sl);
  const size_t rot_size = rot_bytes(sl, nsl, T, hd, rope_base, dtype);
  const size_t es = dtype == ATTN_F32 ? 4 : 2;
  const int G = H / KV;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* rot = ws + need - rot_size;
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
  uint8_t* base = ws;
  for (int s = 0; s < nsl; ++s) {
    const int b0 = sl[s].b0, nb = sl[s].nb, g0 = sl[s].g0, ng = sl[s].ng;
    const SliceBytes sb = slice_bytes(sl[s], T, H, KV, hd, dtype);
    uint8_t *dq = base, *dk = dq + sb.q, *dv = dk + sb.kv, *dout = dv + sb.kv, *dl = dout + sb.q;
    base += slice_total(sb);
    // rows of nb sequences; a row holds this slice's heads (width) out of all heads (pitch)
    const size_t qw = (size_t)ng * G * hd * es, qp = (size_t)H * hd * es;
    const size_t kw = (size_t)ng * hd * es, kp = (size_t)KV * hd * es;
    const size_t rows = (size_t)nb * T;
    const size_t qoff = (size_t)b0 * T * qp + (size_t)g0 * G * hd * es;
    const size_t koff = (size_t)b0 * T * kp + (size_t)g0 * hd * es;
    HP_TRY(cudaMemcpy2DAsync(dq, qw, static_cast<const uint8_t*>(q) + qoff, qp, qw, rows, cudaMemcpyHostToDevice, P.in));
    HP_TRY(cudaMemcpy2DAsync(dk, kw, static_cast<const uint8_t*>(k) + koff, kp, kw, rows, cudaMemcpyHostToDevice, P.in));
    HP_TRY(cudaMemcpy2DAsync(dv, kw, static_cast<const uint8_t*>(v) + koff, kp, kw, rows, cudaMemcpyHostToDevice, P.in));
    HP_TRY(cudaEventRecord(P.landed[s], P.in));
    HP_TRY(cudaStreamWaitEvent(user, P.landed[s], 0));
    const size_t rot_need = attn_prefill_workspace_size(nb, T, ng, hd, rope_base, dtype);
    const int st = attn_prefill_ws(dq, dk, dv, dout, lse ? reinterpret_cast<float*>(dl) : nullptr, nb, T,
                                   ng * G, ng, hd, pos0, rope_base, causal, window,
                                   alibi_slopes ? alibi_slopes + (size_t)g0 * G : nullptr, dtype,
                                   rot_need ? rot : nullptr, rot_need, user);
    if (st != ATTN_OK) return st;
    HP_TRY(cudaEventRecord(P.computed[s], user));
    HP_TRY(cudaStreamWaitEvent(P.out, P.computed[s], 0));
    HP_TRY(cudaMemcpy2DAsync(static_cast<uint8_t*>(out) + qoff, qp, dout, qw, qw, rows, cudaMemcpyDeviceToHost, P.out));
    if (lse) {
      // lse [B][H][T]: a slice's heads of a sequence are contiguous; its sequences are H*T apart
      const size_t lw = (size_t)ng * G * T * sizeof(float);
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
