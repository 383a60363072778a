// Host side of the C ABI declared in include/attn_rope_tile.h: argument checks, the
// per-call rotary/ALiBi tables, dispatch to the kernels, and error reporting. No entry
// point allocates device memory.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "attn_rope_tile.h"
#include "kernels.h"

using namespace attn;

namespace {

thread_local char g_msg[512] = "no error";
thread_local int g_last = ATTN_OK;

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  g_last = code;
  return code;
}

int ok() {
  g_last = ATTN_OK;
  return ATTN_OK;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(ATTN_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

}  // namespace

namespace attn {
int record_error(int code, const char* message) { return fail(code, "%s", message); }
}  // namespace attn

// Per-device status word written by kernels that find a bad device-resident argument or
// give up on a bounded wait. Host code reaches it through cudaGetSymbolAddress.
__device__ int g_attn_device_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
int* g_status_ptr[kMaxDevices] = {};

int* device_status(int* err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = cuda_fail(e == cudaSuccess ? cudaErrorInvalidDevice : e, "cudaGetDevice");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_attn_device_status);
    if (e != cudaSuccess) {
      *err = cuda_fail(e, "cudaGetSymbolAddress(status word)");
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<int*>(ptr);
  }
  return g_status_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(int dtype) { return dtype == ATTN_F32 ? 4 : 2; }

RopeFreqs make_rope(int hd, float base) {
  RopeFreqs r;
  std::memset(&r, 0, sizeof(r));
  r.on = base > 0.f;
  if (!r.on) return r;
  const double two_pi = 6.283185307179586476925286766559;
  for (int c = 0; c < hd / 2; ++c) {
    const double w = std::pow((double)base, -2.0 * c / hd) / two_pi;  // turns per position
    const float hi = (float)w;
    r.hi[c] = hi;
    r.lo[c] = (float)(w - (double)hi);
  }
  return r;
}

int make_alibi(int H, const float* slopes, Alibi* a) {
  std::memset(a, 0, sizeof(*a));
  if (!slopes) return ATTN_OK;
  if (H > ATTN_MAX_ALIBI_HEADS)
    return fail(ATTN_ERR_UNSUPPORTED, "ALiBi supports at most %d heads (got %d)",
                ATTN_MAX_ALIBI_HEADS, H);
  a->on = 1;
  for (int h = 0; h < H; ++h) {
    if (!std::isfinite(slopes[h])) return fail(ATTN_ERR_ARG, "alibi_slopes[%d] is not finite", h);
    a->slope[h] = slopes[h];
  }
  return ATTN_OK;
}

int check_common(int H, int KV, int hd, int dtype, float rope_base) {
  if (dtype != ATTN_F32 && dtype != ATTN_BF16) return fail(ATTN_ERR_ARG, "dtype %d is not ATTN_F32/ATTN_BF16", dtype);
  if (H < 1 || KV < 1) return fail(ATTN_ERR_ARG, "H=%d and KV=%d must be >= 1", H, KV);
  if (H % KV) return fail(ATTN_ERR_ARG, "H=%d is not a multiple of KV=%d", H, KV);
  if (hd < 2 || hd > ATTN_MAX_HD || (hd & 1))
    return fail(ATTN_ERR_ARG, "hd=%d must be even and in [2, %d]", hd, ATTN_MAX_HD);
  if (!std::isfinite(rope_base)) return fail(ATTN_ERR_ARG, "rope_base is not finite");
  return ATTN_OK;
}

}  // namespace

extern "C" {

size_t attn_prefill_workspace_size(int B, int T, int KV, int hd, float rope_base, int dtype) {
  if (B < 1 || T < 1 || KV < 1 || dtype != ATTN_BF16 || (hd != 64 && hd != 128) || !(rope_base > 0.f)) return 0;
  return (size_t)B * T * KV * hd * 2;
}

int attn_prefill_ws(const void* q, const void* k, const void* v, void* out, float* lse, int B, int T,
                    int H, int KV, int hd, long long pos0, float rope_base, int causal, int window,
                    const float* alibi_slopes, int dtype, void* workspace, size_t ws_bytes, void* stream) {
  int st = check_common(H, KV, hd, dtype, rope_base);
  if (st) return st;
  if (!q || !k || !v || !out) return fail(ATTN_ERR_ARG, "q, k, v and out must not be NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned16(lse)))
    return fail(ATTN_ERR_ALIGN, "q, k, v, out and lse must be 16-byte aligned");
  if (B < 1 || T < 1) return fail(ATTN_ERR_ARG, "B=%d and T=%d must be >= 1", B, T);
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_ARG, "causal must be 0 or 1");
  if (window < 0) window = 0;
  if (window > 0 && !causal) return fail(ATTN_ERR_ARG, "a window requires the causal mask");
  if (pos0 < 0 || pos0 + (long long)T >= (1LL << 24))
    return fail(ATTN_ERR_ARG, "positions pos0..pos0+T-1 must lie in [0, 2^24)");
  if ((long long)B * T * H * hd >= (1LL << 40)) return fail(ATTN_ERR_ARG, "tensor too large");
  // the key rotation pass runs when it applies and the caller gave its scratch
  const size_t need = attn_prefill_workspace_size(B, T, KV, hd, rope_base, dtype);
  if (workspace) {
    if (!aligned16(workspace)) return fail(ATTN_ERR_ALIGN, "workspace must be 16-byte aligned");
    if (ws_bytes < need)
      return fail(ATTN_ERR_WORKSPACE, "prefill needs %zu bytes of workspace (got %zu)", need, ws_bytes);
  }
  const bool turn_first = workspace && need > 0;

  PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.out = out; p.lse = lse;
  p.B = B; p.T = T; p.H = H; p.KV = KV; p.hd = hd;
  p.pos0 = (int)pos0; p.causal = causal; p.window = window;
  p.scale = (float)(1.0 / std::sqrt((double)hd));
  p.rope = make_rope(hd, rope_base);
  if ((st = make_alibi(H, alibi_slopes, &p.alibi))) return st;
  int err = 0;
  p.status = device_status(&err);
  if (!p.status) return err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (turn_first) {
    cudaError_t e = launch_rope_keys(k, workspace, B, T, KV, hd, p.pos0, p.rope, s);
    if (e != cudaSuccess) return cuda_fail(e, "attn_prefill_ws key rotation launch");
    p.k = workspace;
    p.k_rotated = 1;
    p.after_key_pass = 1;
  }
  cudaError_t e = prefill_tc_supported(p, dtype) ? launch_prefill_tc(p, s)
                                                 : launch_prefill_simt(p, dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "attn_prefill launch");
  return ok();
}

int attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B, int T,
                 int H, int KV, int hd, long long pos0, float rope_base, int causal, int window,
                 const float* alibi_slopes, int dtype, void* stream) {
  return attn_prefill_ws(q, k, v, out, lse, B, T, H, KV, hd, pos0, rope_base, causal, window,
                         alibi_slopes, dtype, nullptr, 0, stream);
}

int attn_prefill_chunk(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                       const int* qpos0, void* out, float* lse, int B, int Tq, int H, int KV, int hd,
                       int Lmax, float rope_base, int causal, int window, const float* alibi_slopes,
                       int dtype, void* stream) {
  int st = check_common(H, KV, hd, dtype, rope_base);
  if (st) return st;
  if (!q || !kcache || !vcache || !seqlens || !qpos0 || !out)
    return fail(ATTN_ERR_ARG, "q, kcache, vcache, seqlens, qpos0 and out must not be NULL");
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out) || (lse && !aligned16(lse)))
    return fail(ATTN_ERR_ALIGN, "q, kcache, vcache, out and lse must be 16-byte aligned");
  if (B < 1 || Tq < 1 || Lmax < 1 || Lmax >= (1 << 24) || Tq >= (1 << 24))
    return fail(ATTN_ERR_ARG, "B, Tq >= 1 and 1 <= Lmax < 2^24");
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_ARG, "causal must be 0 or 1");
  if (window < 0) window = 0;
  if (window > 0 && !causal) return fail(ATTN_ERR_ARG, "a window requires the causal mask");
  if ((long long)B * Tq * H * hd >= (1LL << 40) || (long long)B * Lmax * KV * hd >= (1LL << 40))
    return fail(ATTN_ERR_ARG, "tensor too large");

  PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.k = kcache; p.v = vcache; p.out = out; p.lse = lse;
  p.B = B; p.T = Tq; p.H = H; p.KV = KV; p.hd = hd;
  p.pos0 = 0; p.causal = causal; p.window = window;
  p.seqlens = seqlens; p.qpos0 = qpos0; p.Lk = Lmax;
  p.scale = (float)(1.0 / std::sqrt((double)hd));
  p.rope = make_rope(hd, rope_base);
  if ((st = make_alibi(H, alibi_slopes, &p.alibi))) return st;
  if (!prefill_tc_supported(p, dtype))
    return fail(ATTN_ERR_UNSUPPORTED, "attn_prefill_chunk runs bf16 with hd 64 or 128 (got dtype %d, hd %d)",
                dtype, hd);
  int err = 0;
  p.status = device_status(&err);
  if (!p.status) return err;
  cudaError_t e = launch_prefill_tc(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_prefill_chunk launch");
  return ok();
}

size_t attn_decode_workspace_size(int B, int H, int KV, int hd, int Lmax) {
  if (B < 1 || H < 1 || KV < 1 || H % KV || hd < 2 || hd > ATTN_MAX_HD || Lmax < 1) return 0;
  return decode_workspace_bytes(B, H, KV, hd, Lmax);
}

int attn_decode(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                const int* qpos, void* out, float* lse, int B, int H, int KV, int hd, int Lmax,
                float rope_base, int window, const float* alibi_slopes, int dtype, void* workspace,
                size_t ws_bytes, void* stream) {
  int st = check_common(H, KV, hd, dtype, rope_base);
  if (st) return st;
  if (!q || !kcache || !vcache || !seqlens || !qpos || !out)
    return fail(ATTN_ERR_ARG, "q, kcache, vcache, seqlens, qpos and out must not be NULL");
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out) ||
      (lse && !aligned16(lse)) || (workspace && !aligned16(workspace)))
    return fail(ATTN_ERR_ALIGN, "q, caches, out, lse and workspace must be 16-byte aligned");
  if (B < 1 || Lmax < 1) return fail(ATTN_ERR_ARG, "B=%d and Lmax=%d must be >= 1", B, Lmax);
  if (Lmax >= (1 << 24)) return fail(ATTN_ERR_ARG, "Lmax must be below 2^24");
  const int G = H / KV;
  if (!(hd == 8 || hd == 16 || hd == 32 || hd == 64 || hd == 128 || hd == 256))
    return fail(ATTN_ERR_UNSUPPORTED, "decode supports hd in {8,16,32,64,128,256} (got %d)", hd);
  if (!(G == 1 || G == 2 || G == 4 || G == 8 || G == 16 || G == 32))
    return fail(ATTN_ERR_UNSUPPORTED, "decode supports H/KV in {1,2,4,8,16,32} (got %d)", G);
  if ((size_t)8 * G * (hd + 2) * sizeof(float) > 200 * 1024)
    return fail(ATTN_ERR_UNSUPPORTED, "decode: H/KV * hd too large for shared memory");
  if (window < 0) window = 0;
  const size_t need = decode_workspace_bytes(B, H, KV, hd, Lmax);
  if (!workspace || ws_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "decode needs %zu bytes of workspace (got %zu)", need, ws_bytes);

  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.kcache = kcache; p.vcache = vcache; p.seqlens = seqlens; p.qpos = qpos;
  p.out = out; p.lse = lse;
  p.B = B; p.H = H; p.KV = KV; p.hd = hd; p.Lmax = Lmax; p.window = window;
  p.scale = (float)(1.0 / std::sqrt((double)hd));
  p.rope = make_rope(hd, rope_base);
  if ((st = make_alibi(H, alibi_slopes, &p.alibi))) return st;
  int err = 0;
  p.status = device_status(&err);
  if (!p.status) return err;
  cudaError_t e = launch_decode(p, dtype, workspace, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode launch");
  return ok();
}

int attn_kv_append(const void* k_new, const void* v_new, void* kcache, void* vcache, const int* pos,
                   int B, int KV, int hd, int Lmax, float rope_base, int dtype, void* stream) {
  int st = check_common(KV, KV, hd, dtype, rope_base);
  if (st) return st;
  if (!k_new || !v_new || !kcache || !vcache || !pos)
    return fail(ATTN_ERR_ARG, "k_new, v_new, kcache, vcache and pos must not be NULL");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kcache) || !aligned16(vcache))
    return fail(ATTN_ERR_ALIGN, "k_new, v_new and the caches must be 16-byte aligned");
  if (B < 1 || Lmax < 1 || Lmax >= (1 << 24)) return fail(ATTN_ERR_ARG, "B >= 1 and 1 <= Lmax < 2^24");
  AppendParams p;
  std::memset(&p, 0, sizeof(p));
  p.k_new = k_new; p.v_new = v_new; p.kcache = kcache; p.vcache = vcache; p.pos = pos;
  p.B = B; p.Tn = 1; p.KV = KV; p.hd = hd; p.Lmax = Lmax;
  p.rope = make_rope(hd, rope_base);
  int err = 0;
  p.status = device_status(&err);
  if (!p.status) return err;
  cudaError_t e = launch_kv_append(p, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_kv_append launch");
  return ok();
}

namespace {
int check_pages(int page_size, int num_pages, int max_blocks) {
  if (!(page_size == 8 || page_size == 16 || page_size == 32 || page_size == 64 || page_size == 128))
    return fail(ATTN_ERR_ARG, "page_size must be 8, 16, 32, 64 or 128 (got %d)", page_size);
  if (num_pages < 1 || max_blocks < 1) return fail(ATTN_ERR_ARG, "num_pages and max_blocks must be >= 1");
  if ((long long)max_blocks * page_size >= (1LL << 24) || (long long)num_pages * page_size >= (1LL << 31))
    return fail(ATTN_ERR_ARG, "max_blocks * page_size must be below 2^24");
  return ATTN_OK;
}
}  // namespace

int attn_decode_paged(const void* q, const void* kpages, const void* vpages, const int* block_table,
                      const int* seqlens, const int* qpos, void* out, float* lse, int B, int H, int KV,
                      int hd, int page_size, int num_pages, int max_blocks, float rope_base, int window,
                      const float* alibi_slopes, int dtype, void* workspace, size_t ws_bytes, void* stream) {
  int st = check_common(H, KV, hd, dtype, rope_base);
  if (st) return st;
  if ((st = check_pages(page_size, num_pages, max_blocks))) return st;
  if (!q || !kpages || !vpages || !block_table || !seqlens || !qpos || !out)
    return fail(ATTN_ERR_ARG, "q, kpages, vpages, block_table, seqlens, qpos and out must not be NULL");
  if (!aligned16(q) || !aligned16(kpages) || !aligned16(vpages) || !aligned16(out) ||
      (lse && !aligned16(lse)) || (workspace && !aligned16(workspace)))
    return fail(ATTN_ERR_ALIGN, "q, page pools, out, lse and workspace must be 16-byte aligned");
  if (B < 1) return fail(ATTN_ERR_ARG, "B=%d must be >= 1", B);
  if (window < 0) window = 0;
  const int Lmax = max_blocks * page_size;
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.kcache = kpages; p.vcache = vpages; p.seqlens = seqlens; p.qpos = qpos;
  p.out = out; p.lse = lse;
  p.B = B; p.H = H; p.KV = KV; p.hd = hd; p.Lmax = Lmax; p.window = window;
  p.block_table = block_table; p.page_size = page_size; p.num_pages = num_pages; p.max_blocks = max_blocks;
  p.scale = (float)(1.0 / std::sqrt((double)hd));
  p.rope = make_rope(hd, rope_base);
  if ((st = make_alibi(H, alibi_slopes, &p.alibi))) return st;
  if (!decode_tc_supported(p, dtype))
    return fail(ATTN_ERR_UNSUPPORTED, "attn_decode_paged runs bf16 with hd 64 or 128 and H/KV <= 32");
  const size_t need = decode_workspace_bytes(B, H, KV, hd, Lmax);
  if (!workspace || ws_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "decode needs %zu bytes of workspace (got %zu)", need, ws_bytes);
  int err = 0;
  p.status = device_status(&err);
  if (!p.status) return err;
  cudaError_t e = launch_decode(p, dtype, workspace, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode_paged launch");
  return ok();
}

int attn_kv_write_paged(const void* k_new, const void* v_new, void* kpages, void* vpages,
                        const int* block_table, const int* pos0, int B, int Tn, int KV, int hd,
                        int page_size, int num_pages, int max_blocks, float rope_base, int dtype,
                        void* stream) {
  int st = check_common(KV, KV, hd, dtype, rope_base);
  if (st) return st;
  if ((st = check_pages(page_size, num_pages, max_blocks))) return st;
  if (!k_new || !v_new || !kpages || !vpages || !block_table || !pos0)
    return fail(ATTN_ERR_ARG, "k_new, v_new, kpages, vpages, block_table and pos0 must not be NULL");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kpages) || !aligned16(vpages))
    return fail(ATTN_ERR_ALIGN, "k_new, v_new and the page pools must be 16-byte aligned");
  if (B < 1 || Tn < 1 || Tn > 65535) return fail(ATTN_ERR_ARG, "B >= 1 and 1 <= Tn <= 65535");
  AppendParams p;
  std::memset(&p, 0, sizeof(p));
  p.k_new = k_new; p.v_new = v_new; p.kcache = kpages; p.vcache = vpages; p.pos = pos0;
  p.B = B; p.Tn = Tn; p.KV = KV; p.hd = hd; p.Lmax = max_blocks * page_size;
  p.block_table = block_table; p.page_size = page_size; p.num_pages = num_pages; p.max_blocks = max_blocks;
  p.rope = make_rope(hd, rope_base);
  int err = 0;
  p.status = device_status(&err);
  if (!p.status) return err;
  cudaError_t e = launch_kv_append(p, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_kv_write_paged launch");
  return ok();
}

namespace {
size_t r256(size_t x) { return (x + 255) & ~(size_t)255; }
}  // namespace

size_t attn_decode_latent_workspace_size(int B, int H, int hd, int dc, int Lmax) {
  if (B < 1 || H < 1 || hd < 2 || (dc != 64 && dc != 128) || Lmax < 1) return 0;
  const size_t vec = r256((size_t)B * H * dc * 2);  // q' (bf16)
  return vec + decode_workspace_bytes(B, H, 1, dc, Lmax);
}

int attn_decode_latent(const void* q, const void* ccache, const void* W_uk, const void* W_uv,
                       const int* seqlens, const int* qpos, void* out, float* lse, int B, int H, int hd,
                       int dc, int Lmax, int window, const float* alibi_slopes, int dtype, void* workspace,
                       size_t ws_bytes, void* stream) {
  int st = check_common(H, 1, hd, dtype, 0.f);
  if (st) return st;
  if (!q || !ccache || !W_uk || !W_uv || !seqlens || !qpos || !out)
    return fail(ATTN_ERR_ARG, "q, ccache, W_uk, W_uv, seqlens, qpos and out must not be NULL");
  if (!aligned16(q) || !aligned16(ccache) || !aligned16(W_uk) || !aligned16(W_uv) || !aligned16(out) ||
      (lse && !aligned16(lse)) || (workspace && !aligned16(workspace)))
    return fail(ATTN_ERR_ALIGN, "q, ccache, weights, out, lse and workspace must be 16-byte aligned");
  if (B < 1 || Lmax < 1 || Lmax >= (1 << 24)) return fail(ATTN_ERR_ARG, "B >= 1 and 1 <= Lmax < 2^24");
  if (dtype != ATTN_BF16 || (dc != 64 && dc != 128) || H > 32 || hd % 8)
    return fail(ATTN_ERR_UNSUPPORTED, "attn_decode_latent runs bf16 with dc 64 or 128, H <= 32 and hd % 8 == 0");
  if (window < 0) window = 0;
  const size_t need = attn_decode_latent_workspace_size(B, H, hd, dc, Lmax);
  if (!workspace || ws_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "latent decode needs %zu bytes of workspace (got %zu)", need, ws_bytes);
  char* ws = static_cast<char*>(workspace);
  const size_t vec = r256((size_t)B * H * dc * 2);
  void* qlat = ws;
  void* dws = ws + vec;

  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = qlat; p.kcache = ccache; p.vcache = ccache;  // keys and values are the same latents
  p.seqlens = seqlens; p.qpos = qpos; p.out = out; p.lse = lse;
  p.W_out = W_uv; p.hd_out = hd;  // the merge applies the value up-projection
  p.B = B; p.H = H; p.KV = 1; p.hd = dc; p.Lmax = Lmax; p.window = window;
  p.scale = (float)(1.0 / std::sqrt((double)hd));  // the scores are q . k of head dimension hd
  p.rope = make_rope(dc, 0.f);                      // no rotation on the latent path
  if ((st = make_alibi(H, alibi_slopes, &p.alibi))) return st;
  if (!decode_tc_supported(p, dtype)) return fail(ATTN_ERR_UNSUPPORTED, "latent decode kernel unavailable");
  int err = 0;
  p.status = device_status(&err);
  if (!p.status) return err;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_latent_fold(q, W_uk, qlat, B, H, dc, hd, s);
  if (e == cudaSuccess) e = launch_decode(p, dtype, dws, s);
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode_latent launch");
  return ok();
}

int attn_kv_write(const void* k_new, const void* v_new, void* kcache, void* vcache, const int* pos0,
                  int B, int Tn, int KV, int hd, int Lmax, float rope_base, int dtype, void* stream) {
  int st = check_common(KV, KV, hd, dtype, rope_base);
  if (st) return st;
  if (!k_new || !v_new || !kcache || !vcache || !pos0)
    return fail(ATTN_ERR_ARG, "k_new, v_new, kcache, vcache and pos0 must not be NULL");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kcache) || !aligned16(vcache))
    return fail(ATTN_ERR_ALIGN, "k_new, v_new and the caches must be 16-byte aligned");
  if (B < 1 || B > 0x7fffffff || Tn < 1 || Tn > 65535 || Lmax < 1 || Lmax >= (1 << 24))
    return fail(ATTN_ERR_ARG, "B >= 1, 1 <= Tn <= 65535 and 1 <= Lmax < 2^24");
  AppendParams p;
  std::memset(&p, 0, sizeof(p));
  p.k_new = k_new; p.v_new = v_new; p.kcache = kcache; p.vcache = vcache; p.pos = pos0;
  p.B = B; p.Tn = Tn; p.KV = KV; p.hd = hd; p.Lmax = Lmax;
  p.rope = make_rope(hd, rope_base);
  int err = 0;
  p.status = device_status(&err);
  if (!p.status) return err;
  cudaError_t e = launch_kv_append(p, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_kv_write launch");
  return ok();
}

namespace {
size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
struct BlockLayout {
  size_t q, k, v, ctx, cs, total;
};
BlockLayout block_layout(int B, int T, int H, int KV, int hd, int dtype) {
  const size_t es = elem_size(dtype);
  BlockLayout L;
  const size_t nq = (size_t)B * T * H * hd * es, nk = (size_t)B * T * KV * hd * es;
  L.q = 0;
  L.k = L.q + round256(nq);
  L.v = L.k + round256(nk);
  L.ctx = L.v + round256(nk);
  L.cs = L.ctx + round256(nq);
  L.total = L.cs + round256((size_t)T * (hd / 2) * sizeof(float2));
  return L;
}
cudaError_t gemm(const void* A, const void* W, void* C, int M, int N, int K, int dtype, int* status,
               cudaStream_t s) {
  if (gemm_tc_supported(M, N, K, dtype)) return launch_gemm_tc(A, W, C, M, N, K, status, s);
  return launch_gemm_simt(A, W, C, M, N, K, dtype, s);
}
// The attention of the blocks: attn_prefill's launch, optionally over keys that the projection
// epilogue already turned (k_rotated).
int block_attention(const void* q, const void* k, const void* v, void* out, int B, int T, int H, int KV, int hd,
                    long long pos0, float rope_base, int causal, int window, const float* alibi_slopes,
                    int dtype, int k_rotated, int* status, cudaStream_t s) {
  PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.k = k; p.v = v; p.out = out;
  p.B = B; p.T = T; p.H = H; p.KV = KV; p.hd = hd;
  p.pos0 = (int)pos0; p.causal = causal; p.window = window < 0 ? 0 : window;
  p.scale = (float)(1.0 / std::sqrt((double)hd));
  p.rope = make_rope(hd, rope_base);
  p.k_rotated = k_rotated;
  p.status = status;
  int st;
  if ((st = make_alibi(H, alibi_slopes, &p.alibi))) return st;
  cudaError_t e = prefill_tc_supported(p, dtype) ? launch_prefill_tc(p, s) : launch_prefill_simt(p, dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "block attention launch");
  return ATTN_OK;
}
}  // namespace

size_t attn_block_workspace_size(int B, int T, int d, int H, int KV, int hd, int dtype) {
  if (B < 1 || T < 1 || d < 1 || H < 1 || KV < 1 || H % KV || hd < 2 ||
      (dtype != ATTN_F32 && dtype != ATTN_BF16))
    return 0;
  return block_layout(B, T, H, KV, hd, dtype).total;
}

int attn_block(const void* x, const void* Wq, const void* Wk, const void* Wv, const void* Wo,
               void* out, int B, int T, int d, int H, int KV, int hd, long long pos0,
               float rope_base, int causal, int window, const float* alibi_slopes, int dtype,
               void* workspace, size_t ws_bytes, void* stream) {
  int st = check_common(H, KV, hd, dtype, rope_base);
  if (st) return st;
  if (!x || !Wq || !Wk || !Wv || !Wo || !out)
    return fail(ATTN_ERR_ARG, "x, Wq, Wk, Wv, Wo and out must not be NULL");
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(Wo) ||
      !aligned16(out) || (workspace && !aligned16(workspace)))
    return fail(ATTN_ERR_ALIGN, "x, weights, out and workspace must be 16-byte aligned");
  if (B < 1 || T < 1 || d < 1) return fail(ATTN_ERR_ARG, "B, T and d must be >= 1");
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_ARG, "causal must be 0 or 1");
  if (window < 0) window = 0;
  if (window > 0 && !causal) return fail(ATTN_ERR_ARG, "a window requires the causal mask");
  if (pos0 < 0 || pos0 + (long long)T >= (1LL << 24))
    return fail(ATTN_ERR_ARG, "positions pos0..pos0+T-1 must lie in [0, 2^24)");
  const size_t need = attn_block_workspace_size(B, T, d, H, KV, hd, dtype);
  if (!workspace || ws_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "block needs %zu bytes of workspace (got %zu)", need, ws_bytes);
  const BlockLayout L = block_layout(B, T, H, KV, hd, dtype);
  char* ws = static_cast<char*>(workspace);
  void *q = ws + L.q, *k = ws + L.k, *v = ws + L.v, *ctx = ws + L.ctx;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int M = B * T;
  int err = 0;
  int* status = device_status(&err);
  if (!status) return err;
  cudaError_t e;
  int k_rotated = 0;
  const int Ns[3] = {H * hd, KV * hd, KV * hd};
  if (gemm_tc_supported(M, H * hd, d, dtype) && gemm_tc_supported(M, KV * hd, d, dtype) &&
      gemm_tc_segments_fit(3, Ns)) {
    // x @ Wq, x @ Wk and x @ Wv as one launch over the three weights side by side; the keys
    // are turned in its epilogue (q, turned once per query tile, is left to the attention)
    const RopeFreqs rope = make_rope(hd, rope_base);
    GemmEpilogue ep;
    std::memset(&ep, 0, sizeof(ep));
    ep.rot_seg = -1;
    if (rope.on && (hd == 64 || hd == 128)) {
      float2* cs = reinterpret_cast<float2*>(ws + L.cs);
      if ((e = launch_rope_table(cs, T, (int)pos0, rope, hd, s)) != cudaSuccess) return cuda_fail(e, "block table");
      ep.rot_seg = 1;
      ep.rope_cs = cs;
      ep.T = T;
      ep.hd = hd;
      k_rotated = 1;
    }
    const void* Ws[3] = {Wq, Wk, Wv};
    void* Cs[3] = {q, k, v};
    if ((e = launch_gemm_tc_multi(x, 3, Ws, Cs, Ns, M, d, status, s, &ep)) != cudaSuccess)
      return cuda_fail(e, "block QKV GEMM");
  } else {
    if ((e = gemm(x, Wq, q, M, H * hd, d, dtype, status, s)) != cudaSuccess) return cuda_fail(e, "block Wq GEMM");
    if ((e = gemm(x, Wk, k, M, KV * hd, d, dtype, status, s)) != cudaSuccess) return cuda_fail(e, "block Wk GEMM");
    if ((e = gemm(x, Wv, v, M, KV * hd, d, dtype, status, s)) != cudaSuccess) return cuda_fail(e, "block Wv GEMM");
  }
  st = block_attention(q, k, v, ctx, B, T, H, KV, hd, pos0, rope_base, causal, window, alibi_slopes, dtype,
                       k_rotated, status, s);
  if (st) return st;
  if ((e = gemm(ctx, Wo, out, M, d, H * hd, dtype, status, s)) != cudaSuccess) return cuda_fail(e, "block Wo GEMM");
  return ok();
}

namespace {
struct FusedLayout {
  size_t wg, rinv, q, k, v, ctx, cs, total;
};
FusedLayout fused_layout(int B, int T, int d, int H, int KV, int hd) {
  FusedLayout L;
  const size_t M = (size_t)B * T;
  L.wg = 0;
  L.rinv = L.wg + round256((size_t)d * (H + 2 * KV) * hd * 2);
  L.q = L.rinv + round256(M * sizeof(float));
  L.k = L.q + round256(M * H * hd * 2);
  L.v = L.k + round256(M * KV * hd * 2);
  L.ctx = L.v + round256(M * KV * hd * 2);
  L.cs = L.ctx + round256(M * H * hd * 2);
  L.total = L.cs + round256((size_t)T * (hd / 2) * sizeof(float2));
  return L;
}
}  // namespace

size_t attn_block_fused_workspace_size(int B, int T, int d, int H, int KV, int hd) {
  if (B < 1 || T < 1 || d < 1 || H < 1 || KV < 1 || H % KV || hd < 2) return 0;
  return fused_layout(B, T, d, H, KV, hd).total;
}

int attn_block_fused(const void* x, const void* gamma, const void* Wqkv, const void* Wo, void* out,
                     void* kcache, void* vcache, int Lmax, int B, int T, int d, int H, int KV, int hd,
                     long long pos0, float rope_base, int causal, int window, const float* alibi_slopes,
                     float eps, int dtype, void* workspace, size_t ws_bytes, void* stream) {
  int st = check_common(H, KV, hd, dtype, rope_base);
  if (st) return st;
  if (!x || !Wqkv || !Wo || !out) return fail(ATTN_ERR_ARG, "x, Wqkv, Wo and out must not be NULL");
  if ((kcache == nullptr) != (vcache == nullptr)) return fail(ATTN_ERR_ARG, "give both caches or neither");
  if (!aligned16(x) || (gamma && !aligned16(gamma)) || !aligned16(Wqkv) || !aligned16(Wo) || !aligned16(out) ||
      (kcache && (!aligned16(kcache) || !aligned16(vcache))) || (workspace && !aligned16(workspace)))
    return fail(ATTN_ERR_ALIGN, "tensors and workspace must be 16-byte aligned");
  if (B < 1 || T < 1 || d < 8 || d % 8) return fail(ATTN_ERR_ARG, "B, T >= 1 and d a multiple of 8");
  if (!std::isfinite(eps) || eps < 0.f) return fail(ATTN_ERR_ARG, "eps must be finite and >= 0");
  if (causal != 0 && causal != 1) return fail(ATTN_ERR_ARG, "causal must be 0 or 1");
  if (window < 0) window = 0;
  if (window > 0 && !causal) return fail(ATTN_ERR_ARG, "a window requires the causal mask");
  if (pos0 < 0 || pos0 + (long long)T >= (1LL << 24))
    return fail(ATTN_ERR_ARG, "positions pos0..pos0+T-1 must lie in [0, 2^24)");
  if (kcache && (Lmax < 1 || pos0 + (long long)T > Lmax))
    return fail(ATTN_ERR_ARG, "the cache must hold slots pos0..pos0+T-1 (Lmax=%d)", Lmax);
  const int M = B * T, Nqkv = (H + 2 * KV) * hd;
  if ((long long)B * T * (H + 2 * KV) * hd >= (1LL << 40) || (long long)B * T * d >= (1LL << 40))
    return fail(ATTN_ERR_ARG, "tensor too large");
  const int Ns[3] = {H * hd, KV * hd, KV * hd};
  if (dtype != ATTN_BF16 || (hd != 64 && hd != 128) || !gemm_tc_supported(M, H * hd, d, dtype) ||
      !gemm_tc_supported(M, KV * hd, d, dtype) || !gemm_tc_segments_fit(3, Ns) ||
      !gemm_tc_supported(M, d, H * hd, dtype))
    return fail(ATTN_ERR_UNSUPPORTED,
                "attn_block_fused runs bf16 with hd 64 or 128 on the tensor-core GEMM");
  const FusedLayout L = fused_layout(B, T, d, H, KV, hd);
  if (!workspace || ws_bytes < L.total)
    return fail(ATTN_ERR_WORKSPACE, "fused block needs %zu bytes of workspace (got %zu)", L.total, ws_bytes);
  int err = 0;
  int* status = device_status(&err);
  if (!status) return err;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const RopeFreqs rope = make_rope(hd, rope_base);
  float2* cs = reinterpret_cast<float2*>(ws + L.cs);
  float* rinv = reinterpret_cast<float*>(ws + L.rinv);
  // RMSNorm folded into the projection: 1 / rms per row, gamma into the weights' rows (here,
  // or once by the caller through attn_fold_rmsnorm_gamma, then gamma is NULL)
  cudaError_t e = cudaSuccess;
  if (rope.on) e = launch_rope_table(cs, T, (int)pos0, rope, hd, s);
  if (e == cudaSuccess) e = launch_rms_inverse(x, rinv, M, d, eps, s);
  if (e == cudaSuccess && gamma) e = launch_fold_gamma(Wqkv, gamma, ws + L.wg, d, Nqkv, s);
  if (e != cudaSuccess) return cuda_fail(e, "fused block norm");
  // (x @ [Wq | Wk | Wv] with gamma folded) / rms, the keys turned, k and v also into the cache
  GemmEpilogue qkv;
  std::memset(&qkv, 0, sizeof(qkv));
  qkv.row_scale = rinv;
  qkv.rot_seg = rope.on ? 1 : -1;
  qkv.rope_cs = rope.on ? cs : nullptr;
  qkv.T = T;
  qkv.hd = hd;
  qkv.cache[1] = kcache;
  qkv.cache[2] = vcache;
  qkv.Lmax = Lmax;
  qkv.pos0 = (int)pos0;
  const char* wg = gamma ? ws + L.wg : static_cast<const char*>(Wqkv);
  const void* Ws[3] = {wg, wg + (size_t)H * hd * 2, wg + (size_t)(H + KV) * hd * 2};
  void* Cs[3] = {ws + L.q, ws + L.k, ws + L.v};
  if ((e = launch_gemm_tc_multi(x, 3, Ws, Cs, Ns, M, d, status, s, &qkv, Nqkv)) != cudaSuccess)
    return cuda_fail(e, "fused block QKV GEMM");
  // the keys arrive turned: the attention turns only q (its masks and ALiBi depend on i - j)
  st = block_attention(ws + L.q, ws + L.k, ws + L.v, ws + L.ctx, B, T, H, KV, hd, pos0, rope_base, causal,
                       window, alibi_slopes, dtype, 1, status, s);
  if (st) return st;
  GemmEpilogue res;
  std::memset(&res, 0, sizeof(res));
  res.mode = 2;
  res.rot_seg = -1;
  res.residual = x;
  if ((e = launch_gemm_tc(ws + L.ctx, Wo, out, M, d, H * hd, status, s, &res)) != cudaSuccess)
    return cuda_fail(e, "fused block Wo GEMM");
  return ok();
}

int attn_fold_rmsnorm_gamma(const void* gamma, const void* W, void* Wg, int d, int N, void* stream) {
  if (!gamma || !W || !Wg) return fail(ATTN_ERR_ARG, "gamma, W and Wg must not be NULL");
  if (!aligned16(gamma) || !aligned16(W) || !aligned16(Wg)) return fail(ATTN_ERR_ALIGN, "16-byte alignment");
  if (d < 1 || N < 8 || N % 8 || (long long)d * N >= (1LL << 40))
    return fail(ATTN_ERR_ARG, "d >= 1 and N a positive multiple of 8 (d=%d, N=%d)", d, N);
  cudaError_t e = launch_fold_gamma(W, gamma, Wg, d, N, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_fold_rmsnorm_gamma launch");
  return ok();
}

void attn_alibi_slopes(int H, float* host_out) {
  if (!host_out || H < 1) return;
  for (int h = 0; h < H; ++h) host_out[h] = (float)std::pow(2.0, -8.0 * (h + 1.0) / H);
}

int attn_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_sync_status: stream synchronise");
  int err = 0;
  int* ptr = device_status(&err);
  if (!ptr) return err;
  int word = 0;
  if ((e = cudaMemcpy(&word, ptr, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "attn_sync_status: read");
  if (word != 0) {
    const int zero = 0;
    if ((e = cudaMemcpy(ptr, &zero, sizeof(int), cudaMemcpyHostToDevice)) != cudaSuccess)
      return cuda_fail(e, "attn_sync_status: clear");
  }
  if (word == DEV_TIMEOUT) return fail(ATTN_ERR_TIMEOUT, "a device-side wait gave up");
  if (word == DEV_BAD_ARG)
    return fail(ATTN_ERR_DEVICE_ARG, "a device-resident length or position was out of range");
  return ok();
}

int attn_last_error(char* buf, size_t n) {
  if (buf && n) {
    std::strncpy(buf, g_msg, n - 1);
    buf[n - 1] = '\0';
  }
  return g_last;
}

const char* attn_version(void) { return "alibi_rope_tile_b200 0.1 (sm_100a)"; }

}  // extern "C"
