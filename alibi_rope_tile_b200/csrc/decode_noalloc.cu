// attn_decode_noalloc: the decode step for callers that cannot allocate device memory
// (declared in include/attn_rope_tile.h). The split partials go to a fixed scratch array
// in the library's device image instead of a caller workspace; the kernels are the ones
// attn_decode runs.
#include <cstdio>
#include <mutex>

#include "attn_rope_tile.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = ATTN_DECODE_NOALLOC_MAX_SCRATCH;

// One array per device that loads the library, kept until the process exits. Host code
// must not pass its name to a kernel (on the host it only stands in for the symbol); the
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device, looked up on the first call
// made with that device current and cached after that.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return attn::record_error(ATTN_ERR_CUDA, "attn_decode_noalloc: no usable current device");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || !ptr) {
      char msg[256];
      std::snprintf(msg, sizeof(msg), "attn_decode_noalloc: cudaGetSymbolAddress failed: %s",
                    cudaGetErrorString(e));
      return attn::record_error(ATTN_ERR_CUDA, msg);
    }
    g_scratch[dev] = ptr;
  }
  *out = g_scratch[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                   const int* seqlens, const int* qpos, void* out, float* lse,
                                   int B, int H, int KV, int hd, int Lmax, float rope_base,
                                   int window, const float* alibi_slopes, int dtype,
                                   void* stream) {
  const size_t need = attn_decode_workspace_size(B, H, KV, hd, Lmax);
  if (need > kScratchBytes) {
    char msg[256];
    std::snprintf(msg, sizeof(msg),
                  "attn_decode_noalloc: these sizes need %zu bytes of scratch, above its fixed "
                  "maximum of %zu bytes; call attn_decode with a workspace instead",
                  need, kScratchBytes);
    return attn::record_error(ATTN_ERR_UNSUPPORTED, msg);
  }
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != ATTN_OK) return st;
  // attn_decode validates every other argument; it allocates nothing either.
  return attn_decode(q, kcache, vcache, seqlens, qpos, out, lse, B, H, KV, hd, Lmax, rope_base,
                     window, alibi_slopes, dtype, scratch, kScratchBytes, stream);
}
