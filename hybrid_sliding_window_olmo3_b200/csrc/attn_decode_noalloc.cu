// olmo3_attn_decode_noalloc: the split-KV decode of olmo3_attn_decode, with its
// partials kept in a fixed buffer that the library itself holds, for callers
// that cannot allocate device memory (see include/olmo3.h).
//
// The buffer is a file-scope __device__ array.  In host code its name is only a
// host-side stand-in, not a device address, so the entry point asks the runtime
// for the real address (cudaGetSymbolAddress) once per device, with that device
// current, and passes that pointer to the kernels.  Nothing here allocates.
#include <mutex>

#include "internal.h"
#include "olmo3.h"

namespace {

constexpr size_t kScratchBytes = OLMO3_NOALLOC_SCRATCH_BYTES;

// Lives on every device that loads this library, until the process exits.
static __device__ __align__(256) float g_decode_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per device).
int scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return OLMO3_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return OLMO3_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return OLMO3_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return OLMO3_OK;
}

}  // namespace

extern "C" int olmo3_attn_decode_noalloc(const void *q, int H, const olmo3_kv_cache *c, const int32_t *kv_len,
                                         int max_kv_len, void *out, float *lse_out, float scale, int num_splits,
                                         int *err_dev, void *stream) {
  if (c != nullptr) {
    const size_t need =
        olmo3_attn_decode_workspace_size(c->B, H, c->G, c->d, max_kv_len, c->layer_type, c->window, num_splits);
    if (need > kScratchBytes) return OLMO3_ERR_WORKSPACE;  // beyond the built-in buffer: nothing launched
  }
  void *scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != OLMO3_OK) return st;
  // Every partial the combine reads is written earlier in the same call, so the
  // previous call's contents never need clearing.
  return olmo3_attn_decode(q, H, c, kv_len, max_kv_len, out, lse_out, scale, num_splits, scratch, kScratchBytes,
                           err_dev, stream);
}
