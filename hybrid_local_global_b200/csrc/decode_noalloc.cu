// decode_noalloc.cu -- gemma_attn_decode for callers that cannot allocate
// device memory.
//
// Some callers of the decode step have no way to obtain device memory for
// the split-K workspace: a plugin hosted by a runtime that owns all device
// memory and exposes no allocator to it, or a latency-critical loop in
// which a cudaMalloc (with its implicit device-wide synchronisation) is not
// acceptable and no pool was planned ahead. This entry point serves them
// from a fixed scratch array compiled into the library instead.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes
// (32 MiB). Every GPU on which the library's device code is loaded holds it
// until the process exits, whether or not this entry point is used.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace hlg {
int record_error(int code, const char* msg);  // api.cu: sets gemma_last_error()
}

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[128] = {nullptr};

// Device address of the scratch array on the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device with that device current and kept for the life of the
// process; a device reset may move the array, so the header asks processes
// that reset a device not to call this entry point on it again.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hlg::record_error(GEMMA_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= 128) return hlg::record_error(GEMMA_ERR_UNSUPPORTED, "device ordinal >= 128");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      char msg[256];
      snprintf(msg, sizeof msg, "scratch set-up (cudaGetSymbolAddress) failed: %s", cudaGetErrorString(e));
      return hlg::record_error(GEMMA_ERR_CUDA, msg);
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return GEMMA_OK;
}

}  // namespace

extern "C" int gemma_attn_decode_noalloc(const void* q, const void* k_new, const void* v_new,
                                         void* k_cache, void* v_cache, int cache_cap,
                                         const int32_t* seq_lens, int max_seq_len, int batch,
                                         int window, int n_q_heads, int n_kv_heads, int head_dim,
                                         float rope_frac, float rope_theta, float scale, void* out,
                                         unsigned flags, void* stream) {
  const size_t need = gemma_attn_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, window,
                                                       max_seq_len);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "gemma_attn_decode_noalloc: this call needs %zu bytes of scratch, more than the fixed "
             "%zu; use gemma_attn_decode with a caller-allocated workspace",
             need, kNoAllocScratchBytes);
    return hlg::record_error(GEMMA_ERR_CAPACITY, msg);
  }
  void* ws = nullptr;
  int rc = noalloc_scratch(&ws);
  if (rc != GEMMA_OK) return rc;
  return gemma_attn_decode(q, k_new, v_new, k_cache, v_cache, cache_cap, seq_lens, max_seq_len, batch,
                           window, n_q_heads, n_kv_heads, head_dim, rope_frac, rope_theta, scale, out,
                           ws, kNoAllocScratchBytes, flags, stream);
}
