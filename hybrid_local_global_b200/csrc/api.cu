// api.cu -- the extern "C" entry points of libgemma_attn.so: argument
// validation, workspace planning, launches, the device status word and the
// host-only KV-share binding. Declarations and contracts: gemma_attn.h.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstddef>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "kernels.h"

using namespace hlg;

namespace {

thread_local std::string t_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

int succeed() {
  t_err.clear();
  return GEMMA_OK;
}

__device__ DevStatus g_dev;  // device status block (see common.cuh)

std::mutex g_mu;
int* g_status_ptr[128] = {nullptr};
int g_sm_count[128] = {0};
std::atomic<long long> g_wait_ns{1000000000LL};
std::atomic<int> g_drop_next{0};

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Device address of g_status for the current device (looked up once).
int* status_ptr() {
  int dev = current_device();
  if (dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = &static_cast<DevStatus*>(p)->status;
  }
  return g_status_ptr[dev];
}

int sm_count() {
  int dev = current_device();
  if (dev < 0 || dev >= 128) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

// Measurement hook state (gemma_attn_profile): event pairs around launches.
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::vector<ProfRec> g_prof;
std::atomic<bool> g_prof_on{false};

struct ProfScope {
  ProfRec rec{-1, nullptr, nullptr};
  cudaStream_t st;
  ProfScope(int kind, cudaStream_t s) : st(s) {
    if (!g_prof_on.load()) return;
    if (cudaEventCreate(&rec.a) != cudaSuccess || cudaEventCreate(&rec.b) != cudaSuccess) return;
    rec.kind = kind;
    cudaEventRecord(rec.a, st);
  }
  void done() {
    if (rec.kind < 0) return;
    cudaEventRecord(rec.b, st);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back(rec);
    rec.kind = -1;
  }
};

void prof_clear() {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  g_prof.clear();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_heads(int Hq, int Hkv, int D, int window, float rope_frac, float rope_theta, float scale) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv)
    return fail(GEMMA_ERR_INVALID_ARG, "n_q_heads (%d) must be a positive multiple of n_kv_heads (%d)", Hq, Hkv);
  if (Hq / Hkv > 8)
    return fail(GEMMA_ERR_UNSUPPORTED, "query heads per KV head %d > 8", Hq / Hkv);
  if (D != 256 && D != 512) return fail(GEMMA_ERR_UNSUPPORTED, "head_dim %d (supported: 256, 512)", D);
  if (window < 0 || window % 16)
    return fail(GEMMA_ERR_INVALID_ARG, "window %d must be 0 or a positive multiple of 16", window);
  if (!(rope_frac >= 0.f && rope_frac <= 1.f))
    return fail(GEMMA_ERR_INVALID_ARG, "rope_frac %g outside [0, 1]", (double)rope_frac);
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta))
    return fail(GEMMA_ERR_INVALID_ARG, "rope_theta %g must be positive and finite", (double)rope_theta);
  if (!std::isfinite(scale)) return fail(GEMMA_ERR_INVALID_ARG, "scale must be finite");
  return GEMMA_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(GEMMA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Split-K plan of a decode call: keys per split (a multiple of 16) and splits
// per (sequence, KV head). Each unit is one CTA and two fit on an SM, so with
// lengths near keys_max a call takes about (waves of units) x (keys per unit
// + a fixed cost per unit). Long ranges aim at ~2048 keys per unit with the
// unit count rounded up to whole waves. Ranges that fit in one such unit (a
// local layer's ring) instead take the split count, 1 to 4 with at least 256
// keys per unit, that minimises that cost: a batch of 64 sequences x 16 KV
// heads is 3.46 waves of whole rings but 6.92 waves of half rings.
void decode_plan(int B, int Hkv, int window, int max_len, int* chunk, int* n_splits) {
  const int64_t keys_max = window > 0 ? std::min<int64_t>(max_len, window) : max_len;
  const int64_t pairs = (int64_t)B * Hkv;
  const int64_t wave = (int64_t)sm_count() * 2;
  const auto up16 = [](int64_t x) { return ((x + 15) / 16) * 16; };
  int64_t units = (keys_max * pairs + 2047) / 2048;
  units = ((units + wave - 1) / wave) * wave;
  int64_t c = (keys_max * pairs + units - 1) / units;
  c = std::max<int64_t>(up16(c), 256);
  if (c >= keys_max) {
    constexpr int64_t kUnitCost = 128;  // per-unit fixed cost, in keys streamed
    int64_t best_cost = INT64_MAX;
    c = up16(keys_max);
    for (int64_t ns = 1; ns <= 4; ++ns) {
      const int64_t cc = up16((keys_max + ns - 1) / ns);
      if (ns > 1 && cc < 256) break;
      if ((keys_max + cc - 1) / cc != ns) continue;  // same plan as a smaller count
      const int64_t cost = ((pairs * ns + wave - 1) / wave) * (cc + kUnitCost);
      if (cost < best_cost) {
        best_cost = cost;
        c = cc;
      }
    }
  }
  *chunk = (int)c;
  *n_splits = (int)((keys_max + c - 1) / c);
}

size_t decode_ws_parts(int B, int Hq, int Hkv, int D, int n_splits, size_t* off_lse, size_t* off_o,
                       size_t* off_kst = nullptr) {
  size_t q = align256((size_t)B * Hq * D * 2);
  size_t lse = align256((size_t)B * Hq * n_splits * 4);
  size_t o = align256((size_t)B * Hq * n_splits * D * 4);
  size_t kst = align256((size_t)B * Hkv * D * 2);  // int8 cache: the rotated new key before quantization
  if (off_kst) *off_kst = q + lse + o;
  *off_lse = q;
  *off_o = q + lse;
  return q + lse + o + kst;
}

// Prefill workspace: rotated Q, then on local layers either the rotated K
// of the chunk (K at off_k) or, for a chunk after cached tokens, the K and V
// windows of window + S rows (K at off_k, V at *off_vw).
size_t prefill_ws_parts(int B, int S, int Hq, int Hkv, int D, int window, size_t* off_k,
                        size_t* off_vw = nullptr, int prefix_rows = 0) {
  size_t q = align256((size_t)B * S * Hq * D * 2);
  // rotated K of the chunk: local layers, and global layers with an int8 cache
  size_t k = align256((size_t)B * S * Hkv * D * 2);
  // K and V windows: chunked local prefill (window + S rows), or the
  // dequantized prefix plus chunk of an int8 global layer (prefix_rows rows)
  size_t win = window > 0     ? align256((size_t)B * (window + S) * Hkv * D * 2)
               : prefix_rows ? align256((size_t)B * prefix_rows * Hkv * D * 2)
                             : 0;
  *off_k = q;
  if (off_vw) *off_vw = q + win;
  return q + std::max(k, 2 * win);
}

// Multi-token decode on the tensor-core kernels (bf16 caches): a global
// layer (contiguous or paged) whose G q heads x tokens rows fit one 128-row
// tile, or an unshared local layer with at most 64 such rows and
// tokens <= window.
bool verify_fast(int tokens, int window, int n_q_heads, int n_kv_heads, int head_dim, unsigned flags) {
  if ((flags & (GEMMA_F_KV_INT8 | GEMMA_F_SOURCE_WINDOW)) || (head_dim != 256 && head_dim != 512)) return false;
  if (window == 0) return (n_q_heads / n_kv_heads) * tokens <= 128;
  return !(flags & GEMMA_F_SHARED) && tokens <= window && tokens <= 128 &&
         verify_tc_rows(n_q_heads, n_kv_heads, tokens, head_dim) != 0;
}

// Keys per split of the multi-token kernel: a multiple of 128 between 1024
// and 8192, aiming at eight CTAs per SM over the planned length (a CTA's
// fixed cost, the Q tile and the partials, is then a few percent of its
// streaming time). The 128-row-tile kernel runs head_dim / 256 CTAs per KV
// head and split, the transposed one a single CTA.
// A local layer splits its ring only when its B x Hkv CTAs fill fewer than
// two waves.
void verify_plan(int B, int Hq, int Hkv, int tokens, int head_dim, int window, int max_len, int* chunk,
                 int* n_splits) {
  if (window > 0) {
    const int64_t ctas = (int64_t)B * Hkv, wave2 = (int64_t)sm_count() * 2;
    int64_t c = ctas >= wave2 ? window : ((int64_t)window * ctas + wave2 - 1) / wave2;
    c = std::min<int64_t>(((std::max<int64_t>(c, 1) + 127) / 128) * 128, ((window + 127) / 128) * 128);
    *chunk = (int)c;
    *n_splits = (int)((window + c - 1) / c);
    return;
  }
  const int per_head = verify_tc_rows(Hq, Hkv, tokens, head_dim) ? 1 : head_dim / 256;
  const int64_t ctas_per_split = (int64_t)B * Hkv * per_head;
  const int64_t target = (int64_t)sm_count() * 8;
  int64_t c = ((int64_t)max_len * ctas_per_split + target - 1) / target;
  c = ((c + 127) / 128) * 128;
  c = std::min<int64_t>(std::max<int64_t>(c, 1024), 8192);
  *chunk = (int)c;
  *n_splits = (int)((max_len + c - 1) / c);
}

// fast path: rotated Q, split log2-sum-exps, split partial O; local layers
// also the new tokens' rotated keys (the ring is written after attention)
size_t verify_ws_parts(int B, int tokens, int Hq, int Hkv, int D, int window, int n_splits, size_t* off_lse,
                       size_t* off_o, size_t* off_kst) {
  const size_t rows = (size_t)B * tokens * Hq;
  const size_t q = align256(rows * D * 2);
  const size_t lse = align256(rows * n_splits * 4);
  const size_t o = align256(rows * n_splits * D * 4);
  *off_lse = q;
  *off_o = q + lse;
  *off_kst = q + lse + o;
  return q + lse + o + (window > 0 ? align256((size_t)B * tokens * Hkv * D * 2) : 0);
}

// other layers: lengths before the new tokens, then the chunked-prefill workspace
size_t verify_route_ws(int B, int tokens, int Hq, int Hkv, int D, int window, int cache_cap, unsigned flags) {
  size_t off_k;
  const bool prefix = (flags & GEMMA_F_KV_INT8) && window == 0;
  return align256((size_t)B * 4) +
         prefill_ws_parts(B, tokens, Hq, Hkv, D, window, &off_k, nullptr, prefix ? cache_cap : 0);
}

// Multi-token decode on an int8 global layer: the tokens one at a time
// through single-token decode, which is what the call computes (a chunked
// prefill would dequantize the whole cached prefix into the workspace).
// Workspace: per-token lengths, the decode workspace, then one token's q,
// new K and V, and output.
bool verify_by_decode(int window, unsigned flags) { return window == 0 && (flags & GEMMA_F_KV_INT8); }

size_t verify_decode_ws(int B, int Hq, int Hkv, int D, int max_len, size_t* off_dec, size_t* off_q,
                        size_t* off_k, size_t* off_v, size_t* off_o) {
  int chunk, n_splits;
  decode_plan(B, Hkv, 0, max_len, &chunk, &n_splits);
  size_t a, b, o = align256((size_t)B * 4);
  *off_dec = o;
  o += align256(decode_ws_parts(B, Hq, Hkv, D, n_splits, &a, &b));
  *off_q = o;
  o += align256((size_t)B * Hq * D * 2);
  *off_k = o;
  o += align256((size_t)B * Hkv * D * 2);
  *off_v = o;
  o += align256((size_t)B * Hkv * D * 2);
  *off_o = o;
  return o + align256((size_t)B * Hq * D * 2);
}

}  // namespace

namespace hlg {
// Sets the message gemma_last_error() returns on this thread; for entry
// points defined in other translation units of the library.
int record_error(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace hlg

extern "C" {

const char* gemma_last_error(void) { return t_err.c_str(); }

int gemma_attn_set_wait_limit(long long max_ns) {
  if (max_ns < 0) return fail(GEMMA_ERR_INVALID_ARG, "wait limit must be >= 0");
  g_wait_ns.store(max_ns == 0 ? 1000000000LL : max_ns);
  return succeed();
}

int gemma_attn_debug_drop_next_copy(int enable) {
  g_drop_next.store(enable ? 1 : 0);
  return succeed();
}

int gemma_layer_schedule(int n_layers, int ratio, int n_shared, int* is_global, int* share_src) {
  if (n_layers <= 0 || ratio < 0 || n_shared < 0 || n_shared > n_layers || !is_global)
    return fail(GEMMA_ERR_INVALID_ARG, "bad schedule arguments (n_layers %d, ratio %d, n_shared %d)",
                n_layers, ratio, n_shared);
  for (int l = 0; l < n_layers; ++l)
    is_global[l] = (l == n_layers - 1) || ((l + 1) % (ratio + 1) == 0);
  if (share_src) {
    const int first = n_layers - n_shared;
    for (int l = 0; l < n_layers; ++l) {
      if (l < first) {
        share_src[l] = l;
        continue;
      }
      int src = -1;
      for (int s = first - 1; s >= 0; --s)
        if (is_global[s] == is_global[l]) {
          src = s;
          break;
        }
      share_src[l] = src;
    }
  }
  return succeed();
}

// Checks GEMMA_F_SHARED / GEMMA_F_KEQV and the k_new, v_new and v_cache they
// imply. On success *v_cache_io is the cache the values are read from: the
// key cache under K = V.
static int check_kv_flags(unsigned flags, int window, const void* k_new, const void* v_new, void* k_cache,
                          void** v_cache_io) {
  if (flags & ~(GEMMA_F_SHARED | GEMMA_F_KEQV | GEMMA_F_KV_INT8 | GEMMA_F_SOURCE_WINDOW))
    return fail(GEMMA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const bool shared = flags & GEMMA_F_SHARED, keqv = flags & GEMMA_F_KEQV;
  if (keqv && window > 0)
    return fail(GEMMA_ERR_UNSUPPORTED, "GEMMA_F_KEQV: K = V is defined for global layers only");
  if (shared && (k_new || v_new))
    return fail(GEMMA_ERR_INVALID_ARG, "GEMMA_F_SHARED: k_new and v_new must be NULL");
  if (keqv && v_new) return fail(GEMMA_ERR_INVALID_ARG, "GEMMA_F_KEQV: v_new must be NULL (the keys are the values)");
  if (!shared && (!k_new || (!keqv && !v_new)))
    return fail(GEMMA_ERR_INVALID_ARG, "k_new and v_new are required unless GEMMA_F_SHARED (v_new: unless GEMMA_F_KEQV)");
  if (keqv) {
    if (*v_cache_io && *v_cache_io != k_cache)
      return fail(GEMMA_ERR_INVALID_ARG, "GEMMA_F_KEQV: v_cache must be NULL or equal to k_cache");
    *v_cache_io = k_cache;
  }
  return GEMMA_OK;
}

int gemma_kv_share_bind(gemma_kv_desc* dst, const gemma_kv_desc* src) {
  if (!dst || !src) return fail(GEMMA_ERR_INVALID_ARG, "null descriptor");
  if (!src->k_cache || (!src->v_cache && !src->k_eq_v))
    return fail(GEMMA_ERR_INVALID_ARG, "source layer has no cache");
  if (src->layer >= dst->layer)
    return fail(GEMMA_ERR_SHARE_MISMATCH, "source layer %d must precede layer %d", src->layer, dst->layer);
  if ((src->window == 0) != (dst->window == 0))
    return fail(GEMMA_ERR_SHARE_MISMATCH, "layers %d and %d have different attention types", src->layer,
                dst->layer);
  if (src->window != dst->window || src->cache_cap != dst->cache_cap ||
      src->n_kv_heads != dst->n_kv_heads || src->head_dim != dst->head_dim ||
      src->rope_frac != dst->rope_frac || src->rope_theta != dst->rope_theta ||
      (src->k_eq_v != 0) != (dst->k_eq_v != 0) || (src->kv_int8 != 0) != (dst->kv_int8 != 0))
    return fail(GEMMA_ERR_SHARE_MISMATCH,
                "layers %d and %d differ in window, capacity, KV heads, head_dim, RoPE, K = V or int8 KV",
                src->layer, dst->layer);
  dst->k_cache = src->k_cache;
  dst->v_cache = src->v_cache;
  dst->shared_from = src->shared_from >= 0 ? src->shared_from : src->layer;
  return succeed();
}

size_t gemma_kv_codes_bytes(int batch, int n_kv_heads, int cache_cap, int head_dim) {
  if (batch <= 0 || n_kv_heads <= 0 || cache_cap <= 0 || head_dim <= 0) return 0;
  return align256((size_t)batch * n_kv_heads * cache_cap * head_dim);
}

size_t gemma_kv_cache_bytes(int batch, int n_kv_heads, int cache_cap, int head_dim, unsigned flags) {
  if (batch <= 0 || n_kv_heads <= 0 || cache_cap <= 0 || head_dim <= 0) return 0;
  const size_t rows = (size_t)batch * n_kv_heads * cache_cap;
  if (flags & GEMMA_F_KV_INT8) return gemma_kv_codes_bytes(batch, n_kv_heads, cache_cap, head_dim) + rows * 8;
  return rows * head_dim * 2;
}

// int8 cache rows of one call's new tokens: K from the rotated staging rows,
// V from the caller's values (none under K = V)
// Where a layer's cache rows live (see cache_row): a contiguous cache, or
// the pages of a pool named by a page table (global layers).
struct CacheLayout {
  const int32_t* page_table;  // [batch][pages_per_seq], or null
  int page_size, pages_per_seq, n_pages;
};

static CacheLayout contiguous(int cache_cap, int batch) { return CacheLayout{nullptr, cache_cap, 1, batch}; }

// Quantize a chunk's rows into an int8 cache. Sources are [B][rows][Hkv][D]
// with chunk token s at row s (mode 0), window + s (1) or its position (2);
// V from the caller's layout [B][S][Hkv][D] (null under K = V).
static cudaError_t quantize_kv(const bf16* k_src, int k_rows, int k_mode, const bf16* v_src, void* k_cache,
                               void* v_cache, int batch, int S, int Hkv, int D, int window, int cache_cap,
                               const int32_t* pos0, int pos0_minus, const CacheLayout& L, int* status,
                               cudaStream_t st) {
  // an int8 pool is laid out as an int8 cache of n_pages "sequences" of page_size rows
  const size_t off = gemma_kv_codes_bytes(L.n_pages, Hkv, L.page_size, D);
  QuantRowsArgs qa{};
  qa.page_table = L.page_table;
  qa.page_size = L.page_size;
  qa.pages_per_seq = L.pages_per_seq;
  qa.n_pages = L.n_pages;
  qa.src_rows = k_rows;
  qa.src_row_mode = k_mode;
  qa.S = S;
  qa.Hkv = Hkv;
  qa.window = window;
  qa.cache_cap = cache_cap;
  qa.pos0 = pos0;
  qa.pos0_minus = pos0_minus;
  qa.status = status;
  qa.src = k_src;
  qa.codes = static_cast<uint8_t*>(k_cache);
  qa.params = reinterpret_cast<float2*>(static_cast<uint8_t*>(k_cache) + off);
  cudaError_t e = launch_quantize_rows(qa, batch, D, st);
  if (e != cudaSuccess || !v_src) return e;
  qa.src = v_src;
  qa.src_rows = S;
  qa.src_row_mode = 0;
  qa.codes = static_cast<uint8_t*>(v_cache);
  qa.params = reinterpret_cast<float2*>(static_cast<uint8_t*>(v_cache) + off);
  return launch_quantize_rows(qa, batch, D, st);
}

size_t gemma_attn_prefill_workspace_size(int batch, int s_new, int n_q_heads, int n_kv_heads,
                                         int head_dim, int window) {
  if (batch <= 0 || s_new <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0) return 0;
  size_t off_k;
  return prefill_ws_parts(batch, s_new, n_q_heads, n_kv_heads, head_dim, window, &off_k);
}

size_t gemma_attn_prefill_workspace_size_cached(int batch, int s_new, int n_q_heads, int n_kv_heads,
                                                int head_dim, int window, int cache_cap, unsigned flags) {
  if (batch <= 0 || s_new <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || cache_cap <= 0)
    return 0;
  size_t off_k;
  const bool prefix = (flags & GEMMA_F_KV_INT8) && window == 0;
  return prefill_ws_parts(batch, s_new, n_q_heads, n_kv_heads, head_dim, window, &off_k, nullptr,
                          prefix ? cache_cap : 0);
}

static int check_paged(const int32_t* page_table, int page_size, int pages_per_seq, int n_pages) {
  if (!page_table) return fail(GEMMA_ERR_INVALID_ARG, "paged cache: null page table");
  if (page_size <= 0 || page_size % 128)
    return fail(GEMMA_ERR_INVALID_ARG, "paged cache: page_size %d must be a positive multiple of 128", page_size);
  if (pages_per_seq <= 0 || n_pages <= 0)
    return fail(GEMMA_ERR_INVALID_ARG, "paged cache: pages_per_seq %d, n_pages %d", pages_per_seq, n_pages);
  if ((int64_t)pages_per_seq * page_size > INT32_MAX)
    return fail(GEMMA_ERR_INVALID_ARG, "paged cache: pages_per_seq * page_size exceeds 2^31");
  return GEMMA_OK;
}

static int prefill_impl(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                        int cache_cap, const int32_t* seq_lens_before, int batch, int s_new, int window,
                        int n_q_heads, int n_kv_heads, int head_dim, float rope_frac, float rope_theta,
                        float scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                        unsigned flags, void* stream, const CacheLayout& L,
                        const int32_t* lens_after = nullptr) {
  // lens_after (multi-token decode): lengths including the chunk; once the
  // arguments have passed, seq_lens_before (then a device buffer of batch
  // ints) receives lens_after - s_new
  int rc = check_heads(n_q_heads, n_kv_heads, head_dim, window, rope_frac, rope_theta, scale);
  if (rc) return rc;
  rc = check_kv_flags(flags, window, k_new, v_new, k_cache, &v_cache);
  if (rc) return rc;
  if (batch <= 0 || s_new < 0) return fail(GEMMA_ERR_INVALID_ARG, "batch %d, s_new %d", batch, s_new);
  const bool shared = flags & GEMMA_F_SHARED;
  const bool q8 = flags & GEMMA_F_KV_INT8;
  const bool keqv = flags & GEMMA_F_KEQV;
  const bool src_win = flags & GEMMA_F_SOURCE_WINDOW;
  if (q8) {
    if (cache_cap % 2) return fail(GEMMA_ERR_INVALID_ARG, "int8 KV: cache_cap %d must be even", cache_cap);
  }
  if (src_win && (window == 0 || !seq_lens_before))
    return fail(GEMMA_ERR_INVALID_ARG, "GEMMA_F_SOURCE_WINDOW: local layers after cached tokens only");
  if (!q || !out || !k_cache || !v_cache) return fail(GEMMA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)) || !aligned16(workspace))
    return fail(GEMMA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (window > 0) {
    if (cache_cap != window)
      return fail(GEMMA_ERR_INVALID_ARG, "local layer: cache_cap %d must equal window %d", cache_cap, window);
    if (shared && seq_lens_before && !src_win)
      return fail(GEMMA_ERR_UNSUPPORTED,
                  "shared local layer after cached tokens: the source's chunk has replaced ring slots it needs "
                  "(GEMMA_F_SOURCE_WINDOW reads the window its source's call left in the workspace)");
    if (shared && s_new > window)
      return fail(GEMMA_ERR_UNSUPPORTED, "shared local layer: prefill longer than the window");
  } else if (cache_cap < s_new) {
    return fail(GEMMA_ERR_CAPACITY, "global layer: cache_cap %d < s_new %d", cache_cap, s_new);
  }
  if (s_new == 0) return succeed();
  // a local layer's chunk after cached tokens attends to a gathered key
  // window. On an int8 cache so does every chunk that reads cached rows
  // (after cached tokens, or a shared layer's): the rows are dequantized
  // into the window; a global layer's window rows are positions.
  const bool chunked_local = window > 0 && seq_lens_before && !shared;
  // a shared local layer after cached tokens attends to the window its
  // source's call left in this workspace (int8: the chunk's rows are read
  // back from the codes over it, as a shared layer reads every row)
  const bool reuse_local = window > 0 && seq_lens_before && shared && src_win;
  const bool win_local = chunked_local || reuse_local || (q8 && window > 0 && shared);
  const bool prefix_q8 = q8 && window == 0 && (seq_lens_before || shared);
  const int win_rows = win_local ? window + s_new : prefix_q8 ? cache_cap : 0;
  size_t off_k, off_vw;
  size_t need = prefill_ws_parts(batch, s_new, n_q_heads, n_kv_heads, head_dim, window, &off_k, &off_vw,
                                 prefix_q8 ? cache_cap : 0);
  if (!workspace || workspace_bytes < need)
    return fail(GEMMA_ERR_CAPACITY, "workspace %zu bytes < %zu", workspace_bytes, need);
  int* status = status_ptr();
  if (!status) return fail(GEMMA_ERR_CUDA, "no CUDA device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (lens_after) {
    cudaError_t el = launch_lens_minus(lens_after, const_cast<int32_t*>(seq_lens_before), batch, s_new, st);
    if (el != cudaSuccess) return cuda_fail(el, "length launch");
  }

  PrefillRopeArgs ra{};
  ra.q = static_cast<const bf16*>(q);
  ra.k_new = static_cast<const bf16*>(k_new);
  ra.v_new = static_cast<const bf16*>(v_new);
  ra.q_rot = reinterpret_cast<bf16*>(ws);
  ra.k_rot = ((window > 0 && !shared) || q8) ? reinterpret_cast<bf16*>(ws + off_k) : nullptr;
  ra.v_win = (win_local || prefix_q8) ? reinterpret_cast<bf16*>(ws + off_vw) : nullptr;
  ra.win_rows = win_rows;
  ra.win_at_pos = prefix_q8 ? 1 : 0;
  const size_t codes_off = q8 ? gemma_kv_codes_bytes(L.n_pages, n_kv_heads, L.page_size, head_dim) : 0;
  if (q8 && (win_local || prefix_q8)) {
    // before the chunk's rows are quantized into the cache: the cached rows
    // it attends to, dequantized, into the windows (K = V: K only). A shared
    // layer's chunk is in the cache already: its positions come along.
    const uint8_t* kc8 = static_cast<const uint8_t*>(k_cache);
    const uint8_t* vc8 = keqv ? nullptr : static_cast<const uint8_t*>(v_cache);
    cudaError_t eg = launch_gather_q8(kc8, reinterpret_cast<const float2*>(kc8 + codes_off), vc8,
                                      vc8 ? reinterpret_cast<const float2*>(vc8 + codes_off) : nullptr,
                                      seq_lens_before, shared ? s_new : 0, batch, n_kv_heads, head_dim, window,
                                      cache_cap, L.page_table, L.page_size, L.pages_per_seq, L.n_pages, win_rows,
                                      reuse_local ? window : 0, ra.k_rot, ra.v_win, status, st);
    if (eg != cudaSuccess) return cuda_fail(eg, "int8 window gather launch");
  } else if (chunked_local) {
    // before the chunk overwrites ring slots: old keys/values into rows 0..window-1
    cudaError_t eg = launch_ring_gather(static_cast<const bf16*>(k_cache), static_cast<const bf16*>(v_cache),
                                        seq_lens_before, batch, n_kv_heads, head_dim, window, win_rows,
                                        ra.k_rot, ra.v_win, status, st);
    if (eg != cudaSuccess) return cuda_fail(eg, "ring gather launch");
  }
  ra.k_cache = static_cast<bf16*>(k_cache);
  ra.v_cache = static_cast<bf16*>(v_cache);
  ra.cache_cap = cache_cap;
  ra.seq_lens_before = seq_lens_before;
  ra.S = s_new;
  ra.window = window;
  ra.Hq = n_q_heads;
  ra.Hkv = n_kv_heads;
  ra.n_rot = rope_rotated_pairs(head_dim, rope_frac);
  ra.log2_theta = std::log2((double)rope_theta);
  // queries carry scale * log2(e): the attention kernel's logits are then in
  // log2 units (one bf16 rounding either way)
  ra.q_scale = (float)((double)scale * 1.4426950408889634);
  ra.quant = q8 ? 1 : 0;
  ra.page_table = L.page_table;
  ra.page_size = L.page_size;
  ra.pages_per_seq = L.pages_per_seq;
  ra.n_pages = L.n_pages;
  ra.status = status;
  ProfScope p_rope(GEMMA_KERNEL_PREFILL_ROPE, st);
  cudaError_t e = launch_prefill_rope(ra, batch, head_dim, st);
  if (e == cudaSuccess && q8 && !shared)
    e = quantize_kv(ra.k_rot, win_rows ? win_rows : s_new, prefix_q8 ? 2 : chunked_local ? 1 : 0,
                    keqv ? nullptr : ra.v_new, k_cache, v_cache, batch, s_new, n_kv_heads, head_dim, window,
                    cache_cap, seq_lens_before, 0, L, status, st);
  p_rope.done();
  if (e != cudaSuccess) return cuda_fail(e, "prefill rope launch");

  PrefillAttnArgs aa{};
  aa.q_rot = ra.q_rot;
  const int64_t D = head_dim;
  const bool cache_view = (window == 0 || shared) && !q8 && !reuse_local;
  if (cache_view) {
    // head-major views of the cache's pages (a contiguous cache: one page of
    // cache_cap rows per sequence)
    const int64_t ps = L.page_size;
    KVView kc = {static_cast<const bf16*>(k_cache), (int64_t)n_kv_heads * ps * D, D, ps * D};
    KVView vc = {static_cast<const bf16*>(v_cache), kc.stride_b, kc.stride_row, kc.stride_h};
    aa.k = kc;
    aa.v = vc;
    aa.key_cap = cache_cap;
  } else if (win_local || prefix_q8) {
    const bf16* k_win = reinterpret_cast<const bf16*>(ws + off_k);
    KVView kw = {k_win, (int64_t)win_rows * n_kv_heads * D, (int64_t)n_kv_heads * D, D};
    KVView vw = {keqv ? k_win : ra.v_win, kw.stride_b, kw.stride_row, kw.stride_h};
    aa.k = kw;
    aa.v = vw;
    aa.key_cap = win_rows;
  } else {
    // the chunk's rotated K and the caller's V (K = V: the rotated K again)
    KVView kw = {ra.k_rot, (int64_t)s_new * n_kv_heads * D, (int64_t)n_kv_heads * D, D};
    KVView vw = {keqv ? ra.k_rot : static_cast<const bf16*>(v_new), kw.stride_b, kw.stride_row, kw.stride_h};
    aa.k = kw;
    aa.v = vw;
    aa.key_cap = s_new;
  }
  aa.key_off_window = win_local ? 1 : 0;
  aa.seq_lens_before = seq_lens_before;
  aa.S = s_new;
  aa.window = window;
  aa.Hq = n_q_heads;
  aa.Hkv = n_kv_heads;
  aa.scale_log2 = 1.0f;  // already applied to the rotated queries
  aa.out = static_cast<bf16*>(out);
  aa.lse = lse;
  aa.status = status;
  aa.wait_ns = (unsigned long long)g_wait_ns.load();
  aa.page_table = cache_view ? L.page_table : nullptr;
  aa.page_size = L.page_size;
  aa.pages_per_seq = L.pages_per_seq;
  aa.n_pages = cache_view ? L.n_pages : batch;
  ProfScope p_attn(GEMMA_KERNEL_PREFILL_ATTN, st);
  // Head_dim-512 layers run on CTA pairs (cta_group::2, M = 256): each SM
  // loads and reads from shared memory half of every K and V tile. With an
  // even number of q heads per KV head the pair takes two q heads of one
  // query tile (measured on B200: -7% on an 8K-token E2B global layer, -13%
  // on a 32K-token 31B global layer); otherwise two query tiles of one head,
  // which only pays from 16K keys. Head_dim 256 stays on one CTA per tile
  // (both pairings measured slower on local layers).
  // GEMMA_PREFILL_KERNEL=single|pair|hpair overrides the choice.
  enum { K_SINGLE, K_PAIR, K_HPAIR } kern = K_SINGLE;
  if (head_dim == 512) {
    if ((n_q_heads / n_kv_heads) % 2 == 0)
      kern = K_HPAIR;
    else if ((cache_view || prefix_q8 ? cache_cap : s_new) >= 16384)
      kern = K_PAIR;
  }
  if (const char* v = std::getenv("GEMMA_PREFILL_KERNEL")) {
    if (std::string(v) == "single") kern = K_SINGLE;
    if (std::string(v) == "pair") kern = K_PAIR;
    if (std::string(v) == "hpair") kern = K_HPAIR;
  }
  const int key_rows = cache_view ? L.page_size : (int)aa.key_cap;
  const int tok_major = cache_view ? 0 : 1;
  e = kern == K_SINGLE ? launch_prefill_attn_tc(aa, batch, head_dim, key_rows, tok_major, st)
                       : launch_prefill_attn_pair(aa, batch, head_dim, key_rows, tok_major, kern == K_HPAIR, st);
  p_attn.done();
  if (e != cudaSuccess) return cuda_fail(e, "prefill attention launch");
  return succeed();
}

int gemma_attn_prefill(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                       int cache_cap, const int32_t* seq_lens_before, int batch, int s_new, int window,
                       int n_q_heads, int n_kv_heads, int head_dim, float rope_frac, float rope_theta,
                       float scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                       unsigned flags, void* stream) {
  return prefill_impl(q, k_new, v_new, k_cache, v_cache, cache_cap, seq_lens_before, batch, s_new, window,
                      n_q_heads, n_kv_heads, head_dim, rope_frac, rope_theta, scale, out, lse, workspace,
                      workspace_bytes, flags, stream, contiguous(cache_cap, batch));
}

int gemma_attn_prefill_paged(const void* q, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                             const int32_t* page_table, int page_size, int pages_per_seq, int n_pages,
                             const int32_t* seq_lens_before, int batch, int s_new, int n_q_heads,
                             int n_kv_heads, int head_dim, float rope_frac, float rope_theta, float scale,
                             void* out, float* lse, void* workspace, size_t workspace_bytes, unsigned flags,
                             void* stream) {
  int rc = check_paged(page_table, page_size, pages_per_seq, n_pages);
  if (rc) return rc;
  return prefill_impl(q, k_new, v_new, k_pool, v_pool, pages_per_seq * page_size, seq_lens_before, batch, s_new,
                      0, n_q_heads, n_kv_heads, head_dim, rope_frac, rope_theta, scale, out, lse, workspace,
                      workspace_bytes, flags, stream, CacheLayout{page_table, page_size, pages_per_seq, n_pages});
}

size_t gemma_attn_decode_workspace_size(int batch, int n_q_heads, int n_kv_heads, int head_dim, int window,
                                        int max_seq_len) {
  if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || max_seq_len <= 0) return 0;
  int chunk, n_splits;
  decode_plan(batch, n_kv_heads, window, max_seq_len, &chunk, &n_splits);
  size_t a, b;
  return decode_ws_parts(batch, n_q_heads, n_kv_heads, head_dim, n_splits, &a, &b);
}

static int decode_impl(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                       int cache_cap, const int32_t* seq_lens, int max_seq_len, int batch, int window,
                       int n_q_heads, int n_kv_heads, int head_dim, float rope_frac, float rope_theta,
                       float scale, void* out, void* workspace, size_t workspace_bytes, unsigned flags,
                       void* stream, const CacheLayout& L) {
  int rc = check_heads(n_q_heads, n_kv_heads, head_dim, window, rope_frac, rope_theta, scale);
  if (rc) return rc;
  rc = check_kv_flags(flags, window, k_new, v_new, k_cache, &v_cache);
  if (rc) return rc;
  if (flags & GEMMA_F_SOURCE_WINDOW)
    return fail(GEMMA_ERR_INVALID_ARG, "GEMMA_F_SOURCE_WINDOW: a prefill / multi-token flag (one new token "
                                       "never needs a slot its source replaced)");
  if (batch <= 0 || max_seq_len <= 0)
    return fail(GEMMA_ERR_INVALID_ARG, "batch %d, max_seq_len %d", batch, max_seq_len);
  if (!q || !out || !k_cache || !v_cache || !seq_lens)
    return fail(GEMMA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)) || !aligned16(workspace))
    return fail(GEMMA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (window > 0 && cache_cap != window)
    return fail(GEMMA_ERR_INVALID_ARG, "local layer: cache_cap %d must equal window %d", cache_cap, window);
  if (window == 0 && cache_cap < max_seq_len)
    return fail(GEMMA_ERR_CAPACITY, "global layer: cache_cap %d < max_seq_len %d", cache_cap, max_seq_len);
  const bool q8 = flags & GEMMA_F_KV_INT8;
  if (q8 && cache_cap % 2) return fail(GEMMA_ERR_INVALID_ARG, "int8 KV: cache_cap %d must be even", cache_cap);
  int chunk, n_splits;
  decode_plan(batch, n_kv_heads, window, max_seq_len, &chunk, &n_splits);
  size_t off_lse, off_o, off_kst;
  size_t need = decode_ws_parts(batch, n_q_heads, n_kv_heads, head_dim, n_splits, &off_lse, &off_o, &off_kst);
  if (!workspace || workspace_bytes < need)
    return fail(GEMMA_ERR_CAPACITY, "workspace %zu bytes < %zu", workspace_bytes, need);
  int* status = status_ptr();
  if (!status) return fail(GEMMA_ERR_CUDA, "no CUDA device");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);

  DecodeRopeArgs ra{};
  ra.tokens = 1;
  ra.q_scale = 1.f;
  ra.q = static_cast<const bf16*>(q);
  ra.k_new = static_cast<const bf16*>(k_new);
  ra.v_new = static_cast<const bf16*>(v_new);
  ra.q_rot = reinterpret_cast<bf16*>(ws);
  ra.k_cache = static_cast<bf16*>(k_cache);
  ra.v_cache = static_cast<bf16*>(v_cache);
  ra.cache_cap = cache_cap;
  ra.seq_lens = seq_lens;
  ra.max_len = max_seq_len;
  ra.window = window;
  ra.Hq = n_q_heads;
  ra.Hkv = n_kv_heads;
  ra.n_rot = rope_rotated_pairs(head_dim, rope_frac);
  ra.log2_theta = std::log2((double)rope_theta);
  ra.k_stage = q8 ? reinterpret_cast<bf16*>(ws + off_kst) : nullptr;
  ra.page_table = L.page_table;
  ra.page_size = L.page_size;
  ra.pages_per_seq = L.pages_per_seq;
  ra.n_pages = L.n_pages;
  ra.status = status;
  // rotates q; also appends the new K/V unless the layer is shared (int8:
  // the rotated key is staged, then both rows are quantized into the cache)
  ProfScope p_app(GEMMA_KERNEL_DECODE_APPEND, st);
  cudaError_t e = launch_decode_rope_append(ra, batch, head_dim, st);
  if (e == cudaSuccess && q8 && k_new)
    e = quantize_kv(ra.k_stage, 1, 0, (flags & GEMMA_F_KEQV) ? nullptr : ra.v_new, k_cache, v_cache, batch, 1,
                    n_kv_heads, head_dim, window, cache_cap, seq_lens, 1, L, status, st);
  p_app.done();
  if (e != cudaSuccess) return cuda_fail(e, "decode append launch");

  DecodeAttnArgs da{};
  da.tokens = 1;
  da.q_rot = ra.q_rot;
  da.k_cache = static_cast<const bf16*>(k_cache);
  da.v_cache = static_cast<const bf16*>(v_cache);
  da.cache_cap = cache_cap;
  da.seq_lens = seq_lens;
  da.max_len = max_seq_len;
  da.window = window;
  da.Hq = n_q_heads;
  da.Hkv = n_kv_heads;
  da.chunk = chunk;
  da.n_splits = n_splits;
  da.scale_log2 = (float)((double)scale * 1.4426950408889634);
  da.part_lse = reinterpret_cast<float*>(ws + off_lse);
  da.part_o = reinterpret_cast<float*>(ws + off_o);
  da.out = static_cast<bf16*>(out);
  da.status = status;
  da.wait_ns = (unsigned long long)g_wait_ns.load();
  da.drop_first_copy = g_drop_next.exchange(0);
  da.keqv = (flags & GEMMA_F_KEQV) ? 1 : 0;
  da.page_table = L.page_table;
  da.page_size = L.page_size;
  da.pages_per_seq = L.pages_per_seq;
  da.n_pages = L.n_pages;
  if (q8) {
    const size_t off = gemma_kv_codes_bytes(L.n_pages, n_kv_heads, L.page_size, head_dim);
    da.k_codes = static_cast<const uint8_t*>(k_cache);
    da.v_codes = static_cast<const uint8_t*>(v_cache);
    da.k_params = reinterpret_cast<const float2*>(static_cast<const uint8_t*>(k_cache) + off);
    da.v_params = reinterpret_cast<const float2*>(static_cast<const uint8_t*>(v_cache) + off);
  }
  {
    ProfScope p_split(GEMMA_KERNEL_DECODE_SPLIT, st);
    e = q8 ? launch_decode_split_q8(da, batch, head_dim, st) : launch_decode_split(da, batch, head_dim, st);
    p_split.done();
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode attention launch");
  {
    ProfScope p_comb(GEMMA_KERNEL_DECODE_COMBINE, st);
    e = launch_decode_combine(da, batch, head_dim, st);
    p_comb.done();
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  return succeed();
}

int gemma_attn_decode(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                      int cache_cap, const int32_t* seq_lens, int max_seq_len, int batch, int window,
                      int n_q_heads, int n_kv_heads, int head_dim, float rope_frac, float rope_theta,
                      float scale, void* out, void* workspace, size_t workspace_bytes, unsigned flags,
                      void* stream) {
  return decode_impl(q, k_new, v_new, k_cache, v_cache, cache_cap, seq_lens, max_seq_len, batch, window, n_q_heads,
                     n_kv_heads, head_dim, rope_frac, rope_theta, scale, out, workspace, workspace_bytes, flags,
                     stream, contiguous(cache_cap, batch));
}

int gemma_attn_decode_paged(const void* q, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                            const int32_t* page_table, int page_size, int pages_per_seq, int n_pages,
                            const int32_t* seq_lens, int max_seq_len, int batch, int n_q_heads, int n_kv_heads,
                            int head_dim, float rope_frac, float rope_theta, float scale, void* out,
                            void* workspace, size_t workspace_bytes, unsigned flags, void* stream) {
  int rc = check_paged(page_table, page_size, pages_per_seq, n_pages);
  if (rc) return rc;
  return decode_impl(q, k_new, v_new, k_pool, v_pool, pages_per_seq * page_size, seq_lens, max_seq_len, batch, 0,
                     n_q_heads, n_kv_heads, head_dim, rope_frac, rope_theta, scale, out, workspace, workspace_bytes,
                     flags, stream, CacheLayout{page_table, page_size, pages_per_seq, n_pages});
}

size_t gemma_attn_decode_multi_workspace_size(int batch, int tokens, int n_q_heads, int n_kv_heads, int head_dim,
                                              int window, int max_seq_len, int cache_cap, unsigned flags) {
  if (batch <= 0 || tokens <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || max_seq_len <= 0 ||
      cache_cap <= 0)
    return 0;
  if (verify_by_decode(window, flags)) {
    size_t a, b, c, d, e;
    return verify_decode_ws(batch, n_q_heads, n_kv_heads, head_dim, max_seq_len, &a, &b, &c, &d, &e);
  }
  if (verify_fast(tokens, window, n_q_heads, n_kv_heads, head_dim, flags)) {
    int chunk, n_splits;
    verify_plan(batch, n_q_heads, n_kv_heads, tokens, head_dim, window, max_seq_len, &chunk, &n_splits);
    size_t a, b, c;
    return verify_ws_parts(batch, tokens, n_q_heads, n_kv_heads, head_dim, window, n_splits, &a, &b, &c);
  }
  return verify_route_ws(batch, tokens, n_q_heads, n_kv_heads, head_dim, window, cache_cap, flags);
}

static int multi_impl(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                      int cache_cap, const int32_t* seq_lens, int max_seq_len, int batch, int tokens, int window,
                      int n_q_heads, int n_kv_heads, int head_dim, float rope_frac, float rope_theta, float scale,
                      void* out, void* workspace, size_t workspace_bytes, unsigned flags, void* stream,
                      const CacheLayout& L) {
  int rc = check_heads(n_q_heads, n_kv_heads, head_dim, window, rope_frac, rope_theta, scale);
  if (rc) return rc;
  if (batch <= 0 || tokens <= 0 || max_seq_len <= 0 || tokens > max_seq_len)
    return fail(GEMMA_ERR_INVALID_ARG, "batch %d, tokens %d, max_seq_len %d (tokens <= max_seq_len)", batch, tokens,
                max_seq_len);
  if (!seq_lens) return fail(GEMMA_ERR_INVALID_ARG, "null seq_lens");
  if (window == 0 && cache_cap < max_seq_len)
    return fail(GEMMA_ERR_CAPACITY, "global layer: cache_cap %d < max_seq_len %d", cache_cap, max_seq_len);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (verify_by_decode(window, flags)) {
    rc = check_kv_flags(flags, window, k_new, v_new, k_cache, &v_cache);
    if (rc) return rc;
    if (flags & GEMMA_F_SOURCE_WINDOW)
      return fail(GEMMA_ERR_INVALID_ARG, "GEMMA_F_SOURCE_WINDOW: local layers after cached tokens only");
    if (!q || !out || !k_cache || !v_cache) return fail(GEMMA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)) || !aligned16(workspace))
      return fail(GEMMA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (cache_cap % 2) return fail(GEMMA_ERR_INVALID_ARG, "int8 KV: cache_cap %d must be even", cache_cap);
    size_t off_dec, off_q, off_k, off_v, off_o;
    const size_t need =
        verify_decode_ws(batch, n_q_heads, n_kv_heads, head_dim, max_seq_len, &off_dec, &off_q, &off_k, &off_v, &off_o);
    if (!workspace || workspace_bytes < need)
      return fail(GEMMA_ERR_CAPACITY, "workspace %zu bytes < %zu", workspace_bytes, need);
    // token t of every sequence: its rows out of [B][tokens][..] into the
    // workspace, a decode at length seq_lens - (tokens - 1 - t), its output back
    int32_t* lens_t = reinterpret_cast<int32_t*>(ws);
    const size_t qrow = (size_t)n_q_heads * head_dim * 2, kvrow = (size_t)n_kv_heads * head_dim * 2;
    const size_t dec_bytes = off_q - off_dec;
    for (int t = 0; t < tokens; ++t) {
      cudaError_t e = launch_lens_minus(seq_lens, lens_t, batch, tokens - 1 - t, st);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(ws + off_q, qrow, static_cast<const unsigned char*>(q) + t * qrow, tokens * qrow, qrow,
                              batch, cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess && k_new)
        e = cudaMemcpy2DAsync(ws + off_k, kvrow, static_cast<const unsigned char*>(k_new) + t * kvrow,
                              tokens * kvrow, kvrow, batch, cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess && v_new)
        e = cudaMemcpy2DAsync(ws + off_v, kvrow, static_cast<const unsigned char*>(v_new) + t * kvrow,
                              tokens * kvrow, kvrow, batch, cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return cuda_fail(e, "multi-token decode staging");
      rc = decode_impl(ws + off_q, k_new ? ws + off_k : nullptr, v_new ? ws + off_v : nullptr, k_cache,
                       (flags & GEMMA_F_KEQV) ? nullptr : v_cache, cache_cap, lens_t, max_seq_len, batch, 0,
                       n_q_heads, n_kv_heads, head_dim, rope_frac, rope_theta, scale, ws + off_o, ws + off_dec,
                       dec_bytes, flags, stream, L);
      if (rc) return rc;
      e = cudaMemcpy2DAsync(static_cast<unsigned char*>(out) + t * qrow, tokens * qrow, ws + off_o, qrow, qrow,
                            batch, cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return cuda_fail(e, "multi-token decode output copy");
    }
    return succeed();
  }
  if (!verify_fast(tokens, window, n_q_heads, n_kv_heads, head_dim, flags)) {
    // the new tokens as a chunk after seq_lens - tokens cached tokens
    const size_t need = verify_route_ws(batch, tokens, n_q_heads, n_kv_heads, head_dim, window, cache_cap, flags);
    if (!workspace || workspace_bytes < need)
      return fail(GEMMA_ERR_CAPACITY, "workspace %zu bytes < %zu", workspace_bytes, need);
    if (!aligned16(workspace)) return fail(GEMMA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    int32_t* before = reinterpret_cast<int32_t*>(ws);
    const size_t head = align256((size_t)batch * 4);
    return prefill_impl(q, k_new, v_new, k_cache, v_cache, cache_cap, before, batch, tokens, window, n_q_heads,
                        n_kv_heads, head_dim, rope_frac, rope_theta, scale, out, nullptr, ws + head,
                        workspace_bytes - head, flags, stream, L, seq_lens);
  }
  rc = check_kv_flags(flags, window, k_new, v_new, k_cache, &v_cache);
  if (rc) return rc;
  if (!q || !out || !k_cache || !v_cache) return fail(GEMMA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)) || !aligned16(workspace))
    return fail(GEMMA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (window > 0 && cache_cap != window)
    return fail(GEMMA_ERR_INVALID_ARG, "local layer: cache_cap %d must equal window %d", cache_cap, window);
  int chunk, n_splits;
  verify_plan(batch, n_q_heads, n_kv_heads, tokens, head_dim, window, max_seq_len, &chunk, &n_splits);
  size_t off_lse, off_o, off_kst;
  const size_t need =
      verify_ws_parts(batch, tokens, n_q_heads, n_kv_heads, head_dim, window, n_splits, &off_lse, &off_o, &off_kst);
  if (!workspace || workspace_bytes < need)
    return fail(GEMMA_ERR_CAPACITY, "workspace %zu bytes < %zu", workspace_bytes, need);
  int* status = status_ptr();
  if (!status) return fail(GEMMA_ERR_CUDA, "no CUDA device");

  DecodeRopeArgs ra{};
  ra.tokens = tokens;
  // queries carry scale * log2(e), as in prefill: logits arrive in log2 units
  ra.q_scale = (float)((double)scale * 1.4426950408889634);
  ra.q = static_cast<const bf16*>(q);
  ra.k_new = static_cast<const bf16*>(k_new);
  ra.v_new = static_cast<const bf16*>(v_new);
  ra.q_rot = reinterpret_cast<bf16*>(ws);
  ra.k_cache = static_cast<bf16*>(k_cache);
  ra.v_cache = static_cast<bf16*>(v_cache);
  ra.cache_cap = cache_cap;
  ra.seq_lens = seq_lens;
  ra.max_len = max_seq_len;
  ra.window = window;
  ra.Hq = n_q_heads;
  ra.Hkv = n_kv_heads;
  ra.n_rot = rope_rotated_pairs(head_dim, rope_frac);
  ra.log2_theta = std::log2((double)rope_theta);
  // a local layer's new rows would overwrite ring slots that the earlier new
  // tokens still see: its rotated keys wait in the workspace, and the ring
  // is written once the attention is done
  ra.k_stage = window > 0 ? reinterpret_cast<bf16*>(ws + off_kst) : nullptr;
  ra.page_table = L.page_table;
  ra.page_size = L.page_size;
  ra.pages_per_seq = L.pages_per_seq;
  ra.n_pages = L.n_pages;
  ra.status = status;
  ProfScope p_app(GEMMA_KERNEL_DECODE_APPEND, st);
  cudaError_t e = launch_decode_rope_append(ra, batch, head_dim, st);
  p_app.done();
  if (e != cudaSuccess) return cuda_fail(e, "decode append launch");

  const int64_t D = head_dim;
  VerifyAttnArgs va{};
  va.q_rot = ra.q_rot;
  const int64_t ps = L.page_size;  // rows of a view: a page, or a sequence's cache
  va.k = KVView{static_cast<const bf16*>(k_cache), (int64_t)n_kv_heads * ps * D, D, ps * D};
  va.v = KVView{static_cast<const bf16*>(v_cache), va.k.stride_b, va.k.stride_row, va.k.stride_h};
  va.cache_cap = cache_cap;
  va.page_table = L.page_table;
  va.page_size = L.page_size;
  va.pages_per_seq = L.pages_per_seq;
  va.n_pages = L.n_pages;
  va.window = window;
  va.k_tail = ra.k_stage;
  va.v_tail = ra.v_new;
  va.seq_lens = seq_lens;
  va.tokens = tokens;
  va.Hq = n_q_heads;
  va.Hkv = n_kv_heads;
  va.chunk = chunk;
  va.n_splits = n_splits;
  va.part_o = reinterpret_cast<float*>(ws + off_o);
  va.part_lse = reinterpret_cast<float*>(ws + off_lse);
  // a single split (a local ring that B x Hkv CTAs cover) writes the output itself
  const bool direct = n_splits == 1 && verify_tc_rows(n_q_heads, n_kv_heads, tokens, head_dim) != 0;
  va.out = direct ? static_cast<bf16*>(out) : nullptr;
  va.status = status;
  va.wait_ns = (unsigned long long)g_wait_ns.load();
  va.drop_first_copy = verify_tc_rows(n_q_heads, n_kv_heads, tokens, head_dim) ? g_drop_next.exchange(0) : 0;
  {
    ProfScope p_split(GEMMA_KERNEL_DECODE_SPLIT, st);
    e = launch_verify_attn_tc(va, batch, head_dim, st);
    p_split.done();
  }
  if (e != cudaSuccess) return cuda_fail(e, "multi-token attention launch");
  if (window > 0) {
    DecodeRopeArgs rb = ra;
    rb.skip_q = 1;
    rb.k_stage = nullptr;
    ProfScope p_app2(GEMMA_KERNEL_DECODE_APPEND, st);
    e = launch_decode_rope_append(rb, batch, head_dim, st);
    p_app2.done();
    if (e != cudaSuccess) return cuda_fail(e, "decode append launch");
  }
  if (direct) return succeed();

  DecodeAttnArgs da{};
  da.tokens = tokens;
  da.every_split = window > 0 ? 1 : 0;
  da.seq_lens = seq_lens;
  da.max_len = max_seq_len;
  da.window = window;
  da.Hq = n_q_heads;
  da.Hkv = n_kv_heads;
  da.chunk = chunk;
  da.n_splits = n_splits;
  da.part_lse = va.part_lse;
  da.part_o = va.part_o;
  da.out = static_cast<bf16*>(out);
  da.status = status;
  {
    ProfScope p_comb(GEMMA_KERNEL_DECODE_COMBINE, st);
    e = launch_decode_combine(da, batch, head_dim, st);
    p_comb.done();
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode combine launch");
  return succeed();
}

int gemma_attn_decode_multi(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                            int cache_cap, const int32_t* seq_lens, int max_seq_len, int batch, int tokens,
                            int window, int n_q_heads, int n_kv_heads, int head_dim, float rope_frac,
                            float rope_theta, float scale, void* out, void* workspace, size_t workspace_bytes,
                            unsigned flags, void* stream) {
  return multi_impl(q, k_new, v_new, k_cache, v_cache, cache_cap, seq_lens, max_seq_len, batch, tokens, window,
                    n_q_heads, n_kv_heads, head_dim, rope_frac, rope_theta, scale, out, workspace, workspace_bytes,
                    flags, stream, contiguous(cache_cap, batch));
}

int gemma_attn_decode_multi_paged(const void* q, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                                  const int32_t* page_table, int page_size, int pages_per_seq, int n_pages,
                                  const int32_t* seq_lens, int max_seq_len, int batch, int tokens, int n_q_heads,
                                  int n_kv_heads, int head_dim, float rope_frac, float rope_theta, float scale,
                                  void* out, void* workspace, size_t workspace_bytes, unsigned flags,
                                  void* stream) {
  int rc = check_paged(page_table, page_size, pages_per_seq, n_pages);
  if (rc) return rc;
  return multi_impl(q, k_new, v_new, k_pool, v_pool, pages_per_seq * page_size, seq_lens, max_seq_len, batch, tokens,
                    0, n_q_heads, n_kv_heads, head_dim, rope_frac, rope_theta, scale, out, workspace,
                    workspace_bytes, flags, stream, CacheLayout{page_table, page_size, pages_per_seq, n_pages});
}

int gemma_attn_visible_ranges(const int32_t* seq_lens_before, int batch, int s_new, int window,
                              int32_t* ranges, void* stream) {
  if (batch <= 0 || s_new < 0 || window < 0 || !ranges)
    return fail(GEMMA_ERR_INVALID_ARG, "bad arguments");
  cudaError_t e = launch_visible_ranges(seq_lens_before, batch, s_new, window, ranges,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "visible ranges launch");
  return succeed();
}

int gemma_attn_debug_timeout_info(long long* info8) {
  if (!info8) return fail(GEMMA_ERR_INVALID_ARG, "null output");
  DevStatus d;
  cudaError_t e = cudaMemcpyFromSymbol(&d, g_dev, sizeof d);
  if (e != cudaSuccess) return cuda_fail(e, "read timeout info");
  for (int i = 0; i < 8; ++i) info8[i] = (long long)d.info[i];
  d.timeout_claim = 0;
  for (int i = 0; i < 8; ++i) d.info[i] = 0;
  e = cudaMemcpyToSymbol(g_dev, &d.timeout_claim, sizeof(DevStatus) - offsetof(DevStatus, timeout_claim),
                         offsetof(DevStatus, timeout_claim));
  if (e != cudaSuccess) return cuda_fail(e, "clear timeout info");
  return succeed();
}

int gemma_attn_profile(int enable) {
  prof_clear();
  g_prof_on.store(enable != 0);
  return succeed();
}

int gemma_attn_profile_read(int kernel, double* total_ms, long long* launches) {
  if (kernel < 0 || kernel >= GEMMA_KERNEL_KINDS || !total_ms || !launches)
    return fail(GEMMA_ERR_INVALID_ARG, "bad profile query");
  std::lock_guard<std::mutex> lk(g_prof_mu);
  double tot = 0.0;
  long long n = 0;
  for (auto& r : g_prof) {
    if (r.kind != kernel) continue;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e, "profile event synchronize");
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "profile elapsed time");
    tot += ms;
    ++n;
  }
  *total_ms = tot;
  *launches = n;
  return succeed();
}

int gemma_attn_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_dev, sizeof v);
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_dev, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "clear device status");
    return fail(v, v == GEMMA_ERR_DEVICE_TIMEOUT ? "a bounded device wait gave up"
                                                 : "a device-side range check failed");
  }
  return succeed();
}

}  // extern "C"
