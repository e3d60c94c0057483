/*
 * gemma_attn.h -- C ABI of libgemma_attn.so: interleaved local (sliding
 * window) / global causal grouped-query attention with (proportional) RoPE,
 * a ring-buffer / append KV cache and last-N-layer KV sharing, for NVIDIA
 * B200 (sm_100a).
 *
 * Passages defining the operations (page title, section):
 *   - "Gemma 4: End-to-End Architecture Walkthrough", 3a "Interleaved
 *     Local/Global Attention": local layers attend to a fixed recent window,
 *     global layers to the whole preceding context; r local layers per
 *     global layer; the final layer is always global.
 *   - same page, 3b "Making the Expensive Global Layers Cheaper": GQA 8:1 on
 *     global layers (2:1 on local ones), doubled key dimension; global
 *     layers cache K/V for the whole context.
 *   - same page, 3c "p-RoPE", and "Gemma 4 Architecture Reference",
 *     "Positional Encoding: Proportional RoPE (p-RoPE)": on global layers
 *     only the first p = 0.25 of the dimension pairs rotate, theta = 1e6.
 *   - "Gemma 4 Architecture Reference", "Attention Architecture" (window
 *     512 / 1024, GQA ratios) and "Shared KV Cache" (the last N layers reuse
 *     K/V of an earlier layer of the same attention type).
 *
 * Conventions for every call:
 *   - Tensors are bf16 (IEEE bfloat16 bit patterns), contiguous, row-major in
 *     the stated shape, in device memory, 16-byte aligned. fp32 outputs and
 *     int32 length arrays are device memory too.
 *   - The caller owns all memory. The library never allocates device memory;
 *     calls that need scratch take a caller-sized workspace.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous on it; argument errors are reported before anything is
 *     enqueued and nothing is enqueued on error.
 *   - Positions are 0-based and absolute. Key j is visible to the query at
 *     position p iff j <= p and (window == 0 or j > p - window).
 *   - RoPE pairs dimensions (2i, 2i+1) and turns pair i by the angle
 *     p * rope_theta^(-2i/head_dim) when i < floor(rope_frac * head_dim / 2);
 *     other pairs are left as they are. V is never rotated.
 *   - Cache layout: [batch][n_kv_heads][cache_cap][head_dim]. A global layer
 *     (window == 0) keeps position p in slot p (cache_cap >= context length).
 *     A local layer keeps a ring of cache_cap == window slots, position p in
 *     slot p % window.
 *   - Return value: a gemma_status. On failure gemma_last_error() gives a
 *     message (thread-local, valid until the next call on that thread).
 */
#ifndef GEMMA_ATTN_H
#define GEMMA_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GEMMA_ATTN_ABI_VERSION 1

typedef enum gemma_status {
    GEMMA_OK = 0,
    GEMMA_ERR_INVALID_ARG = 1,    /* bad pointer, size, ratio or flag */
    GEMMA_ERR_UNSUPPORTED = 2,    /* valid request this build does not implement */
    GEMMA_ERR_SHARE_MISMATCH = 3, /* gemma_kv_share_bind: layers not compatible */
    GEMMA_ERR_CAPACITY = 4,       /* cache or workspace too small */
    GEMMA_ERR_CUDA = 5,           /* a CUDA runtime call failed */
    GEMMA_ERR_DEVICE_TIMEOUT = 6, /* a bounded device wait gave up (see sync_status) */
    GEMMA_ERR_DEVICE_RANGE = 7    /* a device-side length/capacity check failed */
} gemma_status;

/* flags */
#define GEMMA_F_SHARED 1u /* k_cache/v_cache alias an earlier layer (see
                             gemma_kv_share_bind): k_new and v_new must be NULL;
                             nothing is rotated or written into the cache. */
#define GEMMA_F_KEQV 2u   /* K = V ("Gemma 4: End-to-End Architecture
                             Walkthrough", 3b "K = V"; "Gemma 4 Technical Report"
                             summary, Core Model Architecture: only K is cached
                             and the attention weights multiply K). Global
                             layers only (window 0, else GEMMA_ERR_UNSUPPORTED).
                             v_new must be NULL; v_cache must be NULL or equal
                             k_cache. The values are the keys as the cache holds
                             them (rotated); nothing is written for V. */
#define GEMMA_F_KV_INT8 4u /* int8 KV cache ("Gemma 4 Technical Report",
                             Quantization and Efficiency, and its Table 3
                             "+KV int8"). Each cache buffer holds
                               codes  uint8 [batch][n_kv_heads][cache_cap][head_dim]
                             followed, at byte offset
                             gemma_kv_codes_bytes(batch, n_kv_heads, cache_cap,
                             head_dim), by
                               params float2 [batch][n_kv_heads][cache_cap] = (min, step)
                             per cached row; the row's value is
                             min + code * step. A row is quantized after
                             (p-)RoPE and the bf16 rounding: min/max over its
                             head_dim channels, code = round((x - min) * 255 /
                             (max - min)) to nearest even, in fp32; a constant
                             row gets codes 0 and step 0. Size the buffers with
                             gemma_kv_cache_bytes(..., GEMMA_F_KV_INT8);
                             cache_cap must be even. Prefill attends with the
                             chunk's own bf16 K/V and writes codes; the cached
                             rows a chunk also attends to (after cached
                             tokens, or every row on a GEMMA_F_SHARED layer)
                             are read back as min + code * step rounded to
                             bf16 (a global layer then needs the larger
                             workspace of
                             gemma_attn_prefill_workspace_size_cached).
                             Decode reads codes. Combines with GEMMA_F_KEQV
                             and GEMMA_F_SHARED. */

#define GEMMA_F_SOURCE_WINDOW 8u /* KV-shared local layers after cached tokens
                             ("Gemma 4 Architecture Reference", Shared KV Cache:
                             the last layers reuse an earlier local layer's
                             K/V). A chunk after cached tokens on an unshared
                             local layer leaves in its workspace the keys and
                             values it attended to: the ring's last `window`
                             positions before the chunk, then the chunk. With
                             GEMMA_F_SHARED | GEMMA_F_SOURCE_WINDOW a shared
                             local layer's call attends to them; its workspace
                             must be the one of its source layer's call for the
                             same chunk (same batch, s_new, head counts,
                             head_dim, window and seq_lens_before), not written
                             since except by other such shared calls. Without
                             the flag that call is GEMMA_ERR_UNSUPPORTED: the
                             source's chunk has replaced ring slots that the
                             chunk's earlier queries still see. On an int8
                             cache the chunk's own rows are read back from the
                             codes, as a shared layer reads every row. In
                             gemma_attn_decode_multi the flag on an unshared
                             local layer selects the chunked-prefill path, so
                             that the call leaves that window. Only for local
                             layers after cached tokens (else
                             GEMMA_ERR_INVALID_ARG). */

/* Bytes of one layer's K (or V) cache buffer: batch * n_kv_heads *
 * cache_cap * head_dim * 2 for bf16; with GEMMA_F_KV_INT8 the codes, padded
 * to 256 bytes, plus 8 bytes of (min, step) per row. 0 on bad arguments. */
size_t gemma_kv_cache_bytes(int batch, int n_kv_heads, int cache_cap, int head_dim, unsigned flags);
/* Offset of the (min, step) array in an int8 cache buffer. */
size_t gemma_kv_codes_bytes(int batch, int n_kv_heads, int cache_cap, int head_dim);

/* Supported shapes: head_dim 256 or 512; n_q_heads a multiple of n_kv_heads
 * with n_q_heads / n_kv_heads <= 8; window 0 (global) or a multiple of 16. */

/* ---------------------------------------------------------------------- */
/* Prefill: a chunk of s_new tokens per sequence.                          */
/*                                                                        */
/* q      [batch][s_new][n_q_heads][head_dim]   pre-RoPE queries           */
/* k_new  [batch][s_new][n_kv_heads][head_dim]  pre-RoPE keys (NULL if     */
/* v_new  [batch][s_new][n_kv_heads][head_dim]  values        GEMMA_F_SHARED)*/
/* k_cache, v_cache [batch][n_kv_heads][cache_cap][head_dim]               */
/* seq_lens_before  device int32 [batch]: tokens already in the cache per   */
/*        sequence (the chunk starts at that position), or NULL for 0.     */
/*        On a local layer the chunk also attends to the ring's last       */
/*        `window` cached positions (read before the chunk overwrites      */
/*        them); a shared local layer after cached tokens needs            */
/*        GEMMA_F_SOURCE_WINDOW (else GEMMA_ERR_UNSUPPORTED: its source     */
/*        already replaced those slots).                                   */
/* out    [batch][s_new][n_q_heads][head_dim]  bf16 attention output        */
/* lse    optional fp32 [batch][n_q_heads][s_new]: natural-log sum of       */
/*        exp(scale * q.k) over the visible keys; NULL to skip.            */
/* workspace: at least gemma_attn_prefill_workspace_size(...) bytes,       */
/*        256-byte aligned; contents are scratch.                          */
/*                                                                        */
/* Effect: rotated K and V of the chunk are written into the cache (global:*/
/* slots seq_lens_before[b] .. +s_new-1; local: the ring slots of the last */
/* `window` positions), then every query attends causally (window-limited */
/* on local layers) to the cached context plus the chunk. On a global     */
/* layer seq_lens_before[b] + s_new must not exceed cache_cap; a device-   */
/* side check skips the sequence and reports GEMMA_ERR_DEVICE_RANGE       */
/* through gemma_attn_sync_status otherwise.                              */
/* ---------------------------------------------------------------------- */
size_t gemma_attn_prefill_workspace_size(int batch, int s_new, int n_q_heads,
                                         int n_kv_heads, int head_dim, int window);
/* Workspace of a prefill that reads cached rows (seq_lens_before != NULL, */
/* or a GEMMA_F_SHARED layer) on a cache of capacity cache_cap: equal to   */
/* the above, except that an int8 global layer (GEMMA_F_KV_INT8 in flags,  */
/* window 0) also holds its keys and values up to cache_cap rows in bf16   */
/* (2 * batch * cache_cap * n_kv_heads * head_dim * 2 bytes more). 0 on    */
/* bad arguments.                                                          */
size_t gemma_attn_prefill_workspace_size_cached(int batch, int s_new, int n_q_heads,
                                                int n_kv_heads, int head_dim, int window,
                                                int cache_cap, unsigned flags);

int gemma_attn_prefill(const void* q, const void* k_new, const void* v_new,
                       void* k_cache, void* v_cache, int cache_cap,
                       const int32_t* seq_lens_before, int batch, int s_new,
                       int window, int n_q_heads, int n_kv_heads, int head_dim,
                       float rope_frac, float rope_theta, float scale,
                       void* out, float* lse, void* workspace,
                       size_t workspace_bytes, unsigned flags, void* stream);

/* ---------------------------------------------------------------------- */
/* Decode: one new token per sequence, batched.                            */
/*                                                                        */
/* q      [batch][n_q_heads][head_dim]   pre-RoPE query of the new token   */
/* k_new, v_new [batch][n_kv_heads][head_dim] pre-RoPE key / value of the  */
/*        new token (NULL with GEMMA_F_SHARED)                              */
/* seq_lens device int32 [batch]: sequence length INCLUDING the new token; */
/*        the new token sits at position seq_lens[b] - 1; every value must */
/*        be in [1, max_seq_len].                                          */
/* max_seq_len host upper bound of seq_lens (sizes the split-K grid).      */
/* out    [batch][n_q_heads][head_dim] bf16.                                */
/* workspace: at least gemma_attn_decode_workspace_size(...) bytes,        */
/*        256-byte aligned; contents are scratch.                          */
/*                                                                        */
/* Effect: the rotated new key and the new value are written at the slot   */
/* of position seq_lens[b]-1 (unless shared); then the query attends to   */
/* every visible cached position (global: all seq_lens[b] positions;      */
/* local: the last min(seq_lens[b], window) positions held by the ring).  */
/* The cache before the call must hold rotated keys for earlier positions.*/
/* ---------------------------------------------------------------------- */
size_t gemma_attn_decode_workspace_size(int batch, int n_q_heads, int n_kv_heads,
                                        int head_dim, int window, int max_seq_len);

int gemma_attn_decode(const void* q, const void* k_new, const void* v_new,
                      void* k_cache, void* v_cache, int cache_cap,
                      const int32_t* seq_lens, int max_seq_len, int batch,
                      int window, int n_q_heads, int n_kv_heads, int head_dim,
                      float rope_frac, float rope_theta, float scale, void* out,
                      void* workspace, size_t workspace_bytes, unsigned flags,
                      void* stream);

/* ---------------------------------------------------------------------- */
/* Multi-token decode: `tokens` new tokens per sequence, each attending to */
/* the cache and to the earlier new tokens -- the target model's pass that */
/* checks a drafter's proposals in speculative decoding ("Gemma 4: End-to- */
/* End Architecture Walkthrough", Phase 4, multi-token prediction drafters;*/
/* "Gemma 4: Architecture, Training and Local Deployment", 3.4). The       */
/* result equals tokens consecutive gemma_attn_decode calls (or a         */
/* gemma_attn_prefill of the tokens after seq_lens - tokens cached ones).  */
/*                                                                        */
/* q      [batch][tokens][n_q_heads][head_dim] pre-RoPE queries            */
/* k_new, v_new [batch][tokens][n_kv_heads][head_dim] pre-RoPE keys /      */
/*        values (NULL with GEMMA_F_SHARED; v_new NULL with GEMMA_F_KEQV)  */
/* seq_lens device int32 [batch]: sequence length INCLUDING the new        */
/*        tokens; token t sits at position seq_lens[b] - tokens + t. Every */
/*        value must be in [tokens, max_seq_len]; a device-side check      */
/*        reports others as GEMMA_ERR_DEVICE_RANGE.                        */
/* max_seq_len host upper bound of seq_lens (sizes the split grid).        */
/* out    [batch][tokens][n_q_heads][head_dim] bf16.                       */
/* workspace: gemma_attn_decode_multi_workspace_size(...) bytes, 256-byte  */
/*        aligned; scratch.                                                */
/*                                                                        */
/* bf16 layers (global ones contiguous or paged) run one tensor-core      */
/* kernel per split of the cached keys whose tile holds every q head of a */
/* KV head for all the tokens, so the cache is streamed once per step as  */
/* in single-token decode: global layers with (n_q_heads / n_kv_heads) *  */
/* tokens <= 128,                                                         */
/* unshared local layers with that product <= 64 and tokens <= window     */
/* (the ring is read as it was, plus the new rows; it is written after).  */
/* An int8 global layer takes the tokens one at a time through single-   */
/* token decode (its workspace does not grow with the cached length).     */
/* Other layers (int8 local, shared local, larger products) run as a      */
/* chunked prefill of the tokens after seq_lens - tokens cached ones; a   */
/* shared local layer needs GEMMA_F_SOURCE_WINDOW, with its source        */
/* layer's call passing it too (see that flag). Cache effects: the        */
/* rotated new keys and the values are written at their positions' slots, */
/* unless the layer is shared.                                            */
/* ---------------------------------------------------------------------- */
size_t gemma_attn_decode_multi_workspace_size(int batch, int tokens, int n_q_heads,
                                              int n_kv_heads, int head_dim, int window,
                                              int max_seq_len, int cache_cap, unsigned flags);

int gemma_attn_decode_multi(const void* q, const void* k_new, const void* v_new,
                            void* k_cache, void* v_cache, int cache_cap,
                            const int32_t* seq_lens, int max_seq_len, int batch, int tokens,
                            int window, int n_q_heads, int n_kv_heads, int head_dim,
                            float rope_frac, float rope_theta, float scale, void* out,
                            void* workspace, size_t workspace_bytes, unsigned flags,
                            void* stream);

/* ---------------------------------------------------------------------- */
/* Paged global cache ("Gemma 4: End-to-End Architecture Walkthrough", 3b: */
/* a global layer caches K/V for the whole context; paging lets the pool   */
/* grow with the tokens actually held instead of a per-sequence capacity). */
/* Global layers only (window 0); same arguments and behaviour as          */
/* gemma_attn_prefill / gemma_attn_decode except the cache:                */
/* k_pool, v_pool  [n_pages][n_kv_heads][page_size][head_dim] bf16: pages  */
/*        of page_size consecutive positions of one sequence.             */
/* page_table device int32 [batch][pages_per_seq]: position p of sequence */
/*        b is row p % page_size of page page_table[b][p / page_size].    */
/*        Entries for every page a call reads or writes (positions below  */
/*        seq_lens_before + s_new, or below seq_lens) must name a page of  */
/*        the pool; a device-side check reports any other as              */
/*        GEMMA_ERR_DEVICE_RANGE (nothing is written for it). Shared      */
/*        layers pass their source's pool and table. The caller owns the  */
/*        pool, the table and page allocation.                            */
/* page_size: a multiple of 128. pages_per_seq * page_size is the         */
/*        per-sequence capacity (the bound on seq_lens).                   */
/* GEMMA_F_KV_INT8: each pool is an int8 cache buffer of n_pages           */
/*        "sequences" of page_size rows: codes [n_pages][n_kv_heads]       */
/*        [page_size][head_dim], then (min, step) at byte offset           */
/*        gemma_kv_codes_bytes(n_pages, n_kv_heads, page_size, head_dim);  */
/*        size it with gemma_kv_cache_bytes(n_pages, n_kv_heads,           */
/*        page_size, head_dim, GEMMA_F_KV_INT8).                           */
/* ---------------------------------------------------------------------- */
int gemma_attn_prefill_paged(const void* q, const void* k_new, const void* v_new,
                             void* k_pool, void* v_pool, const int32_t* page_table,
                             int page_size, int pages_per_seq, int n_pages,
                             const int32_t* seq_lens_before, int batch, int s_new,
                             int n_q_heads, int n_kv_heads, int head_dim, float rope_frac,
                             float rope_theta, float scale, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, unsigned flags,
                             void* stream);
int gemma_attn_decode_paged(const void* q, const void* k_new, const void* v_new,
                            void* k_pool, void* v_pool, const int32_t* page_table,
                            int page_size, int pages_per_seq, int n_pages,
                            const int32_t* seq_lens, int max_seq_len, int batch,
                            int n_q_heads, int n_kv_heads, int head_dim, float rope_frac,
                            float rope_theta, float scale, void* out, void* workspace,
                            size_t workspace_bytes, unsigned flags, void* stream);
/* Multi-token decode (gemma_attn_decode_multi) on a paged global cache;   */
/* the workspace is gemma_attn_decode_multi_workspace_size(batch, tokens,  */
/* n_q_heads, n_kv_heads, head_dim, 0, max_seq_len, pages_per_seq *        */
/* page_size, flags).                                                      */
int gemma_attn_decode_multi_paged(const void* q, const void* k_new, const void* v_new,
                                  void* k_pool, void* v_pool, const int32_t* page_table,
                                  int page_size, int pages_per_seq, int n_pages,
                                  const int32_t* seq_lens, int max_seq_len, int batch, int tokens,
                                  int n_q_heads, int n_kv_heads, int head_dim, float rope_frac,
                                  float rope_theta, float scale, void* out, void* workspace,
                                  size_t workspace_bytes, unsigned flags, void* stream);

/* ---------------------------------------------------------------------- */
/* Decode without allocation. The pages have no counterpart for this entry */
/* point; it exists for callers that cannot obtain device memory for the  */
/* decode workspace -- e.g. a plugin inside a host runtime that owns all  */
/* device memory and offers it no allocator, or a latency-critical loop   */
/* where a cudaMalloc (and its implicit device-wide synchronisation) is   */
/* not acceptable and no buffer was reserved in advance.                  */
/*                                                                        */
/* Same arguments and effect as gemma_attn_decode without the workspace:  */
/* the split-K scratch comes from a fixed 32 MiB array compiled into the  */
/* library, which every GPU that loads the library's device code holds    */
/* until the process exits. The call allocates nothing (no cudaMalloc,    */
/* no cudaFree, no allocating library routine).                           */
/*   - A call whose gemma_attn_decode_workspace_size(...) exceeds 32 MiB   */
/*     returns GEMMA_ERR_CAPACITY with a message and enqueues nothing.     */
/*   - The first call on a device looks up the array's device address     */
/*     (cudaGetSymbolAddress) with that device current; make that first   */
/*     call before any stream capture. The address is kept for the life   */
/*     of the process: after a cudaDeviceReset (or any teardown of the    */
/*     device's context) the array may move, so a process that resets a  */
/*     device must not call this entry point on it again.                 */
/*   - Every call shares the one array and nothing in it needs to start at */
/*     zero (each call writes the scratch it reads). Calls that overlap on */
/*     the GPU (other streams, other host threads) race on it: serialise   */
/*     them.                                                              */
/* ---------------------------------------------------------------------- */
int gemma_attn_decode_noalloc(const void* q, const void* k_new, const void* v_new,
                              void* k_cache, void* v_cache, int cache_cap,
                              const int32_t* seq_lens, int max_seq_len, int batch,
                              int window, int n_q_heads, int n_kv_heads, int head_dim,
                              float rope_frac, float rope_theta, float scale, void* out,
                              unsigned flags, void* stream);

/* ---------------------------------------------------------------------- */
/* KV sharing ("Gemma 4 Architecture Reference", "Shared KV Cache").       */
/* Host only: no device work, no bytes move.                               */
/* ---------------------------------------------------------------------- */
typedef struct gemma_kv_desc {
    void* k_cache;      /* [batch][n_kv_heads][cache_cap][head_dim] bf16 */
    void* v_cache;
    int layer;          /* index of the layer in its stack */
    int cache_cap;
    int window;         /* 0 = global layer */
    int n_kv_heads;
    int head_dim;
    float rope_frac;
    float rope_theta;
    int shared_from;    /* -1: owns its cache; else the layer whose cache it reads */
    int k_eq_v;         /* 1: a GEMMA_F_KEQV layer (v_cache may be NULL) */
    int kv_int8;        /* 1: the caches are GEMMA_F_KV_INT8 buffers */
} gemma_kv_desc;

/* Makes dst read src's cache: dst->k_cache/v_cache become src's pointers and
 * dst->shared_from the layer that owns them (a chain resolves to its root).
 * Requires src->layer < dst->layer and identical window, cache_cap,
 * n_kv_heads, head_dim, rope_frac, rope_theta, k_eq_v and kv_int8 (same attention type);
 * otherwise returns GEMMA_ERR_SHARE_MISMATCH and leaves dst unchanged.
 * Afterwards call the attention entry points for dst with GEMMA_F_SHARED. */
int gemma_kv_share_bind(gemma_kv_desc* dst, const gemma_kv_desc* src);

/* Layer schedule of an n_layers stack with `ratio` local layers per global
 * layer ("Gemma 4: End-to-End Architecture Walkthrough", 3a): layer l is
 * global iff (l + 1) % (ratio + 1) == 0 or l == n_layers - 1. With the last
 * n_shared layers shared ("Shared KV Cache"), share_src[l] is the latest
 * non-shared earlier layer of the same type, l itself for a non-shared
 * layer, or -1 when a shared layer has no such source (it then keeps its own
 * cache). Host arrays of n_layers ints; share_src may be NULL. */
int gemma_layer_schedule(int n_layers, int ratio, int n_shared,
                         int* is_global, int* share_src);

/* Debug view of the mask logic the kernels use: for every (b, i) of a
 * prefill chunk writes {lo, hi, count} of the visible key positions to the
 * device int32 array ranges[batch][s_new][3] (count 0 -> lo > hi).
 * seq_lens_before as in gemma_attn_prefill. Asynchronous on `stream`. */
int gemma_attn_visible_ranges(const int32_t* seq_lens_before, int batch, int s_new,
                              int window, int32_t* ranges, void* stream);

/* Synchronises `stream`, then returns and clears the library's device error
 * word: GEMMA_OK, GEMMA_ERR_DEVICE_TIMEOUT (a bounded wait inside a kernel
 * gave up; that kernel's output is invalid), GEMMA_ERR_DEVICE_RANGE, or
 * GEMMA_ERR_CUDA if the synchronisation itself failed. */
int gemma_attn_sync_status(void* stream);

/* Message for the last failed call on this thread ("" if none). */
const char* gemma_last_error(void);

/* Deadline of every bounded device wait (pipeline barriers), in nanoseconds
 * of %globaltimer from the start of the waiting kernel's work unit. 0
 * restores the default of one second. Host state, process-wide; affects
 * launches issued afterwards. */
int gemma_attn_set_wait_limit(long long max_ns);

/* Test hook for the same path: when `enable` is nonzero, the next
 * gemma_attn_decode launch (or gemma_attn_decode_multi launch of the
 * tensor-core kernel) does not issue the first key/value copy of its
 * first work unit, so that unit's consumers wait on a barrier nothing will
 * complete; their bounded wait runs out, the unit exits without output and
 * gemma_attn_sync_status reports GEMMA_ERR_DEVICE_TIMEOUT. Nothing faults or
 * hangs. One-shot: the flag clears when that launch is issued. */
int gemma_attn_debug_drop_next_copy(int enable);

/* Diagnostics of the first bounded device wait that gave up since the last
 * call: info8[0] = 1 if one did (0 otherwise), [1] = wait site, [2..4] =
 * site-specific indices (work item, ring slot, stage), [5] = the raw
 * 64-bit barrier word at give-up time, [6] = block index (x | y << 20 |
 * z << 40), [7] = awaited phase parity. Reading clears the record. */
int gemma_attn_debug_timeout_info(long long* info8);

/* ---------------------------------------------------------------------- */
/* Measurement hook. While enabled, every launch of the kernels below is   */
/* bracketed by a pair of CUDA events recorded on the call's stream (event */
/* objects are created by the library; no device memory is allocated).    */
/* gemma_attn_profile_read synchronises the recorded events and returns    */
/* the summed device time and the launch count of one kernel kind since    */
/* the last gemma_attn_profile(1). gemma_attn_profile(0) stops recording   */
/* and releases the events.                                                */
/* ---------------------------------------------------------------------- */
#define GEMMA_KERNEL_PREFILL_ROPE 0     /* RoPE on Q/K + cache write (prefill) */
#define GEMMA_KERNEL_PREFILL_ATTN 1     /* prefill attention */
#define GEMMA_KERNEL_DECODE_APPEND 2    /* RoPE + cache append (decode) */
#define GEMMA_KERNEL_DECODE_SPLIT 3     /* split-K decode attention */
#define GEMMA_KERNEL_DECODE_COMBINE 4   /* log-sum-exp combine of the splits */
#define GEMMA_KERNEL_KINDS 5

int gemma_attn_profile(int enable);
int gemma_attn_profile_read(int kernel, double* total_ms, long long* launches);

#ifdef __cplusplus
}
#endif

#endif /* GEMMA_ATTN_H */
