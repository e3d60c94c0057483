// kernels.h -- launch interfaces between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hlg {

typedef __nv_bfloat16 bf16;

struct PrefillRopeArgs {
  const bf16* q;       // [B][S][Hq][D]
  const bf16* k_new;   // [B][S][Hkv][D] or null (shared layer)
  const bf16* v_new;   // [B][S][Hkv][D] or null
  bf16* q_rot;         // workspace [B][S][Hq][D]
  bf16* k_rot;         // workspace, local layers: [B][S][Hkv][D], or with win_rows > 0
                       // [B][win_rows][Hkv][D] with the chunk at rows window.. (or, with
                       // win_at_pos, at rows seq_lens_before[b]..); else null
  bf16* v_win;         // key windows (chunked prefill): V window [B][win_rows][Hkv][D], else null
  int win_rows;        // 0, or the window rows per sequence: window + S (chunked local prefill)
                       // or cache_cap (int8 global prefill after cached tokens)
  int win_at_pos;      // 1: a chunk token's window row is its position
  bf16* k_cache;       // [B][Hkv][cap][D]
  bf16* v_cache;
  int cache_cap;
  const int32_t* seq_lens_before;  // device [B] or null
  int S, window, Hq, Hkv;
  int n_rot;           // rotated pairs
  double log2_theta;
  float q_scale;       // rotated Q is multiplied by this before the bf16 rounding
  int quant;           // int8 cache: rotated K goes to k_rot ([B][S][Hkv][D], or its window rows
                       // with win_rows > 0) on every layer type and nothing is written into the
                       // cache (launch_quantize_rows does)
  // cache pages (see cache_row): table [B][pages_per_seq] or null for a
  // contiguous cache (page_size = cache_cap, n_pages = B)
  const int32_t* page_table;
  int page_size, pages_per_seq, n_pages;
  int* status;
};

struct DecodeRopeArgs {
  const bf16* q;       // [B][tokens][Hq][D]
  const bf16* k_new;   // [B][tokens][Hkv][D] or null
  const bf16* v_new;
  bf16* q_rot;         // workspace [B][tokens][Hq][D]
  int tokens;          // new tokens per sequence, at positions len - tokens .. len - 1 (decode: 1)
  float q_scale;       // rotated q is multiplied by this before the bf16 rounding (decode: 1)
  int skip_q;          // 1: the new K/V only (q and q_rot are not touched)
  bf16* k_cache;
  bf16* v_cache;
  bf16* k_stage;       // int8 cache: the rotated new key goes here ([B][Hkv][D]) and nothing
                       // is written into the cache (launch_quantize_rows does); else null
  int cache_cap;
  const int32_t* seq_lens;
  int max_len, window, Hq, Hkv;
  int n_rot;
  double log2_theta;
  // cache pages (see cache_row): table [B][pages_per_seq] or null for a
  // contiguous cache (page_size = cache_cap, n_pages = B)
  const int32_t* page_table;
  int page_size, pages_per_seq, n_pages;
  int* status;
};

// int8 cache rows: the bf16 rows src + ((b * S + s) * Hkv + h) * D (b < B,
// s < S, h < Hkv) at positions pos = pos0[b] - pos0_minus + s are quantized
// (per row: min, step = (max - min) / 255, codes round((x - min) * 255 /
// (max - min)), fp32) into slot pos (global) or pos % window (local, only
// the last `window` rows of the chunk) of codes [B][Hkv][cap][D] and
// params [B][Hkv][cap] (min, step).
struct QuantRowsArgs {
  const bf16* src;     // [B][src_rows][Hkv][D]; chunk token s at row s (src_row_mode 0),
  int src_rows;        // window + s (1) or its position (2)
  int src_row_mode;
  int S, Hkv, window, cache_cap;  // cache_cap: positions per sequence (range check)
  const int32_t* pos0;  // device [B], or null for 0
  int pos0_minus;
  uint8_t* codes;       // rows addressed by cache_row (codes [rows][D], params [rows])
  float2* params;
  const int32_t* page_table;  // null: contiguous (page_size = cache_cap, n_pages = B)
  int page_size, pages_per_seq, n_pages;
  int* status;
};

// Keys/values of one prefill layer as strided 4-D views (b, row, head, d);
// row = key position. Global layers read the cache, local layers the
// rotated-K workspace and the caller's V.
struct KVView {
  const bf16* ptr;
  int64_t stride_b, stride_row, stride_h;  // in elements; d is contiguous
};

struct PrefillAttnArgs {
  const bf16* q_rot;   // [B][S][Hq][D]
  KVView k, v;
  int64_t key_cap;     // rows readable per (batch, head) in the K/V views
  int key_off_window;  // 1: view row = position - (seq_lens_before[b] - window) (a key window
                       // gathered for chunked local prefill); 0: view row = position
  const int32_t* seq_lens_before;  // device [B] or null
  int S, window, Hq, Hkv;
  float scale_log2;    // scale * log2(e)
  bf16* out;           // [B][S][Hq][D]
  float* lse;          // [B][Hq][S] or null
  int* status;
  unsigned long long wait_ns;
  // cache pages (see cache_row): table [B][pages_per_seq] or null for a
  // contiguous cache; a paged cache is read through head-major
  // views of the pool: view row = position % page_size, view batch = page
  const int32_t* page_table;
  int page_size, pages_per_seq, n_pages;
};

struct DecodeAttnArgs {
  const bf16* q_rot;       // [B][Hq][D]
  const bf16* k_cache;     // [B][Hkv][cap][D], or a pool [n_pages][Hkv][page_size][D]
  const bf16* v_cache;
  int cache_cap;           // positions per sequence
  const int32_t* seq_lens; // device [B]
  int max_len, window, Hq, Hkv;
  int chunk;               // keys per split (multiple of 16)
  int n_splits;
  float scale_log2;
  float* part_o;           // [B][tokens][Hq][n_splits][D]
  float* part_lse;         // [B][tokens][Hq][n_splits] (log2 domain)
  bf16* out;               // [B][tokens][Hq][D]
  int tokens;              // query tokens per sequence (decode: 1; the combine's rows)
  int* status;
  unsigned long long wait_ns;
  int drop_first_copy;     // test hook: skip the first K/V copy of split 0
  int every_split;         // 1: every planned split wrote a partial (multi-token local layers)
  int keqv;                // K = V: only K rows are loaded and serve as V
  // int8 cache (k_cache/v_cache unused): codes [B][Hkv][cap][D] and per-row (min, step),
  // or the same over the pages of a pool
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const float2* k_params;
  const float2* v_params;
  // cache pages (see cache_row): table [B][pages_per_seq] or null for a
  // contiguous cache (page_size = cache_cap, n_pages = B)
  const int32_t* page_table;
  int page_size, pages_per_seq, n_pages;
};

cudaError_t launch_prefill_rope(const PrefillRopeArgs& a, int B, int D, cudaStream_t st);
// Chunked local prefill: copies the ring's K/V of positions
// seq_lens_before[b] - window .. seq_lens_before[b] - 1 into rows 0..window-1
// of the K and V windows (zeros for negative positions).
cudaError_t launch_ring_gather(const bf16* k_cache, const bf16* v_cache, const int32_t* seq_lens_before,
                               int B, int Hkv, int D, int window, int win_rows, bf16* k_win, bf16* v_win,
                               int* status, cudaStream_t st);
// Int8 caches: dequantize cached rows (min + code * step, rounded to bf16)
// into key windows [B][win_rows][Hkv][D]; pos0 = seq_lens_before[b] (0 if
// null), plus `extra` positions (a shared layer's chunk). window > 0: the
// ring's positions pos0-window .. pos0+extra-1 into rows 0.. (negative
// positions: zeros); window 0: positions 0 .. pos0+extra-1 into rows 0.. .
// Rows below first_row are not written. v_codes null: K only.
// Cached rows are addressed by cache_row (page_table null: contiguous,
// page_size = cache_cap, n_pages = B).
cudaError_t launch_gather_q8(const uint8_t* k_codes, const float2* k_params, const uint8_t* v_codes,
                             const float2* v_params, const int32_t* seq_lens_before, int extra, int B, int Hkv,
                             int D, int window, int cache_cap, const int32_t* page_table, int page_size,
                             int pages_per_seq, int n_pages, int win_rows, int first_row, bf16* k_win, bf16* v_win,
                             int* status, cudaStream_t st);
cudaError_t launch_decode_rope_append(const DecodeRopeArgs& a, int B, int D, cudaStream_t st);
cudaError_t launch_lens_minus(const int32_t* seq_lens, int32_t* lens_before, int B, int tokens, cudaStream_t st);

// Multi-token decode on a global layer (several new tokens per sequence, each
// seeing the cache and the earlier new tokens), over splits of `chunk` keys,
// writing per-split partials for launch_decode_combine. Up to 64 query rows
// (G q heads x tokens) a KV head: the transposed tensor-core kernel (query
// rows as the MMA's N, one CTA per KV head and split); more: the prefill
// kernel's 128-row tile over those rows (launch_verify_attn_rows; two CTAs
// per KV head at head_dim 512). verify_tc_rows gives the first kernel's
// padded row count, 0 when the second one runs.
struct VerifyAttnArgs {
  const bf16* q_rot;        // [B][tokens][Hq][D], times scale * log2(e)
  KVView k, v;              // head-major cache views [B][Hkv][cap][D]
  int cache_cap;
  // window > 0 (local layer, transposed kernel only): the cache is the ring
  // of `window` slots as it was before the new tokens (slot = position %
  // window); the new tokens' rotated keys and values are read from k_tail /
  // v_tail [B][tokens][Hkv][D], and every split writes a partial.
  int window;
  const bf16* k_tail;
  const bf16* v_tail;
  // cache pages (global layers): k / v are head-major views of a pool of
  // n_pages pages of page_size rows, position p of sequence b at row
  // p % page_size of page page_table[b][p / page_size]; page_table null:
  // contiguous (page_size = cache_cap, n_pages = B)
  const int32_t* page_table;
  int page_size, pages_per_seq, n_pages;
  const int32_t* seq_lens;  // device [B], including the new tokens
  int tokens, Hq, Hkv;
  int chunk, n_splits;      // keys per split (a multiple of 128), splits planned
  float* part_o;            // [B][tokens][Hq][n_splits][D]
  float* part_lse;          // [B][tokens][Hq][n_splits] (log2 domain)
  bf16* out;                // transposed kernel, one split: the output [B][tokens][Hq][D]
                            // written directly (no partials); else null
  int* status;
  unsigned long long wait_ns;
  int drop_first_copy;      // test hook (transposed kernel): skip the first K copy of unit 0
};
cudaError_t launch_verify_attn_tc(const VerifyAttnArgs& a, int B, int D, cudaStream_t st);
cudaError_t launch_verify_attn_rows(const VerifyAttnArgs& a, int B, int D, cudaStream_t st);
int verify_tc_rows(int Hq, int Hkv, int tokens, int D);
cudaError_t launch_quantize_rows(const QuantRowsArgs& a, int B, int D, cudaStream_t st);
// tcgen05 prefill (head_dim 256 or 512). key_rows_total = rows of the K/V
// views; kv_token_major: views are [B][rows][Hkv][D] (1) or [B][Hkv][rows][D] (0).
// _tc: one CTA per 128-row query tile; _pair: two query tiles on a CTA pair
// sharing each MMA (cta_group::2).
cudaError_t launch_prefill_attn_tc(const PrefillAttnArgs& a, int B, int D, int key_rows_total,
                                   int kv_token_major, cudaStream_t st);
// head_pair: the pair takes two q heads of one KV head on the same query
// tile (used when q heads per KV head is even) instead of two query tiles.
cudaError_t launch_prefill_attn_pair(const PrefillAttnArgs& a, int B, int D, int key_rows_total,
                                     int kv_token_major, int head_pair, cudaStream_t st);
cudaError_t launch_decode_split(const DecodeAttnArgs& a, int B, int D, cudaStream_t st);
// int8 cache: the same split-K decode reading codes and (min, step) rows
cudaError_t launch_decode_split_q8(const DecodeAttnArgs& a, int B, int D, cudaStream_t st);
cudaError_t launch_decode_combine(const DecodeAttnArgs& a, int B, int D, cudaStream_t st);
cudaError_t launch_visible_ranges(const int32_t* seq_lens_before, int B, int S, int window,
                                  int32_t* ranges, cudaStream_t st);

}  // namespace hlg
