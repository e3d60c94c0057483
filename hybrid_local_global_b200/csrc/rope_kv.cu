// rope_kv.cu -- (p-)RoPE on Q/K and the KV-cache write path.
//
// RoPE ("Gemma 4: End-to-End Architecture Walkthrough", 3c "p-RoPE";
// "Gemma 4 Architecture Reference", "Positional Encoding: Proportional RoPE"):
// pair i = (2i, 2i+1) of a head vector turns by pos * theta^(-2i/D) when
// i < floor(rope_frac * D / 2) and is copied unchanged otherwise. Local layers
// use rope_frac = 1 (standard RoPE); global layers rope_frac = 0.25,
// theta = 1e6.
//
// Cache ("Gemma 4: End-to-End Architecture Walkthrough", 3b; "Gemma 4 Deep
// Dive" talk): a global layer appends position p at slot p; a local layer
// keeps a ring of `window` slots, position p at slot p % window.
//
// Precision: the angle pos * inv_freq is formed in half-turns (units of pi)
// and reduced to [-1, 1] in fp64 (an fp32 product has an ulp of 1/64 rad
// near position 2.6e5), then sincospif of the reduced angle, which needs no
// further argument reduction; the rotation itself is fp32 and the result is
// rounded to bf16 (round to nearest even).
//
// Thread map: threadIdx.x owns 8 consecutive elements (4 pairs) of the head
// vector, so its inverse frequencies are computed once and each angle once
// per position, then reused for every Q and K head of that position.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace hlg {

namespace {

constexpr double kInvPi = 0.31830988618379067153776752674503;

struct PairTrig {
  float c[4], s[4];
  bool any_rot;  // false -> the whole 8-element chunk is copied unchanged
};

__device__ __forceinline__ void chunk_inv_freq(int e0, int D, int n_rot, double log2_theta,
                                               double (&inv_freq)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    int i = e0 / 2 + j;
    // theta^(-2i/D) radians per position, expressed in half-turns
    inv_freq[j] = (i < n_rot) ? exp2(-(2.0 * (double)i / (double)D) * log2_theta) * kInvPi : 0.0;
  }
}

__device__ __forceinline__ PairTrig chunk_trig(int64_t pos, int e0, int n_rot,
                                               const double (&inv_freq)[4]) {
  PairTrig t;
  t.any_rot = (e0 / 2) < n_rot;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (e0 / 2 + j < n_rot) {
      const double a = (double)pos * inv_freq[j];  // half-turns
      const double r = a - 2.0 * rint(0.5 * a);     // in [-1, 1]
      sincospif((float)r, &t.s[j], &t.c[j]);
    } else {
      t.c[j] = 1.f;
      t.s[j] = 0.f;
    }
  }
  return t;
}

__device__ __forceinline__ uint4 rotate_chunk(uint4 x, const PairTrig& t, int e0, int n_rot) {
  if (!t.any_rot) return x;
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (e0 / 2 + j < n_rot) {
      float2 v = unpack_bf16x2(w[j]);
      float y0 = v.x * t.c[j] - v.y * t.s[j];
      float y1 = v.x * t.s[j] + v.y * t.c[j];
      w[j] = pack_bf16x2(y0, y1);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Rotation followed by a multiplication by `qs`, rounded to bf16 once (the
// prefill attention kernel takes queries pre-multiplied by scale * log2(e),
// so its logits come out in log2 units without a per-score multiply).
__device__ __forceinline__ uint4 rotate_scale_chunk(uint4 x, const PairTrig& t, int e0, int n_rot, float qs) {
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float2 v = unpack_bf16x2(w[j]);
    float y0 = v.x, y1 = v.y;
    if (e0 / 2 + j < n_rot) {
      y0 = v.x * t.c[j] - v.y * t.s[j];
      y1 = v.x * t.s[j] + v.y * t.c[j];
    }
    w[j] = pack_bf16x2(y0 * qs, y1 * qs);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 ld16(const bf16* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st16(bf16* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// Streaming read of an input that is not read again: L2 evict-first, so the
// rotated outputs that the attention kernel reads next stay in L2.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint4 ld16_stream(const bf16* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

constexpr int ROPE_HB = 8;     // head vectors loaded before the first store
constexpr int ROPE_RPT = 2;    // positions per thread, unless that leaves fewer than
constexpr int ROPE_MIN_CTAS = 512;  // this many CTAs (about 3.5 per SM): then one

// Prefill: rotate the chunk's Q into q_rot (times q_scale), rotate K and write
// it (global: cache slot pos; local: the k_rot workspace the attention kernel
// reads, plus the ring slot for the last `window` positions); V goes to the
// cache slot (global) or, only for the last `window` positions, the ring
// (local: the attention kernel reads the caller's V directly). With an int8
// cache (a.quant) every layer type writes only k_rot; the quantize kernel
// fills the cache from k_rot and the caller's V.
//
// threadIdx.x owns 8 elements of the head vector, threadIdx.y one position
// (of one or ROPE_RPT per thread, as the grid was sized: a CTA covers
// ceil(S / (gridDim.x * blockDim.y)) rows of blockDim.y positions, so every
// position has exactly one thread): the angles of a position are formed once and
// serve all Hq + 2 Hkv head vectors, which are loaded ROPE_HB at a time so
// several 16-byte loads are in flight per thread.
// WIN: chunked local prefill, where the chunk's rotated K and its V go to
// rows window.. of the K and V windows (a.win_rows rows per sequence).
template <int D, bool WIN>
__global__ void __launch_bounds__(256, 2) k_prefill_rope(PrefillRopeArgs a) {
  const int b = blockIdx.y;
  const int e0 = threadIdx.x * 8;
  const int64_t pos0 = a.seq_lens_before ? (int64_t)a.seq_lens_before[b] : 0;
  if (pos0 < 0 || (a.window == 0 && pos0 + a.S > a.cache_cap)) {
    if (threadIdx.x == 0 && threadIdx.y == 0 && blockIdx.x == 0)
      set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  const uint64_t pol = policy_evict_first();
  double inv_freq[4];
  chunk_inv_freq(e0, D, a.n_rot, a.log2_theta, inv_freq);
  const int rpt = (a.S + gridDim.x * blockDim.y - 1) / (gridDim.x * blockDim.y);
#pragma unroll 1
  for (int rep = 0; rep < rpt; ++rep) {
    const int s = (blockIdx.x * rpt + rep) * blockDim.y + threadIdx.y;
    if (s >= a.S) break;
    const int64_t pos = pos0 + s;
    const PairTrig t = chunk_trig(pos, e0, a.n_rot, inv_freq);
    const int64_t row = (int64_t)b * a.S + s;
    // queries
#pragma unroll 1
    for (int h0 = 0; h0 < a.Hq; h0 += ROPE_HB) {
      uint4 x[ROPE_HB];
#pragma unroll
      for (int u = 0; u < ROPE_HB; ++u)
        if (h0 + u < a.Hq) x[u] = ld16_stream(a.q + (row * a.Hq + h0 + u) * D + e0, pol);
#pragma unroll
      for (int u = 0; u < ROPE_HB; ++u)
        if (h0 + u < a.Hq)
          st16(a.q_rot + (row * a.Hq + h0 + u) * D + e0, rotate_scale_chunk(x[u], t, e0, a.n_rot, a.q_scale));
    }
    if (!a.k_new) continue;  // shared layer: no K/V of its own
    const bool to_ring = a.window > 0 && s >= a.S - a.window && !a.quant;
    const int64_t slot = a.window > 0 ? pos % a.window : pos;
#pragma unroll 1
    for (int h0 = 0; h0 < a.Hkv; h0 += ROPE_HB / 2) {
      uint4 kx[ROPE_HB / 2], vx[ROPE_HB / 2];
#pragma unroll
      for (int u = 0; u < ROPE_HB / 2; ++u) kx[u] = vx[u] = make_uint4(0, 0, 0, 0);
      // no v_new: K = V; the V window (WIN) takes every position of the chunk
      const bool want_v = a.v_new && (WIN || (!a.quant && (a.window == 0 || to_ring)));
      // k_rot / V window row
      const int64_t wrow = WIN ? (int64_t)b * a.win_rows + (a.win_at_pos ? pos : a.window + s) : row;
#pragma unroll
      for (int u = 0; u < ROPE_HB / 2; ++u)
        if (h0 + u < a.Hkv) {
          const int64_t off = (row * a.Hkv + h0 + u) * D + e0;
          kx[u] = ld16_stream(a.k_new + off, pol);
          if (want_v) vx[u] = ld16_stream(a.v_new + off, pol);
        }
#pragma unroll
      for (int u = 0; u < ROPE_HB / 2; ++u)
        if (h0 + u < a.Hkv) {
          const int kh = h0 + u;
          const uint4 kr = rotate_chunk(kx[u], t, e0, a.n_rot);
          int64_t crow = 0;
          if ((a.window == 0 && !a.quant) || to_ring) {
            crow = cache_row(a.page_table, a.pages_per_seq, a.page_size, a.n_pages, a.Hkv, b, kh, slot);
            if (crow < 0) {  // a page outside the pool: report, write nothing
              set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
              continue;
            }
          }
          const int64_t cslot = crow * D + e0;
          if (a.window == 0 && !a.quant) {
            st16(a.k_cache + cslot, kr);
            if (want_v) st16(a.v_cache + cslot, vx[u]);
          } else {
            st16(a.k_rot + (wrow * a.Hkv + kh) * D + e0, kr);
            if (WIN) st16(a.v_win + (wrow * a.Hkv + kh) * D + e0, vx[u]);
            if (to_ring) {
              st16(a.k_cache + cslot, kr);
              if (want_v) st16(a.v_cache + cslot, vx[u]);
            }
          }
        }
    }
  }
}

// Chunked local prefill: before the chunk overwrites ring slots, copy the
// ring's keys and values of positions pos0-window .. pos0-1 (pos0 =
// seq_lens_before[b]) into rows 0..window-1 of the K and V windows; the
// RoPE kernel then writes the chunk at rows window.. . Negative positions
// become zeros (they are never visible). One CTA per 8 rows of a sequence.
template <int D>
__global__ void __launch_bounds__(256) k_ring_gather(const bf16* __restrict__ k_cache,
                                                     const bf16* __restrict__ v_cache,
                                                     const int32_t* seq_lens_before, int Hkv, int window,
                                                     int win_rows, bf16* k_win, bf16* v_win, int* status) {
  const int b = blockIdx.y;
  const int64_t pos0 = seq_lens_before[b];
  if (pos0 < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  constexpr int CH = D / 8;  // 16-byte chunks per head vector
  const int r0 = blockIdx.x * 8;
  for (int idx = threadIdx.x; idx < 8 * Hkv * CH; idx += blockDim.x) {
    const int r = r0 + idx / (Hkv * CH);
    if (r >= window) break;
    const int h = (idx / CH) % Hkv, c = (idx % CH) * 8;
    const int64_t p = pos0 - window + r;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (p >= 0) {
      const int64_t src = (((int64_t)b * Hkv + h) * window + p % window) * D + c;
      kv = ld16(k_cache + src);
      vv = ld16(v_cache + src);
    }
    const int64_t dst = (((int64_t)b * win_rows + r) * Hkv + h) * D + c;
    st16(k_win + dst, kv);
    st16(v_win + dst, vv);
  }
}

// Int8 caches: the key windows of a prefill that reads cached rows, from
// the codes. A warp dequantizes one cached row (one position, one KV head):
// value = min + code * step in fp32, rounded to bf16. With pos0 =
// seq_lens_before[b] (0 if null) and `extra` more positions (a shared
// layer's chunk, already in the cache): window > 0: rows 0..window+extra-1
// take positions pos0-window .. pos0+extra-1 (slot p mod window; negative
// positions give zeros, never visible); window 0: rows 0..pos0+extra-1 take
// positions 0..pos0+extra-1 (slot = position). Rows below first_row are
// left as they are (a shared layer's chunk re-read over its source's window).
template <int D>
__global__ void __launch_bounds__(256) k_gather_q8(const uint8_t* __restrict__ k_codes,
                                                   const float2* __restrict__ k_params,
                                                   const uint8_t* __restrict__ v_codes,
                                                   const float2* __restrict__ v_params,
                                                   const int32_t* seq_lens_before, int extra, int Hkv,
                                                   int window, int cache_cap, const int32_t* page_table,
                                                   int page_size, int pages_per_seq, int n_pages, int win_rows,
                                                   int first_row, bf16* k_win, bf16* v_win, int* status) {
  constexpr int E = D / 32;  // codes per lane: 8 or 16
  const int b = blockIdx.y;
  const int64_t pos0 = seq_lens_before ? (int64_t)seq_lens_before[b] : 0;
  const int64_t rows = window > 0 ? (int64_t)window + extra : pos0 + extra;
  if (pos0 < 0 || rows > win_rows || (window == 0 && rows > cache_cap)) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int64_t n_items = rows * Hkv;
  for (int64_t it = (int64_t)first_row * Hkv + (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); it < n_items;
       it += (int64_t)gridDim.x * 8) {
    const int64_t r = it / Hkv;
    const int h = (int)(it % Hkv);
    const int64_t p = window > 0 ? pos0 - window + r : r;
    const int64_t dst = (((int64_t)b * win_rows + r) * Hkv + h) * D + lane * E;
    for (int kv = 0; kv < (v_codes ? 2 : 1); ++kv) {
      bf16* out = (kv ? v_win : k_win) + dst;
      uint32_t packed[E / 2];
      const int64_t crow =
          p < 0 ? -1 : cache_row(page_table, pages_per_seq, page_size, n_pages, Hkv, b, h, window > 0 ? p % window : p);
      if (p >= 0 && crow < 0 && lane == 0) set_status(status, GEMMA_ERR_DEVICE_RANGE);  // page outside the pool
      if (crow < 0) {
#pragma unroll
        for (int i = 0; i < E / 2; ++i) packed[i] = 0;
      } else {
        const float2 mp = (kv ? v_params : k_params)[crow];
        const uint8_t* cp = (kv ? v_codes : k_codes) + crow * D + lane * E;
        uint32_t w[E / 4];
        if constexpr (E == 8) {
          const uint2 u = *reinterpret_cast<const uint2*>(cp);
          w[0] = u.x;
          w[1] = u.y;
        } else {
          const uint4 u = *reinterpret_cast<const uint4*>(cp);
          w[0] = u.x;
          w[1] = u.y;
          w[2] = u.z;
          w[3] = u.w;
        }
#pragma unroll
        for (int i = 0; i < E / 2; ++i) {
          const uint32_t word = w[i / 2];
          const float c0 = (float)((word >> (16 * (i % 2))) & 0xffu);
          const float c1 = (float)((word >> (16 * (i % 2) + 8)) & 0xffu);
          packed[i] = pack_bf16x2(__fmaf_rn(c0, mp.y, mp.x), __fmaf_rn(c1, mp.y, mp.x));
        }
      }
      if constexpr (E == 8) {
        *reinterpret_cast<uint4*>(out) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      } else {
        *reinterpret_cast<uint4*>(out) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        *reinterpret_cast<uint4*>(out + 8) = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      }
    }
  }
}

// Decode: one token per sequence at position seq_lens[b]-1.
template <int D>
__global__ void __launch_bounds__(256) k_decode_rope_append(DecodeRopeArgs a) {
  // one block per (sequence, new token): bt = b * tokens + t, the layout of
  // q, k_new, v_new and q_rot
  const int bt = blockIdx.x;
  const int b = bt / a.tokens;
  const int e0 = threadIdx.x * 8;
  const int64_t len = a.seq_lens[b];
  if (len < a.tokens || len > a.max_len) {
    if (threadIdx.x == 0 && threadIdx.y == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  const int64_t pos = len - a.tokens + bt % a.tokens;
  const int64_t slot = a.window > 0 ? pos % a.window : pos;
  if (slot >= a.cache_cap) {
    if (threadIdx.x == 0 && threadIdx.y == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  double inv_freq[4];
  chunk_inv_freq(e0, D, a.n_rot, a.log2_theta, inv_freq);
  const PairTrig t = chunk_trig(pos, e0, a.n_rot, inv_freq);
  // q heads, then K heads, then V heads (none when shared, none for V under
  // K = V, none with an int8 cache: the quantize kernel reads the caller's V)
  const int n_heads = a.Hq + (a.k_new ? a.Hkv : 0) + ((a.v_new && !a.k_stage) ? a.Hkv : 0);
  for (int h = threadIdx.y + (a.skip_q ? a.Hq : 0); h < n_heads; h += blockDim.y) {
    if (h < a.Hq) {
      const int64_t off = ((int64_t)bt * a.Hq + h) * D + e0;
      const uint4 x = ld16(a.q + off);
      st16(a.q_rot + off, a.q_scale == 1.f ? rotate_chunk(x, t, e0, a.n_rot)
                                           : rotate_scale_chunk(x, t, e0, a.n_rot, a.q_scale));
      continue;
    }
    const bool is_k = h < a.Hq + a.Hkv;
    const int kh = is_k ? h - a.Hq : h - a.Hq - a.Hkv;
    const int64_t src_off = ((int64_t)bt * a.Hkv + kh) * D + e0;
    uint4 v = is_k ? rotate_chunk(ld16(a.k_new + src_off), t, e0, a.n_rot)
                   : ld16(a.v_new + src_off);
    if (a.k_stage) {  // int8 cache: the rotated key waits for the quantize kernel
      st16(a.k_stage + src_off, v);
      continue;
    }
    bf16* cache = is_k ? a.k_cache : a.v_cache;
    const int64_t crow = cache_row(a.page_table, a.pages_per_seq, a.page_size, a.n_pages, a.Hkv, b, kh, slot);
    if (crow < 0) {  // a page outside the pool: report, write nothing
      set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
      continue;
    }
    st16(cache + crow * D + e0, v);
  }
}

// int8 cache rows ("Gemma 4 Technical Report", Quantization and Efficiency:
// code = round((x - min) * (2^b - 1) / (max - min)), value min + code /
// scale; here b = 8 and one (min, step) per cached row). One warp per row,
// D / 32 elements per lane; every step of the code decision is fp32 with
// round-to-nearest (IEEE division, no contraction), ties to even; a
// constant row gets codes 0 and step 0.
template <int D>
__global__ void __launch_bounds__(256) k_quantize_rows(QuantRowsArgs a, int n_rows) {
  constexpr int E = D / 32;  // 8 or 16
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const int h = row % a.Hkv;
  const int s = (row / a.Hkv) % a.S;
  const int b = row / (a.Hkv * a.S);
  const int64_t pos = (a.pos0 ? (int64_t)a.pos0[b] - a.pos0_minus : 0) + s;
  if (pos < 0) {
    if (lane == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  if (a.window > 0 && s < a.S - a.window) return;  // only the chunk's last `window` rows reach the ring
  const int64_t slot = a.window > 0 ? pos % a.window : pos;
  if (slot >= a.cache_cap) {
    if (lane == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  const int64_t srow = a.src_row_mode == 0 ? s : a.src_row_mode == 1 ? (int64_t)a.window + s : pos;
  const bf16* src = a.src + (((int64_t)b * a.src_rows + srow) * a.Hkv + h) * D + lane * E;
  float x[E];
#pragma unroll
  for (int c = 0; c < E / 8; ++c) {
    const uint4 u = ld16(src + c * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf16x2(w[j]);
      x[c * 8 + 2 * j] = f.x;
      x[c * 8 + 2 * j + 1] = f.y;
    }
  }
  float lo = x[0], hi = x[0];
#pragma unroll
  for (int e = 1; e < E; ++e) {
    lo = fminf(lo, x[e]);
    hi = fmaxf(hi, x[e]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const float range = __fsub_rn(hi, lo);
  uint32_t packed[E / 4];
#pragma unroll
  for (int i = 0; i < E / 4; ++i) packed[i] = 0;
  if (range > 0.f) {
    const float scale = __fdiv_rn(255.f, range);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      int c = __float2int_rn(__fmul_rn(__fsub_rn(x[e], lo), scale));
      c = c < 0 ? 0 : (c > 255 ? 255 : c);
      packed[e / 4] |= (uint32_t)c << (8 * (e % 4));
    }
  }
  const int64_t crow = cache_row(a.page_table, a.pages_per_seq, a.page_size, a.n_pages, a.Hkv, b, h, slot);
  if (crow < 0) {  // a page outside the pool: report, write nothing
    if (lane == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  uint8_t* dst = a.codes + crow * D + lane * E;
  if (E == 8)
    *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
  else
    *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[E / 4 > 2 ? 2 : 0], packed[E / 4 > 3 ? 3 : 0]);
  if (lane == 0) a.params[crow] = make_float2(lo, range > 0.f ? __fdiv_rn(range, 255.f) : 0.f);
}

}  // namespace

cudaError_t launch_quantize_rows(const QuantRowsArgs& a, int B, int D, cudaStream_t st) {
  const int n_rows = B * a.S * a.Hkv;
  if (n_rows <= 0) return cudaSuccess;
  const int grid = (n_rows + 7) / 8;
  if (D == 256)
    k_quantize_rows<256><<<grid, 256, 0, st>>>(a, n_rows);
  else
    k_quantize_rows<512><<<grid, 256, 0, st>>>(a, n_rows);
  return cudaGetLastError();
}

cudaError_t launch_prefill_rope(const PrefillRopeArgs& a, int B, int D, cudaStream_t st) {
  const int tx = D / 8;
  dim3 block(tx, 256 / tx);
  int per_cta = block.y * ROPE_RPT;
  if ((int64_t)((a.S + per_cta - 1) / per_cta) * B < ROPE_MIN_CTAS) per_cta = block.y;
  dim3 grid((a.S + per_cta - 1) / per_cta, B);
  const bool win = a.win_rows > 0 && a.v_win;
  if (D == 256) {
    if (win) k_prefill_rope<256, true><<<grid, block, 0, st>>>(a);
    else k_prefill_rope<256, false><<<grid, block, 0, st>>>(a);
  } else {
    if (win) k_prefill_rope<512, true><<<grid, block, 0, st>>>(a);
    else k_prefill_rope<512, false><<<grid, block, 0, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_ring_gather(const bf16* k_cache, const bf16* v_cache, const int32_t* seq_lens_before,
                               int B, int Hkv, int D, int window, int win_rows, bf16* k_win, bf16* v_win,
                               int* status, cudaStream_t st) {
  dim3 grid((window + 7) / 8, B);
  if (D == 256)
    k_ring_gather<256><<<grid, 256, 0, st>>>(k_cache, v_cache, seq_lens_before, Hkv, window, win_rows, k_win,
                                             v_win, status);
  else
    k_ring_gather<512><<<grid, 256, 0, st>>>(k_cache, v_cache, seq_lens_before, Hkv, window, win_rows, k_win,
                                             v_win, status);
  return cudaGetLastError();
}

cudaError_t launch_gather_q8(const uint8_t* k_codes, const float2* k_params, const uint8_t* v_codes,
                             const float2* v_params, const int32_t* seq_lens_before, int extra, int B, int Hkv,
                             int D, int window, int cache_cap, const int32_t* page_table, int page_size,
                             int pages_per_seq, int n_pages, int win_rows, int first_row, bf16* k_win,
                             bf16* v_win, int* status, cudaStream_t st) {
  if (first_row < 0) return cudaErrorInvalidValue;
  const int64_t rows = std::max(win_rows - first_row, 1);  // an upper bound; blocks stride over the rest
  const int64_t blocks = std::min<int64_t>((rows * Hkv + 7) / 8, 1184);
  dim3 grid((unsigned)std::max<int64_t>(blocks, 1), B);
  if (D == 256)
    k_gather_q8<256><<<grid, 256, 0, st>>>(k_codes, k_params, v_codes, v_params, seq_lens_before, extra, Hkv,
                                           window, cache_cap, page_table, page_size, pages_per_seq, n_pages,
                                           win_rows, first_row, k_win, v_win, status);
  else
    k_gather_q8<512><<<grid, 256, 0, st>>>(k_codes, k_params, v_codes, v_params, seq_lens_before, extra, Hkv,
                                           window, cache_cap, page_table, page_size, pages_per_seq, n_pages,
                                           win_rows, first_row, k_win, v_win, status);
  return cudaGetLastError();
}

// lens_before[b] = seq_lens[b] - tokens: the cached length before a
// multi-token step, for the chunked-prefill route of such a step.
__global__ void k_lens_minus(const int32_t* __restrict__ seq_lens, int32_t* __restrict__ lens_before, int B,
                             int tokens) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) lens_before[b] = seq_lens[b] - tokens;
}

cudaError_t launch_lens_minus(const int32_t* seq_lens, int32_t* lens_before, int B, int tokens, cudaStream_t st) {
  k_lens_minus<<<(B + 127) / 128, 128, 0, st>>>(seq_lens, lens_before, B, tokens);
  return cudaGetLastError();
}

cudaError_t launch_decode_rope_append(const DecodeRopeArgs& a, int B, int D, cudaStream_t st) {
  const int tx = D / 8;
  dim3 block(tx, 256 / tx);
  if (a.tokens < 1) return cudaErrorInvalidValue;
  if (D == 256)
    k_decode_rope_append<256><<<B * a.tokens, block, 0, st>>>(a);
  else
    k_decode_rope_append<512><<<B * a.tokens, block, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace hlg
