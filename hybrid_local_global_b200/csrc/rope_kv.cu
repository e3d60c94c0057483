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
// Precision: the angle pos * inv_freq is formed and reduced modulo 2*pi in
// fp64 (an fp32 product has an ulp of 1/64 rad near position 2.6e5), then
// sincosf of the reduced angle; the rotation itself is fp32 and the result
// is rounded to bf16 (round to nearest even).
//
// Thread map: threadIdx.x owns 8 consecutive elements (4 pairs) of the head
// vector, so its inverse frequencies are computed once and each angle once
// per position, then reused for every Q and K head of that position.
#include "common.cuh"
#include "kernels.h"

namespace hlg {

namespace {

constexpr double kTwoPi = 6.283185307179586476925286766559;
constexpr double kInvTwoPi = 0.15915494309189533576888376337251;

struct PairTrig {
  float c[4], s[4];
  bool any_rot;  // false -> the whole 8-element chunk is copied unchanged
};

__device__ __forceinline__ void chunk_inv_freq(int e0, int D, int n_rot, double log2_theta,
                                               double (&inv_freq)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    int i = e0 / 2 + j;
    inv_freq[j] = (i < n_rot) ? exp2(-(2.0 * (double)i / (double)D) * log2_theta) : 0.0;
  }
}

__device__ __forceinline__ PairTrig chunk_trig(int64_t pos, int e0, int n_rot,
                                               const double (&inv_freq)[4]) {
  PairTrig t;
  t.any_rot = (e0 / 2) < n_rot;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (e0 / 2 + j < n_rot) {
      double a = (double)pos * inv_freq[j];
      double r = a - rint(a * kInvTwoPi) * kTwoPi;
      sincosf((float)r, &t.s[j], &t.c[j]);
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

// Prefill: rotate the chunk's Q into q_rot (times q_scale), rotate K and write it (global:
// cache slot pos; local: k_rot workspace for the attention kernel, plus the
// ring slot for the last `window` positions), copy V likewise.
template <int D>
__global__ void __launch_bounds__(256) k_prefill_rope(PrefillRopeArgs a) {
  const int b = blockIdx.y;
  const int e0 = threadIdx.x * 8;
  const int64_t pos0 = a.seq_lens_before ? (int64_t)a.seq_lens_before[b] : 0;
  if (pos0 < 0 || (a.window == 0 && pos0 + a.S > a.cache_cap)) {
    if (threadIdx.x == 0 && threadIdx.y == 0 && blockIdx.x == 0)
      set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  double inv_freq[4];
  chunk_inv_freq(e0, D, a.n_rot, a.log2_theta, inv_freq);
  const int n_heads = a.Hq + (a.k_new ? 2 * a.Hkv : 0);
  const int s_begin = blockIdx.x * a.rows_per_cta;
  const int s_end = min(a.S, s_begin + a.rows_per_cta);
  for (int s = s_begin; s < s_end; ++s) {
    const int64_t pos = pos0 + s;
    const PairTrig t = chunk_trig(pos, e0, a.n_rot, inv_freq);
    const int64_t row = (int64_t)b * a.S + s;
    for (int h = threadIdx.y; h < n_heads; h += blockDim.y) {
      if (h < a.Hq) {
        const int64_t off = (row * a.Hq + h) * D + e0;
        st16(a.q_rot + off, rotate_scale_chunk(ld16(a.q + off), t, e0, a.n_rot, a.q_scale));
        continue;
      }
      const bool is_k = h < a.Hq + a.Hkv;
      const int kh = is_k ? h - a.Hq : h - a.Hq - a.Hkv;
      const int64_t src_off = (row * a.Hkv + kh) * D + e0;
      uint4 v = is_k ? rotate_chunk(ld16(a.k_new + src_off), t, e0, a.n_rot)
                     : ld16(a.v_new + src_off);
      bf16* cache = is_k ? a.k_cache : a.v_cache;
      const int64_t head_base = ((int64_t)b * a.Hkv + kh) * a.cache_cap;
      if (a.window == 0) {
        st16(cache + (head_base + pos) * D + e0, v);
      } else {
        if (is_k) st16(a.k_rot + src_off, v);
        if (s >= a.S - a.window) st16(cache + (head_base + pos % a.window) * D + e0, v);
      }
    }
  }
}

// Decode: one token per sequence at position seq_lens[b]-1.
template <int D>
__global__ void __launch_bounds__(256) k_decode_rope_append(DecodeRopeArgs a) {
  const int b = blockIdx.x;
  const int e0 = threadIdx.x * 8;
  const int64_t len = a.seq_lens[b];
  if (len < 1 || len > a.max_len) {
    if (threadIdx.x == 0 && threadIdx.y == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  const int64_t pos = len - 1;
  const int64_t slot = a.window > 0 ? pos % a.window : pos;
  if (slot >= a.cache_cap) {
    if (threadIdx.x == 0 && threadIdx.y == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  double inv_freq[4];
  chunk_inv_freq(e0, D, a.n_rot, a.log2_theta, inv_freq);
  const PairTrig t = chunk_trig(pos, e0, a.n_rot, inv_freq);
  const int n_heads = a.Hq + (a.k_new ? 2 * a.Hkv : 0);
  for (int h = threadIdx.y; h < n_heads; h += blockDim.y) {
    if (h < a.Hq) {
      const int64_t off = ((int64_t)b * a.Hq + h) * D + e0;
      st16(a.q_rot + off, rotate_chunk(ld16(a.q + off), t, e0, a.n_rot));
      continue;
    }
    const bool is_k = h < a.Hq + a.Hkv;
    const int kh = is_k ? h - a.Hq : h - a.Hq - a.Hkv;
    const int64_t src_off = ((int64_t)b * a.Hkv + kh) * D + e0;
    uint4 v = is_k ? rotate_chunk(ld16(a.k_new + src_off), t, e0, a.n_rot)
                   : ld16(a.v_new + src_off);
    bf16* cache = is_k ? a.k_cache : a.v_cache;
    st16(cache + (((int64_t)b * a.Hkv + kh) * a.cache_cap + slot) * D + e0, v);
  }
}

}  // namespace

cudaError_t launch_prefill_rope(const PrefillRopeArgs& a, int B, int D, cudaStream_t st) {
  const int tx = D / 8;
  dim3 block(tx, 256 / tx);
  dim3 grid((a.S + a.rows_per_cta - 1) / a.rows_per_cta, B);
  if (D == 256)
    k_prefill_rope<256><<<grid, block, 0, st>>>(a);
  else
    k_prefill_rope<512><<<grid, block, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode_rope_append(const DecodeRopeArgs& a, int B, int D, cudaStream_t st) {
  const int tx = D / 8;
  dim3 block(tx, 256 / tx);
  if (D == 256)
    k_decode_rope_append<256><<<B, block, 0, st>>>(a);
  else
    k_decode_rope_append<512><<<B, block, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace hlg
