// decode_q8.cu -- batched single-token decode over an int8 KV cache.
//
// The cache holds, per cached row (one token of one KV head), D codes c in
// 0..255 and a pair (min, step); the row's value is min + c * step ("Gemma 4
// Technical Report", Quantization and Efficiency: the quantizer and its
// dequantizer; Table 3 "+KV int8"). Attention is the same split-K
// flash-decode as decode.cu ("Gemma 4: End-to-End Architecture
// Walkthrough", 3a/3b), computed without dequantizing element by element:
//   s_j = <q, min_j + step_j c_j> = step_j <q, c_j> + min_j sum(q)
//   o   = sum_j p_j (min_j + step_j c_j) = sum_j (p_j step_j) c_j + sum_j p_j min_j
// so the MMAs multiply the codes themselves (exact in fp16), and the affine
// part is applied per key (S) and as one scalar per head (O).
//
// Per CTA = (split, KV head, sequence), 128 threads:
//   warp 3      producer: per 16-key sub-block, four bulk copies into a ring
//               slot: the K codes (16 rows x D bytes, contiguous in the
//               cache), the V codes, and their (min, step) rows.
//   warps 0..2  consumers: sub-block t goes to warp t % 3 (and ring slot
//               t % NSLOT). The warp widens its slot's codes to fp16 in its
//               own padded staging rows (a byte permute puts each code in
//               the mantissa of 1024.0, and subtracting 1024 leaves the code
//               exactly), releases the slot, then runs the mma.sync path of
//               decode.cu in fp16: S = Q C_K^T, then O^T += C_V^T P'^T.
// Scaling: Q is staged as fp16 times 2^-eq with max|q| <= 1, and P' = p *
// step_j * 2^-ev with 2^ev >= every step of the CTA's key range (read in a
// pre-pass over the (min, step) rows), so neither leaves fp16's range; both
// powers of two are undone exactly in fp32.
//
// Every barrier wait is bounded (%globaltimer deadline); on a timeout the CTA
// raises its abort flag, records GEMMA_ERR_DEVICE_TIMEOUT, waits (bounded)
// for its own copies in flight, and exits without output.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace hlg {

namespace {

using namespace ms;

constexpr int NCW = 3;  // consumer warps

template <int D>
struct Q8Cfg {
  static constexpr int KB = 16;                      // keys per sub-block
  static constexpr int CODES_B = 2 * KB * D;         // K codes [16][D], then V codes (K = V: 32 K rows)
  static constexpr int RAW_B = CODES_B + 2 * KB * 8; // then K (min, step) [16], V [16] (K = V: 32 K)
  static constexpr int NSLOT = 6;
  static_assert(NSLOT % NCW == 0, "each ring slot needs a single consumer warp");
  static constexpr int ROW = D + 8;                  // fp16 staging row (elements), 16 B pad
  static constexpr int ROWB = ROW * 2;
  static constexpr int STG_B = 2 * KB * ROWB;        // per consumer warp: 32 rows
  static constexpr int RING_B = NSLOT * RAW_B;
  static constexpr int STG_OFF = RING_B;
  static constexpr int Q_OFF = STG_OFF + NCW * STG_B;
  static constexpr int Q_B = 8 * ROWB;
  static constexpr int QSUM_OFF = Q_OFF + Q_B;       // float [8] sum of each head's staged q
  static constexpr int BAR_OFF = QSUM_OFF + 64;
  static constexpr int MISC_OFF = BAR_OFF + 2 * NSLOT * 8;
  static constexpr int SMEM = MISC_OFF + (4 + 2 * NSLOT + 64) * 4;
  static constexpr int OSTR = D + 4;                 // merge-buffer row (floats)
  static constexpr int MERGE_B = NCW * 8 * OSTR * 4;
  static_assert(MERGE_B <= NCW * STG_B, "merge buffer must fit in the staging rows");
  static_assert(RAW_B % 16 == 0 && ROWB % 16 == 0 && STG_OFF % 16 == 0, "16-byte alignment");
  static constexpr int MIN_BLOCKS = (SMEM * 2 <= 227 * 1024) ? 2 : 1;
};

// Two codes (bytes `sel` picks) -> fp16x2 holding them exactly.
__device__ __forceinline__ uint32_t codes_to_h2(uint32_t w, uint32_t sel) {
  uint32_t h = __byte_perm(w, 0x64u, sel);  // bytes c, 0x64, c', 0x64: fp16 1024 + c, 1024 + c'
  __half2 v = *reinterpret_cast<__half2*>(&h);
  v = __hsub2(v, __half2half2(__ushort_as_half((unsigned short)0x6400)));
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 2^e with e the smallest integer such that 2^e >= x (x > 0), as a float;
// 1 for x <= 0.
__device__ __forceinline__ float pow2_ceil(float x) {
  if (!(x > 0.f)) return 1.f;
  int e;
  const float m = frexpf(x, &e);  // x = m * 2^e, m in [0.5, 1)
  return ldexpf(1.f, m == 0.5f ? e - 1 : e);
}

template <int D>
__global__ void __launch_bounds__(32 * (NCW + 1), Q8Cfg<D>::MIN_BLOCKS) k_decode_split_q8(DecodeAttnArgs a) {
  using C = Q8Cfg<D>;
  extern __shared__ __align__(128) unsigned char sm[];
  unsigned char* ring = sm;
  unsigned char* stg_all = sm + C::STG_OFF;
  __half* qs = reinterpret_cast<__half*>(sm + C::Q_OFF);
  float* qsum = reinterpret_cast<float*>(sm + C::QSUM_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::BAR_OFF);
  uint64_t* empty = full + C::NSLOT;
  int* misc = reinterpret_cast<int*>(sm + C::MISC_OFF);
  volatile int* abort_flag = misc;
  int* issued = misc + 1;
  int* consumed = issued + C::NSLOT;
  float* m_w = reinterpret_cast<float*>(consumed + C::NSLOT);  // [NCW][8]
  float* l_w = m_w + 8 * NCW;                                   // [NCW][8]
  float* red = l_w + 8 * NCW;                                   // [8] reduction scratch

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv;
  const int64_t len = a.seq_lens[b];
  if (len < 1 || len > a.max_len) {
    if (threadIdx.x == 0 && split == 0 && g == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
    return;
  }
  const int64_t n_valid = a.window > 0 ? (len < a.window ? len : (int64_t)a.window) : len;
  const int64_t k_begin = (int64_t)split * a.chunk;
  if (k_begin >= n_valid) return;
  const int64_t k_end = (k_begin + a.chunk < n_valid) ? k_begin + a.chunk : n_valid;
  // keys per ring slot: 16 K rows + 16 V rows, or 32 K rows under K = V
  const int kps = a.keqv ? 2 * C::KB : C::KB;
  const int n_sub = (int)((k_end - k_begin + kps - 1) / kps);
  const int64_t row0 = ((int64_t)b * a.Hkv + g) * (int64_t)a.cache_cap;  // first cache row of (b, g)
  const uint8_t* kcode = a.k_codes + row0 * D;
  const uint8_t* vcode = a.v_codes + row0 * D;
  const float2* kpar = a.k_params + row0;
  const float2* vpar = a.keqv ? kpar : a.v_params + row0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      issued[s] = 0;
      consumed[s] = 0;
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // max |q| over the group's heads and the largest V step of this split's
  // keys: both become powers of two that keep the fp16 operands in range
  float qmax = 0.f, vmax = 0.f;
  for (int idx = threadIdx.x; idx < G * (D / 8); idx += blockDim.x) {
    const int r = idx / (D / 8), c = (idx % (D / 8)) * 8;
    const uint4 u = *reinterpret_cast<const uint4*>(a.q_rot + ((int64_t)b * a.Hq + g * G + r) * D + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf16x2(w[j]);
      qmax = fmaxf(qmax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  for (int64_t k = k_begin + threadIdx.x; k < k_end; k += blockDim.x) vmax = fmaxf(vmax, vpar[k].y);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
  if (lane == 0) {
    red[warp] = qmax;
    red[4 + warp] = vmax;
  }
  __syncthreads();
  qmax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  vmax = fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7]));
  const float fq = pow2_ceil(qmax), fv = pow2_ceil(vmax);
  const float inv_fq = 1.f / fq, inv_fv = 1.f / fv;  // exact: powers of two
  for (int idx = threadIdx.x; idx < 8 * (D / 8); idx += blockDim.x) {
    const int r = idx / (D / 8), c = (idx % (D / 8)) * 8;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (r < G) u = *reinterpret_cast<const uint4*>(a.q_rot + ((int64_t)b * a.Hq + g * G + r) * D + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf16x2(w[j]);
      h[j] = pack_h2(f.x * inv_fq, f.y * inv_fq);
    }
    *reinterpret_cast<uint4*>(qs + r * C::ROW + c) = make_uint4(h[0], h[1], h[2], h[3]);
  }
  __syncthreads();
  // sum of each head's staged q (the same fp16 values the MMA reads)
  for (int r = warp; r < 8; r += NCW + 1) {
    float acc = 0.f;
    for (int d = lane; d < D; d += 32) acc += __half2float(qs[r * C::ROW + d]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) qsum[r] = acc;
  }
  __syncwarp();
  __syncthreads();
  const uint64_t deadline = globaltimer_ns() + a.wait_ns;

  if (warp == NCW) {
    // ---------------- producer ----------------
    for (int t = 0; t < n_sub; ++t) {
      const int slot = t % C::NSLOT;
      bool ok = true;
      if (lane == 0) {
        if (t >= C::NSLOT)
          ok = mbar_wait_bounded_at(&empty[slot], ((t / C::NSLOT) - 1) & 1, abort_flag, deadline,
                                    a.status, 1, t, slot, n_sub);
        if (ok && *abort_flag) ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int64_t key0 = k_begin + (int64_t)t * kps;
      const int nk = (int)((k_end - key0) < kps ? (k_end - key0) : kps);
      // (min, step) rows go in pairs (16-byte copies): key0 is a multiple of 16
      // and the cache capacity is even, so the pair of an odd last row exists
      const int np = (nk + 1) & ~1;
      const bool drop = a.drop_first_copy && t == 0 && split == 0 && g == 0 && b == 0;
      if (drop) continue;
      unsigned char* dst = ring + slot * C::RAW_B;
      if (lane == 0) {
        const uint32_t bytes = a.keqv ? (uint32_t)(nk * D + np * 8) : (uint32_t)(2 * (nk * D + np * 8));
        mbar_arrive_expect_tx(&full[slot], bytes);
        issued[slot] += 1;
      }
      __syncwarp();
      if (lane == 0) bulk_g2s(dst, kcode + key0 * D, (uint32_t)(nk * D), &full[slot]);
      if (lane == 1) bulk_g2s(dst + C::CODES_B, kpar + key0, (uint32_t)(np * 8), &full[slot]);
      if (!a.keqv) {
        if (lane == 2) bulk_g2s(dst + C::KB * D, vcode + key0 * D, (uint32_t)(nk * D), &full[slot]);
        if (lane == 3) bulk_g2s(dst + C::CODES_B + C::KB * 8, vpar + key0, (uint32_t)(np * 8), &full[slot]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int gq = lane >> 2, tg = lane & 3;
    unsigned char* stg = stg_all + warp * C::STG_B;  // rows 0..15 K, 16..31 V (K = V: 32 K rows)
    float o[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
    float m_h = -INFINITY, l_t = 0.f, corr = 0.f;  // corr: sum of p * min of V over this lane's keys
    const float qsum_h = qsum[gq] * fq;           // sum of head gq's q
    const float sl_fq = a.scale_log2 * fq;
    const uint32_t q_addr = smem_u32(qs) + ((lane & 7) * C::ROW + ((lane >> 3) & 1) * 8) * 2;
    const uint32_t frag_off = (((lane >> 4) * 8 + (lane & 7)) * C::ROW + ((lane >> 3) & 1) * 8) * 2;

    for (int t = warp; t < n_sub; t += NCW) {
      const int slot = t % C::NSLOT;
      const bool ok = mbar_wait_bounded_at(&full[slot], (t / C::NSLOT) & 1, abort_flag, deadline,
                                           a.status, 2, t, slot, warp);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int64_t key0_slot = k_begin + (int64_t)t * kps;
      const int nk_slot = (int)((k_end - key0_slot) < kps ? (k_end - key0_slot) : kps);
      const unsigned char* raw = ring + slot * C::RAW_B;
      // widen the codes to fp16 staging rows; rows past the end become zeros
      constexpr int CPR = D / 16;  // 16-code chunks per row
      for (int idx = lane; idx < 2 * C::KB * CPR; idx += 32) {
        const int r = idx / CPR, c = idx % CPR;
        const int key = a.keqv ? r : (r & (C::KB - 1));
        uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = make_uint4(0, 0, 0, 0);
        if (key < nk_slot) {
          const uint4 u = *reinterpret_cast<const uint4*>(raw + r * D + c * 16);
          lo4 = make_uint4(codes_to_h2(u.x, 0x4140), codes_to_h2(u.x, 0x4342), codes_to_h2(u.y, 0x4140),
                           codes_to_h2(u.y, 0x4342));
          hi4 = make_uint4(codes_to_h2(u.z, 0x4140), codes_to_h2(u.z, 0x4342), codes_to_h2(u.w, 0x4140),
                           codes_to_h2(u.w, 0x4342));
        }
        uint4* d = reinterpret_cast<uint4*>(stg + r * C::ROWB + c * 32);
        d[0] = lo4;
        d[1] = hi4;
      }
      // this lane's keys of each 16-key half: 2tg, 2tg+1, 8+2tg, 9+2tg
      const float2* praw = reinterpret_cast<const float2*>(raw + C::CODES_B);  // K [16] then V [16] (K = V: 32 K)
      float2 kp[2][4], vp[2][4];
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = (i < 2 ? 2 * tg + i : 8 + 2 * tg + (i - 2));
          const int kk = half * C::KB + j;
          const bool have = a.keqv ? kk < nk_slot : (half == 0 && j < nk_slot);
          kp[half][i] = have ? praw[kk] : make_float2(0.f, 0.f);
          vp[half][i] = have ? (a.keqv ? kp[half][i] : praw[C::KB + j]) : make_float2(0.f, 0.f);
        }
      // the codes and rows are in registers and staging: the slot can refill
      __syncwarp();
      if (lane == 0) {
        consumed[slot] += 1;
        mbar_arrive(&empty[slot]);
      }
      for (int half = 0; half < (a.keqv ? 2 : 1); ++half) {
        const int nk = nk_slot - half * C::KB;
        if (nk <= 0) break;
        unsigned char* kst = stg + half * C::KB * C::ROWB;
        unsigned char* vst = a.keqv ? kst : stg + C::KB * C::ROWB;
        // raw S = Q' C^T (Q' = q / fq): rows = query heads (8 real of 16), cols = 16 keys
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t k_addr = smem_u32(kst) + frag_off;
#pragma unroll 8
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t qa0, qa2, b0, b1, b2, b3;
          ldsm_x2(q_addr + ks * 32, qa0, qa2);
          ldsm_x4(k_addr + ks * 32, b0, b1, b2, b3);
          mma_f16(s0, qa0, 0u, qa2, 0u, b0, b1);
          mma_f16(s1, qa0, 0u, qa2, 0u, b2, b3);
        }
        // s_j = step_j <q, c_j> + min_j sum(q), in log2 units
        const float raw_s[4] = {s0[0], s0[1], s1[0], s1[1]};
        float sv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = (i < 2 ? 2 * tg + i : 8 + 2 * tg + (i - 2));
          sv[i] = (j < nk) ? (kp[half][i].y * raw_s[i] * sl_fq + kp[half][i].x * qsum_h * a.scale_log2)
                           : -INFINITY;
        }
        float tmax = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const float m_new = fmaxf(m_h, tmax);
        const float base = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = exp2f(m_h - base);
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = exp2f(sv[i] - base);
        l_t = l_t * alpha + (p[0] + p[1]) + (p[2] + p[3]);
        corr = corr * alpha + ((p[0] * vp[half][0].x + p[1] * vp[half][1].x) +
                               (p[2] * vp[half][2].x + p[3] * vp[half][3].x));
        m_h = m_new;
        const float al0 = __shfl_sync(0xffffffffu, alpha, (2 * tg) * 4);
        const float al1 = __shfl_sync(0xffffffffu, alpha, (2 * tg + 1) * 4);
        if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            o[mt][0] *= al0;
            o[mt][1] *= al1;
            o[mt][2] *= al0;
            o[mt][3] *= al1;
          }
        }
        // P' = p * step_j / fv: the codes' weights, within fp16's range
        const uint32_t pb0 = pack_h2(p[0] * (vp[half][0].y * inv_fv), p[1] * (vp[half][1].y * inv_fv));
        const uint32_t pb1 = pack_h2(p[2] * (vp[half][2].y * inv_fv), p[3] * (vp[half][3].y * inv_fv));
        // O'^T += C_V^T P'^T : rows = head dims, cols = query heads, k = 16 keys
        const uint32_t v_addr = smem_u32(vst) + frag_off;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          uint32_t va0, va1, va2, va3;
          ldsm_x4_t(v_addr + mt * 32, va0, va1, va2, va3);
          mma_f16(o[mt], va0, va1, va2, va3, pb0, pb1);
        }
      }  // half
      __syncwarp();  // the staging rows are rewritten by this warp's next slot
    }
    // per head: the sum over the 4 lanes holding its keys
    float l_q = l_t + __shfl_xor_sync(0xffffffffu, l_t, 1);
    l_q += __shfl_xor_sync(0xffffffffu, l_q, 2);
    float corr_h = corr + __shfl_xor_sync(0xffffffffu, corr, 1);
    corr_h += __shfl_xor_sync(0xffffffffu, corr_h, 2);
    const float c0 = __shfl_sync(0xffffffffu, corr_h, (2 * tg) * 4);      // head 2tg
    const float c1 = __shfl_sync(0xffffffffu, corr_h, (2 * tg + 1) * 4);  // head 2tg + 1
    if (tg == 0) {
      m_w[warp * 8 + gq] = m_h;
      l_w[warp * 8 + gq] = l_q;
    }
    __syncwarp();
    __syncthreads();  // (A) pairs with the producer's (A)
    if (*abort_flag) return;
    // this warp's O = fv * O' + corr, scaled into the merge buffer (over the staging rows)
    float* obuf = reinterpret_cast<float*>(stg_all);
    float f[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int hh = 2 * tg + j;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, m_w[w * 8 + hh]);
      const float mw = m_w[warp * 8 + hh];
      f[j] = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      float* row0 = obuf + (warp * 8 + 2 * tg) * C::OSTR + mt * 16 + gq;
      float* row1 = row0 + C::OSTR;
      row0[0] = (o[mt][0] * fv + c0) * f[0];
      row1[0] = (o[mt][1] * fv + c1) * f[1];
      row0[8] = (o[mt][2] * fv + c0) * f[0];
      row1[8] = (o[mt][3] * fv + c1) * f[1];
    }
    __syncwarp();
    named_bar_sync(1, 32 * NCW);
    for (int idx = threadIdx.x; idx < G * D; idx += 32 * NCW) {
      const int hh = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, m_w[w * 8 + hh]);
      float L = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = m_w[w * 8 + hh];
        L += (mw == -INFINITY) ? 0.f : l_w[w * 8 + hh] * exp2f(mw - M);
        acc += obuf[(w * 8 + hh) * C::OSTR + d];
      }
      const int64_t pr = ((int64_t)b * a.Hq + g * G + hh) * a.n_splits + split;
      a.part_o[pr * D + d] = acc / L;
      if (d == 0) a.part_lse[pr] = M + log2f(L);
    }
    return;
  }
  // producer reaches here
  __syncwarp();
  __syncthreads();  // (A)
  if (*abort_flag && lane == 0) {
    // drain: wait (bounded) for copies that were issued but never consumed
    const uint64_t dl = globaltimer_ns() + 200000000ull;
    volatile int dummy = 0;
    for (int s = 0; s < C::NSLOT; ++s)
      if (issued[s] > consumed[s])
        mbar_wait_bounded_at(&full[s], (issued[s] - 1) & 1, &dummy, dl, a.status, 3, issued[s], s,
                             consumed[s]);
  }
}

template <int D>
cudaError_t launch_q8(const DecodeAttnArgs& a, int B, cudaStream_t st) {
  using C = Q8Cfg<D>;
  cudaError_t e = cudaFuncSetAttribute(k_decode_split_q8<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  k_decode_split_q8<D><<<dim3(a.n_splits, a.Hkv, B), 32 * (NCW + 1), C::SMEM, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_split_q8(const DecodeAttnArgs& a, int B, int D, cudaStream_t st) {
  return D == 256 ? launch_q8<256>(a, B, st) : launch_q8<512>(a, B, st);
}

}  // namespace hlg
