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
// so the MMAs multiply the codes themselves (exact in fp16, offset by 1024),
// and the affine part and the offset are applied per key (S) and as one
// scalar per head (O).
//
// Per CTA = (split, KV head, sequence), 128 threads, two CTAs per SM:
//   warp 3      producer: per 16-key sub-block, one bulk copy per pair of
//               consecutive K (or V) code rows (contiguous in the cache) into
//               padded row pairs of a ring slot, plus one copy each of the K
//               and V (min, step) rows.
//   warps 0..2  consumers: sub-block t goes to warp t % 3 (and ring slot
//               t % NSLOT). The MMA fragments (mma.sync m16n8k16, fp16) come
//               straight from the code rows: a byte permute puts a code in
//               the mantissa of fp16 1024.0 and subtracting 1024 leaves it
//               exactly. The k positions of S and the output rows of P.V
//               stand for dims in an order that makes each lane's codes 16
//               contiguous bytes, and a fixed key order (key_at) spreads the
//               rows a quarter warp reads over different banks.
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
  static constexpr int PAIRB = 2 * D + 16;           // two consecutive code rows + 16 B pad
  static constexpr int REGION_B = (KB / 2) * PAIRB;  // 16 code rows as 8 padded pairs
  static constexpr int PAR_OFF = 2 * REGION_B;       // K region, V region (K = V: 32 K rows), then
  static constexpr int RAW_B = PAR_OFF + 2 * KB * 8; // K (min, step) [16], V [16] (K = V: 32 K)
  static constexpr int NSLOT = 6;
  static_assert(NSLOT % NCW == 0, "each ring slot needs a single consumer warp");
  static constexpr int ROW = D + 8;                  // fp16 Q row (elements), 16 B pad
  static constexpr int RING_B = NSLOT * RAW_B;
  static constexpr int Q_OFF = RING_B;
  static constexpr int Q_B = 8 * ROW * 2;
  static constexpr int QSUM_OFF = Q_OFF + Q_B;       // float [8] sum of each head's staged q
  static constexpr int BAR_OFF = QSUM_OFF + 64;
  static constexpr int MISC_OFF = BAR_OFF + 2 * NSLOT * 8;
  static constexpr int SMEM = MISC_OFF + (4 + 2 * NSLOT + 64) * 4;
  static constexpr int OSTR = D + 4;                 // merge-buffer row (floats)
  static constexpr int MERGE_B = NCW * 8 * OSTR * 4;
  static_assert(MERGE_B <= RING_B, "merge buffer must fit in the drained ring");
  static_assert(PAIRB % 16 == 0 && RAW_B % 16 == 0 && Q_OFF % 16 == 0, "16-byte alignment");
  static_assert(2 * SMEM <= 227 * 1024, "two CTAs per SM");
  static constexpr int VCH = D / 128;                // 16-dim chunks of V per lane (D/8 dims per lane)
};

// Byte offset of code row r (0..31) in a slot: rows go in padded pairs.
template <int D>
__device__ __forceinline__ int code_row_off(int r) {
  return (r >> 1) * Q8Cfg<D>::PAIRB + (r & 1) * D;
}

// The key (0..15 within a 16-key half) that MMA column / P.V index j stands
// for. The S fragments read rows key_at(gq) and key_at(8 + gq) with the 8
// lanes of a quarter warp on two of them, the P.V fragments rows key_at(2tg)
// .. key_at(9 + 2tg) with four lanes on four rows; this order puts each such
// set of rows in row pairs whose 16-byte pads shift them onto disjoint banks
// (head_dim 512; head_dim 256 keeps a 2-way overlap on the P.V side).
__device__ __forceinline__ int key_at(int j) {
  const int q = (j & 7) >> 1;
  return (j & 8) ? ((j & 1) ? 9 + 2 * q : 2 * q + 1) : ((j & 1) ? 8 + 2 * q : 2 * q);
}

// Two codes (bytes `sel` picks) -> fp16x2 (1024 + c, 1024 + c'), exactly:
// the code lands in the mantissa of 1024.0. The MMAs take the codes with
// this offset and the 1024 comes off once per key (S) and per head (O).
__device__ __forceinline__ uint32_t codes_h2(uint32_t w, uint32_t sel) { return __byte_perm(w, 0x64u, sel); }

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
__global__ void __launch_bounds__(32 * (NCW + 1), 2) k_decode_split_q8(DecodeAttnArgs a) {
  using C = Q8Cfg<D>;
  extern __shared__ __align__(128) unsigned char sm[];
  unsigned char* ring = sm;
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
  __syncthreads();  // the barriers exist before the producer arms them
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
      // lanes 0..7: K row pairs, 8..15: V row pairs (K = V: lanes 0..15, the
      // 16 pairs of 32 K rows); lanes 16, 17: the (min, step) rows
      if (lane < 16) {
        const bool isv = !a.keqv && lane >= 8;
        const int pr = a.keqv ? lane : (lane & 7);
        const int left = nk - 2 * pr;
        if (left > 0)
          bulk_g2s(dst + (isv ? C::REGION_B : 0) + pr * C::PAIRB, (isv ? vcode : kcode) + (key0 + 2 * pr) * D,
                   (uint32_t)((left >= 2 ? 2 : 1) * D), &full[slot]);
      } else if (lane == 16) {
        bulk_g2s(dst + C::PAR_OFF, kpar + key0, (uint32_t)(np * 8), &full[slot]);
      } else if (lane == 17 && !a.keqv) {
        bulk_g2s(dst + C::PAR_OFF + C::KB * 8, vpar + key0, (uint32_t)(np * 8), &full[slot]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    // Consumer prologue, overlapping the producer's first copies: max |q|
    // over the group's heads and the largest V step of this split's keys
    // become powers of two that keep the fp16 operands in range; then Q
    // (scaled) in fp16 and each head's sum of it.
    float qmax = 0.f, vmax = 0.f;
    for (int idx = threadIdx.x; idx < G * (D / 8); idx += 32 * NCW) {
      const int r = idx / (D / 8), c = (idx % (D / 8)) * 8;
      const uint4 u = *reinterpret_cast<const uint4*>(a.q_rot + ((int64_t)b * a.Hq + g * G + r) * D + c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = unpack_bf16x2(w[j]);
        qmax = fmaxf(qmax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    for (int64_t k = k_begin + threadIdx.x; k < k_end; k += 32 * NCW) vmax = fmaxf(vmax, vpar[k].y);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (lane == 0) {
      red[warp] = qmax;
      red[4 + warp] = vmax;
    }
    named_bar_sync(1, 32 * NCW);
    qmax = fmaxf(fmaxf(red[0], red[1]), red[2]);
    vmax = fmaxf(fmaxf(red[4], red[5]), red[6]);
    const float fq = pow2_ceil(qmax), fv = pow2_ceil(vmax);
    const float inv_fq = 1.f / fq, inv_fv = 1.f / fv;  // exact: powers of two
    for (int idx = threadIdx.x; idx < 8 * (D / 8); idx += 32 * NCW) {
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
    named_bar_sync(1, 32 * NCW);
    // sum of each head's fp16 q (the values the MMAs read)
    for (int r = warp; r < 8; r += NCW) {
      float acc = 0.f;
      for (int d = lane; d < D; d += 32) acc += __half2float(qs[r * C::ROW + d]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) qsum[r] = acc;
    }
    named_bar_sync(1, 32 * NCW);
    // The MMA fragments come straight from the copied code rows. S: the 16
    // k positions of k-step s of 64-dim group grp stand for dims
    // 64 grp + 16 tg' + 4 s + {0, 1} (k = 2tg', 2tg'+1) and + {2, 3} (k = 8+2tg',
    // 9+2tg'), so a lane's K codes for four k-steps are 16 contiguous bytes,
    // and its Q fragments 16 contiguous fp16. P.V: output row m of m-tile mt
    // is dim (D/8) gq' + 16 (mt / 8) + 2 (mt % 8) (+1 for row m + 8), so a
    // lane's V codes for eight m-tiles are 16 contiguous bytes of each of its
    // four key rows; the merge puts the dims back in order.
    const int gq = lane >> 2, tg = lane & 3;
    float o[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
    // corr: sum of p * min of V over this lane's keys; psum: sum of the fp16
    // weights P' the MMAs used (the codes carry +1024)
    float m_h = -INFINITY, l_t = 0.f, corr = 0.f, psum = 0.f;
    const float qsum_h = qsum[gq] * fq;           // sum of head gq's q
    const float sl_fq = a.scale_log2 * fq;
    const unsigned char* q_row = reinterpret_cast<const unsigned char*>(qs) + (gq * C::ROW + 16 * tg) * 2;
    // this lane's keys: S columns / P.V positions 2tg, 2tg+1, 8+2tg, 9+2tg
    int key_l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) key_l[i] = key_at(i < 2 ? 2 * tg + i : 8 + 2 * tg + (i - 2));
    const int kro_a = code_row_off<D>(key_at(gq)) + 16 * tg;       // S rows: n-tile 0
    const int kro_b = code_row_off<D>(key_at(8 + gq)) + 16 * tg;   // n-tile 1
    int vro[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) vro[i] = code_row_off<D>(key_l[i]) + (D / 8) * gq;

    for (int t = warp; t < n_sub; t += NCW) {
      const int slot = t % C::NSLOT;
      const bool ok = mbar_wait_bounded_at(&full[slot], (t / C::NSLOT) & 1, abort_flag, deadline,
                                           a.status, 2, t, slot, warp);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int64_t key0_slot = k_begin + (int64_t)t * kps;
      const int nk_slot = (int)((k_end - key0_slot) < kps ? (k_end - key0_slot) : kps);
      const unsigned char* raw = ring + slot * C::RAW_B;
      const float2* praw = reinterpret_cast<const float2*>(raw + C::PAR_OFF);  // K [16], V [16] (K = V: 32 K)
      for (int half = 0; half < (a.keqv ? 2 : 1); ++half) {
        const int nk = nk_slot - half * C::KB;
        if (nk <= 0) break;
        const unsigned char* kreg = raw + half * C::REGION_B;
        const unsigned char* vreg = a.keqv ? kreg : raw + C::REGION_B;
        float2 kp[4], vp[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool have = key_l[i] < nk;  // rows past the end hold stale (finite) codes: masked below
          kp[i] = have ? praw[half * C::KB + key_l[i]] : make_float2(0.f, 0.f);
          vp[i] = have ? (a.keqv ? kp[i] : praw[C::KB + key_l[i]]) : make_float2(0.f, 0.f);
        }
        // S' = Q' (1024 + C)^T (Q' = q / fq): rows = query heads (8 real of 16),
        // cols = 16 keys; even and odd k-steps accumulate apart
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        float s2[4] = {0.f, 0.f, 0.f, 0.f}, s3[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
        for (int grp = 0; grp < D / 64; ++grp) {
          const uint4 qa = *reinterpret_cast<const uint4*>(q_row + grp * 128);
          const uint4 qb = *reinterpret_cast<const uint4*>(q_row + grp * 128 + 16);
          const uint4 ka = *reinterpret_cast<const uint4*>(kreg + kro_a + grp * 64);
          const uint4 kb = *reinterpret_cast<const uint4*>(kreg + kro_b + grp * 64);
          const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
          const uint32_t kwa[4] = {ka.x, ka.y, ka.z, ka.w}, kwb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
          for (int st = 0; st < 4; st += 2) {
            mma_f16(s0, qw[2 * st], 0u, qw[2 * st + 1], 0u, codes_h2(kwa[st], 0x4140), codes_h2(kwa[st], 0x4342));
            mma_f16(s1, qw[2 * st], 0u, qw[2 * st + 1], 0u, codes_h2(kwb[st], 0x4140), codes_h2(kwb[st], 0x4342));
            mma_f16(s2, qw[2 * st + 2], 0u, qw[2 * st + 3], 0u, codes_h2(kwa[st + 1], 0x4140),
                    codes_h2(kwa[st + 1], 0x4342));
            mma_f16(s3, qw[2 * st + 2], 0u, qw[2 * st + 3], 0u, codes_h2(kwb[st + 1], 0x4140),
                    codes_h2(kwb[st + 1], 0x4342));
          }
        }
        // s_j = step_j <q, c_j> + min_j sum(q) = step_j fq S'_j + (min_j - 1024 step_j) sum(q),
        // in log2 units
        const float raw_s[4] = {s0[0] + s2[0], s0[1] + s2[1], s1[0] + s3[0], s1[1] + s3[1]};
        float sv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          sv[i] = (key_l[i] < nk) ? (kp[i].y * raw_s[i] * sl_fq + (kp[i].x - 1024.f * kp[i].y) * qsum_h * a.scale_log2)
                                  : -INFINITY;
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
        corr = corr * alpha + ((p[0] * vp[0].x + p[1] * vp[1].x) + (p[2] * vp[2].x + p[3] * vp[3].x));
        psum *= alpha;
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
        const uint32_t pb0 = pack_h2(p[0] * (vp[0].y * inv_fv), p[1] * (vp[1].y * inv_fv));
        const uint32_t pb1 = pack_h2(p[2] * (vp[2].y * inv_fv), p[3] * (vp[3].y * inv_fv));
        {
          const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&pb0));
          const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&pb1));
          psum += (f0.x + f0.y) + (f1.x + f1.y);
        }
        // O'^T += C_V^T P'^T : rows = head dims, cols = query heads, k = 16 keys
#pragma unroll
        for (int c = 0; c < C::VCH; ++c) {
          const uint4 r0 = *reinterpret_cast<const uint4*>(vreg + vro[0] + 16 * c);
          const uint4 r1 = *reinterpret_cast<const uint4*>(vreg + vro[1] + 16 * c);
          const uint4 r2 = *reinterpret_cast<const uint4*>(vreg + vro[2] + 16 * c);
          const uint4 r3 = *reinterpret_cast<const uint4*>(vreg + vro[3] + 16 * c);
          const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
          const uint32_t w2[4] = {r2.x, r2.y, r2.z, r2.w}, w3[4] = {r3.x, r3.y, r3.z, r3.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // keys (2tg, 2tg+1) and (8+2tg, 9+2tg) interleaved per dim
            const uint32_t t01 = __byte_perm(w0[i], w1[i], 0x5140), t23 = __byte_perm(w0[i], w1[i], 0x7362);
            const uint32_t u01 = __byte_perm(w2[i], w3[i], 0x5140), u23 = __byte_perm(w2[i], w3[i], 0x7362);
            mma_f16(o[8 * c + 2 * i], codes_h2(t01, 0x4140), codes_h2(t01, 0x4342),
                    codes_h2(u01, 0x4140), codes_h2(u01, 0x4342), pb0, pb1);
            mma_f16(o[8 * c + 2 * i + 1], codes_h2(t23, 0x4140), codes_h2(t23, 0x4342),
                    codes_h2(u23, 0x4140), codes_h2(u23, 0x4342), pb0, pb1);
          }
        }
      }  // half
      // every lane is done with the slot's rows: it can refill
      __syncwarp();
      if (lane == 0) {
        consumed[slot] += 1;
        mbar_arrive(&empty[slot]);
      }
    }
    // per head: the sum over the 4 lanes holding its keys
    float l_q = l_t + __shfl_xor_sync(0xffffffffu, l_t, 1);
    l_q += __shfl_xor_sync(0xffffffffu, l_q, 2);
    // O = fv (O' - 1024 sum P') + sum p min: the offset goes into the per-head term
    float corr_h = corr - 1024.f * fv * psum;
    corr_h += __shfl_xor_sync(0xffffffffu, corr_h, 1);
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
    // this warp's O = fv * O' + corr, scaled into the merge buffer (over the drained ring)
    float* obuf = reinterpret_cast<float*>(ring);
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
      const int dim = (D / 8) * gq + 16 * (mt / 8) + 2 * (mt % 8);  // row gq of m-tile mt; row gq+8 is dim+1
      float* row0 = obuf + (warp * 8 + 2 * tg) * C::OSTR + dim;
      float* row1 = row0 + C::OSTR;
      row0[0] = (o[mt][0] * fv + c0) * f[0];
      row1[0] = (o[mt][1] * fv + c1) * f[1];
      row0[1] = (o[mt][2] * fv + c0) * f[0];
      row1[1] = (o[mt][3] * fv + c1) * f[1];
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
