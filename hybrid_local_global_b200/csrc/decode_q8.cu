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
// Per CTA = (split, KV head, sequence), 128 threads; four CTAs per SM at
// head_dim 256 (measured on the 31B-shaped local layer, B64, ring 1024:
// 154 us with two CTAs of a 12-slot ring, 132 with three, 126 with four of
// a 6-slot ring: the short local splits are latency-bound, so more resident
// warps pay), two at head_dim 512, whose O accumulators need the registers:
//   warp 3      producer: per 16-key sub-block, the K and the V code rows
//               arrive as TMA tiles of 16 rows x 128 bytes (one per 128-byte
//               column chunk), 128-byte swizzled, plus one bulk copy each of
//               the K and V (min, step) rows: 6 copies (head_dim 256) or 10
//               (head_dim 512) per 16 keys. The copy engine takes about one
//               copy per 44 cycles per SM, so copies of one or two rows
//               would bound the stream well below HBM.
//   warps 0..2  consumers: sub-block t goes to warp t % 3 (and ring slot
//               t % NSLOT). The MMA fragments (mma.sync m16n8k16, fp16) come
//               straight from the code rows: a byte permute puts a code in
//               the mantissa of fp16 1024.0 and subtracting 1024 leaves it
//               exactly. The k positions of S and the output rows of P.V
//               stand for dims in an order that makes each lane's codes 16
//               contiguous bytes, and a fixed key order (key_at) puts the
//               rows a quarter warp reads on swizzle phases that land its
//               eight 16-byte reads on disjoint banks.
// Every barrier wait is bounded (%globaltimer deadline); on a timeout the CTA
// raises its abort flag, records GEMMA_ERR_DEVICE_TIMEOUT, waits (bounded)
// for its own copies in flight, and exits without output.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"
#include "tc.cuh"
#include "tmap.h"

namespace hlg {

namespace {

using namespace ms;

constexpr int NCW = 3;  // consumer warps

template <int D>
struct Q8Cfg {
  static constexpr int KB = 16;                      // keys per sub-block
  static constexpr int NCH = D / 128;                // 128-byte column chunks of a code row
  static constexpr int BOX_B = KB * 128;             // one TMA tile: 16 rows x 128 bytes
  static constexpr int REGION_B = NCH * BOX_B;       // 16 code rows, chunk-major, swizzled
  static constexpr int SLOT_B = 2 * REGION_B;        // K region, V region (K = V: 32 K rows)
  static constexpr int NSLOT = 6;
  static_assert(NSLOT % NCW == 0, "each ring slot needs a single consumer warp");
  static constexpr int RING_B = NSLOT * SLOT_B;
  static constexpr int PAR_B = 2 * KB * 8;           // K (min, step) [16], V [16] (K = V: 32 K)
  static constexpr int PAR_OFF = RING_B;
  static constexpr int ROW = D + 8;                  // fp16 Q row (elements), 16 B pad
  static constexpr int Q_OFF = PAR_OFF + NSLOT * PAR_B;
  static constexpr int Q_B = 8 * ROW * 2;
  static constexpr int QSUM_OFF = Q_OFF + Q_B;       // float [8] sum of each head's staged q
  static constexpr int BAR_OFF = QSUM_OFF + 64;
  static constexpr int MISC_OFF = BAR_OFF + 2 * NSLOT * 8;
  static constexpr int ALIGN_B = 1024;               // 128-byte swizzle: tiles on 1024-byte boundaries
  static constexpr int SMEM = ALIGN_B + MISC_OFF + (4 + 2 * NSLOT + 64) * 4;
  static constexpr int OSTR = D + 4;                 // merge-buffer row (floats)
  static constexpr int MERGE_B = NCW * 8 * OSTR * 4;
  static_assert(MERGE_B <= RING_B, "merge buffer must fit in the drained ring");
  static_assert(BOX_B % 1024 == 0 && SLOT_B % 1024 == 0 && Q_OFF % 16 == 0, "alignment");
  static constexpr int CTAS_PER_SM = D == 256 ? 4 : 2;  // see the launch bounds
  static_assert(CTAS_PER_SM * (SMEM + 1024) <= 228 * 1024, "resident CTAs per SM");
  static constexpr int VCH = D / 128;                // 16-byte units of V codes per lane and key row
  static constexpr int PPL = 4 / VCH;                // lane pairs per 128-byte line (P.V reads)
};

// The key (0..15 within a 16-key half) that MMA column / P.V index j stands
// for: j = 8a + 2t + e holds row t + 4e + 8a. The S fragments read rows
// key_at(2i) and key_at(2i + 1) with the 8 lanes of a quarter warp, whose
// swizzle phases (row mod 8) then differ in bit 2; the P.V fragments read
// rows key_at(2t + s), t = 0..3, whose phases differ mod 4. With the
// 16-byte units each lane reads (code_unit, pv_off) every quarter warp
// touches eight distinct units of a 128-byte line: no bank conflicts.
__device__ __forceinline__ int key_at(int j) { return ((j >> 1) & 3) | ((j & 1) << 2) | (j & 8); }

// Byte address, within a region, of the 16-byte unit `u` (0..7) of 128-byte
// chunk `ch` of code row `r`: TMA's 128-byte swizzle XORs the unit with the
// row's line index mod 8 (each tile is 16 lines of 128 bytes).
__device__ __forceinline__ int code_unit(int ch, int r, int u) {
  return ch * (16 * 128) + r * 128 + ((u ^ (r & 7)) << 4);
}

// Dim (= byte offset in a code row) of the first of the 16 codes lane group
// gq reads for P.V unit c (0..VCH-1). Lanes 2p and 2p + 1 take units u and
// u ^ 4 of one 128-byte line; every dim is covered once.
template <int D>
__host__ __device__ __forceinline__ int pv_off(int gq, int c) {
  using C = Q8Cfg<D>;
  const int p = gq >> 1, h = gq & 1;
  return (p / C::PPL) * 128 + 16 * (4 * h + C::VCH * (p % C::PPL) + c);
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

// PAGED: the cache is a pool named by a.page_table (see cache_row); the
// contiguous instance keeps the plain row arithmetic of one (b, g) range.
template <int D, bool PAGED>
__global__ void __launch_bounds__(32 * (NCW + 1), Q8Cfg<D>::CTAS_PER_SM)
    k_decode_split_q8(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      DecodeAttnArgs a) {
  using C = Q8Cfg<D>;
  extern __shared__ __align__(128) unsigned char sm_raw[];
  const uint32_t raw_u32 = smem_u32(sm_raw);
  unsigned char* sm = sm_raw + (((raw_u32 + C::ALIGN_B - 1) & ~uint32_t(C::ALIGN_B - 1)) - raw_u32);
  unsigned char* ring = sm;
  unsigned char* pring = sm + C::PAR_OFF;
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
  // (min, step) rows, addressed like the codes: from the first row of (b, g)
  // in a contiguous cache, through cache_row in a pool
  const int64_t row0 = PAGED ? 0 : ((int64_t)b * a.Hkv + g) * (int64_t)a.cache_cap;
  const float2* kpar = a.k_params + row0;
  const float2* vpar = (a.keqv ? a.k_params : a.v_params) + row0;

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
    if (lane == 0) {
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      for (int t = 0; t < n_sub; ++t) {
        const int slot = t % C::NSLOT;
        if (t >= C::NSLOT &&
            !mbar_wait_bounded_at(&empty[slot], ((t / C::NSLOT) - 1) & 1, abort_flag, deadline, a.status, 1, t,
                                  slot, n_sub))
          break;
        if (*abort_flag) break;
        const int64_t key0 = k_begin + (int64_t)t * kps;
        const int nk = (int)((k_end - key0) < kps ? (k_end - key0) : kps);
        // (min, step) rows go in pairs (16-byte copies): key0 is a multiple of 16
        // and the cache capacity is even, so the pair of an odd last row exists
        const int np = (nk + 1) & ~1;
        const bool drop = a.drop_first_copy && t == 0 && split == 0 && g == 0 && b == 0;
        if (drop) continue;
        // the slot's page and first row in it (a slot never straddles a page:
        // pages hold a multiple of 128 rows, slots start at multiples of 16/32)
        int pg = b;
        int prow = (int)key0;
        int64_t par0 = key0;  // (min, step) row of key0, from kpar / vpar
        if constexpr (PAGED) {
          const int pi = (int)key0 / a.page_size;
          pg = a.page_table[(int64_t)b * a.pages_per_seq + pi];
          prow = (int)key0 - pi * a.page_size;
          if (pg < 0 || pg >= a.n_pages) {  // a page outside the pool: report it, read page 0
            set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
            pg = 0;
          }
          par0 = ((int64_t)pg * a.Hkv + g) * a.page_size + prow;
        }
        // regions that hold rows: K and V, or (K = V) the first 16 K rows and,
        // when there are more, the next 16
        const int n_reg = a.keqv ? (nk > C::KB ? 2 : 1) : 2;
        const uint32_t bytes = (uint32_t)(n_reg * C::REGION_B) + (uint32_t)((a.keqv ? 1 : 2) * np * 8);
        mbar_arrive_expect_tx(&full[slot], bytes);
        issued[slot] += 1;
        const uint32_t dst = smem_u32(ring + slot * C::SLOT_B);
        const uint32_t bar = smem_u32(&full[slot]);
        for (int r = 0; r < n_reg; ++r) {
          const CUtensorMap* m = (a.keqv || r == 0) ? &tm_k : &tm_v;
          const int y = prow + (a.keqv ? r * C::KB : 0);  // rows past the page read as 0
#pragma unroll
          for (int ch = 0; ch < C::NCH; ++ch)
            tc::tma_load_4d(dst + r * C::REGION_B + ch * C::BOX_B, m, ch * 128, y, g, pg, bar);
        }
        unsigned char* pdst = pring + slot * C::PAR_B;
        bulk_g2s(pdst, kpar + par0, (uint32_t)(np * 8), &full[slot]);
        if (!a.keqv) bulk_g2s(pdst + C::KB * 8, vpar + par0, (uint32_t)(np * 8), &full[slot]);
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
    for (int64_t k = k_begin + threadIdx.x; k < k_end; k += 32 * NCW) {
      if constexpr (PAGED) {
        const int64_t r = cache_row(a.page_table, a.pages_per_seq, a.page_size, a.n_pages, a.Hkv, b, g, k);
        if (r >= 0) vmax = fmaxf(vmax, vpar[r].y);  // (a page outside the pool: the producer reports it)
      } else {
        vmax = fmaxf(vmax, vpar[k].y);
      }
    }
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
    // S rows (n-tile 0: key_at(gq), n-tile 1: key_at(8 + gq)): 64-dim group
    // 2 ch + hb of a row is units 4 hb + tg of chunk ch
    const int ra = key_at(gq), rb = key_at(8 + gq);
    const int ka_lo = code_unit(0, ra, tg), ka_hi = code_unit(0, ra, 4 + tg);
    const int kb_lo = code_unit(0, rb, tg), kb_hi = code_unit(0, rb, 4 + tg);
    // P.V rows key_l[i]: units pv_off(gq, c) of each
    const int pv0 = pv_off<D>(gq, 0);
    int vrow[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) vrow[i] = (pv0 >> 7) * C::BOX_B + key_l[i] * 128;
    const int pv_u = (pv0 >> 4) & 7;  // unit of c = 0; unit c is pv_u + c

    for (int t = warp; t < n_sub; t += NCW) {
      const int slot = t % C::NSLOT;
      const bool ok = mbar_wait_bounded_at(&full[slot], (t / C::NSLOT) & 1, abort_flag, deadline,
                                           a.status, 2, t, slot, warp);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int64_t key0_slot = k_begin + (int64_t)t * kps;
      const int nk_slot = (int)((k_end - key0_slot) < kps ? (k_end - key0_slot) : kps);
      const unsigned char* raw = ring + slot * C::SLOT_B;
      const float2* praw = reinterpret_cast<const float2*>(pring + slot * C::PAR_B);  // K [16], V [16] (K = V: 32 K)
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
          const unsigned char* kch = kreg + (grp >> 1) * C::BOX_B;
          const uint4 ka = *reinterpret_cast<const uint4*>(kch + ((grp & 1) ? ka_hi : ka_lo));
          const uint4 kb = *reinterpret_cast<const uint4*>(kch + ((grp & 1) ? kb_hi : kb_lo));
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
          const uint4 r0 = *reinterpret_cast<const uint4*>(vreg + vrow[0] + (((pv_u + c) ^ (key_l[0] & 7)) << 4));
          const uint4 r1 = *reinterpret_cast<const uint4*>(vreg + vrow[1] + (((pv_u + c) ^ (key_l[1] & 7)) << 4));
          const uint4 r2 = *reinterpret_cast<const uint4*>(vreg + vrow[2] + (((pv_u + c) ^ (key_l[2] & 7)) << 4));
          const uint4 r3 = *reinterpret_cast<const uint4*>(vreg + vrow[3] + (((pv_u + c) ^ (key_l[3] & 7)) << 4));
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
      const int dim = pv_off<D>(gq, mt / 8) + 2 * (mt % 8);  // row gq of m-tile mt; row gq+8 is dim+1
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
  // codes [pages][Hkv][page_size][D] bytes (a contiguous cache: B pages of
  // its capacity) as 4-D maps (dims innermost first), tiles of 128 bytes x
  // 16 rows
  CUtensorMap mk, mv;
  const uint64_t ps = (uint64_t)a.page_size;
  const uint64_t dims[4] = {(uint64_t)D, ps, (uint64_t)a.Hkv, (uint64_t)a.n_pages};
  const uint64_t str[3] = {(uint64_t)D, ps * D, (uint64_t)a.Hkv * ps * D};
  const uint32_t box[4] = {128, (uint32_t)C::KB, 1, 1};
  if (!make_map_u8_4d(&mk, a.k_codes, dims, str, box)) return cudaErrorInvalidValue;
  if (a.keqv)
    mv = mk;
  else if (!make_map_u8_4d(&mv, a.v_codes, dims, str, box))
    return cudaErrorInvalidValue;
  auto kern = a.page_table ? k_decode_split_q8<D, true> : k_decode_split_q8<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.n_splits, a.Hkv, B), 32 * (NCW + 1), C::SMEM, st>>>(mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_split_q8(const DecodeAttnArgs& a, int B, int D, cudaStream_t st) {
  return D == 256 ? launch_q8<256>(a, B, st) : launch_q8<512>(a, B, st);
}

}  // namespace hlg
