// decode.cu -- batched single-token decode over the KV cache (split-K
// flash-decode) and the log-sum-exp combine of the splits.
//
// For the new token of sequence b (position len-1) and q head h (KV head
// g = h / G): out = sum_j softmax_j(scale <q~, k~_j>) v_j over the visible
// cached keys: every position on a global layer, the ring's last
// min(len, window) positions on a local layer ("Gemma 4: End-to-End
// Architecture Walkthrough", 3a/3b; "Gemma 4 Deep Dive" talk: the window
// bounds what a local layer has to keep). Softmax order does not matter, so
// ring slots are read in slot order.
//
// The step is HBM-bound: every cached K/V byte is read once per KV head and
// shared by its G query heads. Work unit = (split of `chunk` keys, KV head,
// sequence). Per CTA:
//   warp 3      producer: for each 16-key sub-block, one lane arms the slot's
//               full barrier with the byte count and the lanes issue one bulk
//               copy per group of RPC consecutive K or V rows (contiguous in
//               the cache) into a ring of padded shared-memory row groups
//               (group stride RPC*D*2+16 bytes). The copy engine takes about
//               one bulk copy per 44 cycles per SM (measured on B200), which
//               held one 512-byte row per copy (head_dim 256) to half the HBM
//               rate; 2 KB copies (4 rows at head_dim 256, 2 at 512) lift
//               that. The MMA fragments take the keys of a sub-block in an
//               order (key_of) that spreads each ldmatrix over row groups.
//   warps 0..2  consumers: sub-block t goes to warp t % 3 and ring slot
//               t % NSLOT, with NSLOT a multiple of 3, so every slot has a
//               single consumer that waits its phases strictly in order
//               (two waiters on consecutive phases of one mbarrier would
//               alias under parity waits). S = Q K^T with
//               mma.sync m16n8k16 (A = the G query heads padded to 16 rows,
//               B = K rows), online softmax in fp32 (log2 domain), then
//               O^T += V^T P^T with the S accumulators reused directly as the
//               B fragment of P^T (the GQA group is the MMA's N dimension).
// K = V ("Gemma 4: End-to-End Architecture Walkthrough", 3b): only the K
// rows are copied and the PV product reads them as V, halving the bytes.
// The consumer warps' (m, l, O) merge in shared memory; each split writes its
// normalised partial and its log2-sum-exp, and the combine kernel merges the
// splits of a (sequence, head).
//
// Every barrier wait is bounded (%globaltimer deadline). On a timeout the
// CTA raises its abort flag, records GEMMA_ERR_DEVICE_TIMEOUT, waits (again
// bounded) for its own copies still in flight, and exits without output.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace hlg {

namespace {

using namespace ms;

constexpr int NCW = 3;  // consumer warps

template <int D, int RPC_>
struct DecCfg {
  static constexpr int KB = 16;                 // keys per sub-block
  static constexpr int ROW = D + 8;             // padded smem row of Q (elements)
  static constexpr int ROWB = ROW * 2;          // bytes
  static constexpr int RPC = RPC_;                 // rows per bulk copy
  static constexpr int GROUPB = RPC * D * 2 + 16;  // RPC consecutive K (or V) rows + 16 B pad
  static constexpr int GPR = KB / RPC;             // row groups per 16-row region
  static constexpr int SLOT_B = 2 * GPR * GROUPB;  // K region then V region (two K regions under K = V)
  static constexpr int NSLOT = 3;  // head_dim 256: with four CTAs per SM (see the launch bounds)
  static_assert(NSLOT % NCW == 0, "each ring slot needs a single consumer warp");
  static constexpr int RING_B = NSLOT * SLOT_B;
  static constexpr int Q_B = 8 * ROWB;
  static constexpr int OSTR = D + 4;            // merge-buffer row (floats)
  static constexpr int MERGE_B = NCW * 8 * OSTR * 4;
  static_assert(MERGE_B <= RING_B, "merge buffer must fit in the ring");
  static constexpr int BAR_OFF = RING_B + Q_B;
  static constexpr int MISC_OFF = BAR_OFF + 2 * NSLOT * 8;
  static constexpr int SMEM = MISC_OFF + (1 + 2 * NSLOT + 64) * 4;
};

// byte offset of row r within a run of row groups
template <int D, int RPC>
__device__ __forceinline__ int group_row_off(int r) {
  using C = DecCfg<D, RPC>;
  return (r / C::RPC) * C::GROUPB + (r % C::RPC) * (D * 2);
}

// The key that MMA index n (0..15) of a 16-key sub-block stands for. S and
// P.V only need the same order for the K and V fragments and the mask, so
// the 8 rows each ldmatrix reads are taken from different row groups where
// possible: rows of one group are D*2 bytes apart and share bank groups,
// while consecutive groups are shifted by the 16-byte pad.
template <int RPC>
__device__ __forceinline__ int key_of(int n) {
  constexpr int NG = 16 / RPC;  // row groups per 16 keys
  return (n % NG) * RPC + n / NG;
}

// PAGED: the cache is a pool named by a.page_table (see cache_row); the
// contiguous instance keeps the plain row arithmetic of one (b, g) range.
// Head_dim 256 (local layers) runs four CTAs per SM with a 3-slot ring: the
// short ring splits are latency-bound, and the extra resident warps pay
// (measured on the 31B-shaped B64 block: its five local layers ~10 % faster
// than two CTAs with a 6-slot ring). Head_dim 512 keeps two.
template <int D, int RPC, bool PAGED>
__global__ void __launch_bounds__(32 * (NCW + 1), D == 256 ? 4 : 2) k_decode_split(DecodeAttnArgs a) {
  using C = DecCfg<D, RPC>;
  extern __shared__ __align__(128) unsigned char sm[];
  unsigned char* ring = sm;
  bf16* qs = reinterpret_cast<bf16*>(sm + C::RING_B);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::BAR_OFF);
  uint64_t* empty = full + C::NSLOT;
  int* misc = reinterpret_cast<int*>(sm + C::MISC_OFF);
  volatile int* abort_flag = misc;
  int* issued = misc + 1;
  int* consumed = issued + C::NSLOT;
  float* m_w = reinterpret_cast<float*>(consumed + C::NSLOT);  // [NCW][8]
  float* l_w = m_w + 32;                                         // [NCW][8]

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
  // (the same bytes per slot, so as many bytes stay in flight)
  const int kps = a.keqv ? 2 * C::KB : C::KB;
  const int n_sub = (int)((k_end - k_begin + kps - 1) / kps);
  // a sub-block's rows are contiguous: pages hold a multiple of 32 rows and
  // sub-blocks start at multiples of 16 (32 under K = V)
  const int64_t head_off = PAGED ? 0 : ((int64_t)b * a.Hkv + g) * (int64_t)a.cache_cap * D;

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
  for (int idx = threadIdx.x; idx < 8 * (D / 8); idx += blockDim.x) {
    const int r = idx / (D / 8), c = (idx % (D / 8)) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < G)
      v = *reinterpret_cast<const uint4*>(a.q_rot + ((int64_t)b * a.Hq + g * G + r) * D + c);
    *reinterpret_cast<uint4*>(qs + r * C::ROW + c) = v;
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
      const bool drop = a.drop_first_copy && t == 0 && split == 0 && g == 0 && b == 0;
      if (drop) continue;
      int64_t boff = head_off + key0 * D;  // element offset of the sub-block's first row
      if constexpr (PAGED) {
        int64_t brow = cache_row(a.page_table, a.pages_per_seq, a.page_size, a.n_pages, a.Hkv, b, g, key0);
        if (brow < 0) {  // a page outside the pool: report it and read pool row 0 (finite, wrong)
          if (lane == 0) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
          brow = 0;
        }
        boff = brow * D;
      }
      const bf16* kbase = a.k_cache + boff;
      const bf16* vbase = a.v_cache + boff;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[slot], (uint32_t)((a.keqv ? 1 : 2) * nk * D * 2));
        issued[slot] += 1;
      }
      __syncwarp();
      // lanes 0..GPR-1: K row groups, GPR..2*GPR-1: V row groups (K = V:
      // all 2*GPR lanes copy K rows, which are the values); a short tail
      // group copies only the rows that exist
      if (lane < 2 * C::GPR) {
        const bool isv = !a.keqv && lane >= C::GPR;
        const int grp = a.keqv ? lane : lane % C::GPR;
        const int left = nk - grp * C::RPC;
        if (left > 0)
          bulk_g2s(ring + slot * C::SLOT_B + (isv ? C::GPR * C::GROUPB : 0) + grp * C::GROUPB,
                   (isv ? vbase : kbase) + (int64_t)grp * C::RPC * D,
                   (left >= C::RPC ? C::RPC : left) * D * 2, &full[slot]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int gq = lane >> 2, tg = lane & 3;
    float o[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
    float m_h = -INFINITY, l_t = 0.f;
    const uint32_t q_addr = smem_u32(qs) + ((lane & 7) * C::ROW + ((lane >> 3) & 1) * 8) * 2;
    const uint32_t frag_off = group_row_off<D, RPC>(key_of<RPC>((lane >> 4) * 8 + (lane & 7))) + ((lane >> 3) & 1) * 16;

    for (int t = warp; t < n_sub; t += NCW) {
      const int slot = t % C::NSLOT;
      const bool ok = mbar_wait_bounded_at(&full[slot], (t / C::NSLOT) & 1, abort_flag, deadline,
                                           a.status, 2, t, slot, warp);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int64_t key0_slot = k_begin + (int64_t)t * kps;
      const int nk_slot = (int)((k_end - key0_slot) < kps ? (k_end - key0_slot) : kps);
      if (nk_slot < kps) {
        // rows past the end were not copied: make them finite zeros
        // (slot rows 0..15 are K, 16..31 V; under K = V all 32 are keys,
        // and either way row r sits at group_row_off(r))
        unsigned char* rows = ring + slot * C::SLOT_B;
        for (int idx = lane; idx < 2 * C::KB * (D / 8); idx += 32) {
          const int r = idx / (D / 8), c = (idx % (D / 8)) * 8;
          const int key = a.keqv ? r : (r & (C::KB - 1));
          if (key >= nk_slot) *reinterpret_cast<uint4*>(rows + group_row_off<D, RPC>(r) + c * 2) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      // one 16-key sub-block per slot, or two under K = V
      for (int half = 0; half < (a.keqv ? 2 : 1); ++half) {
      const int nk = nk_slot - half * C::KB;
      if (nk <= 0) break;
      unsigned char* kslot = ring + slot * C::SLOT_B + half * C::GPR * C::GROUPB;
      unsigned char* vslot = a.keqv ? kslot : kslot + C::GPR * C::GROUPB;
      // S = Q K^T : rows = query heads (8 real of 16), cols = 16 keys
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t k_addr = smem_u32(kslot) + frag_off;
#pragma unroll 8
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t qa0, qa2, b0, b1, b2, b3;
        ldsm_x2(q_addr + ks * 32, qa0, qa2);
        ldsm_x4(k_addr + ks * 32, b0, b1, b2, b3);
        mma_bf16(s0, qa0, 0u, qa2, 0u, b0, b1);
        mma_bf16(s1, qa0, 0u, qa2, 0u, b2, b3);
      }
      // online softmax for head gq; this thread holds MMA columns 2tg, 2tg+1,
      // 8+2tg, 9+2tg, i.e. keys key_of() of those
      float sv[4];
      sv[0] = (key_of<RPC>(2 * tg) < nk) ? s0[0] * a.scale_log2 : -INFINITY;
      sv[1] = (key_of<RPC>(2 * tg + 1) < nk) ? s0[1] * a.scale_log2 : -INFINITY;
      sv[2] = (key_of<RPC>(8 + 2 * tg) < nk) ? s1[0] * a.scale_log2 : -INFINITY;
      sv[3] = (key_of<RPC>(9 + 2 * tg) < nk) ? s1[1] * a.scale_log2 : -INFINITY;
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
      const uint32_t pb0 = pack_bf16x2(p[0], p[1]);
      const uint32_t pb1 = pack_bf16x2(p[2], p[3]);
      // O^T += V^T P^T : rows = head dims, cols = query heads, k = 16 keys
      const uint32_t v_addr = smem_u32(vslot) + frag_off;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t va0, va1, va2, va3;
        ldsm_x4_t(v_addr + mt * 32, va0, va1, va2, va3);
        mma_bf16(o[mt], va0, va1, va2, va3, pb0, pb1);
      }
      }  // half
      __syncwarp();
      if (lane == 0) {
        consumed[slot] += 1;
        mbar_arrive(&empty[slot]);
      }
    }
    float l_q = l_t + __shfl_xor_sync(0xffffffffu, l_t, 1);
    l_q += __shfl_xor_sync(0xffffffffu, l_q, 2);
    if (tg == 0) {
      m_w[warp * 8 + gq] = m_h;
      l_w[warp * 8 + gq] = l_q;
    }
    __syncwarp();
    __syncthreads();  // (A) pairs with the producer's (A)
    if (*abort_flag) return;
    // scale this warp's O into the merge buffer (overlays the drained ring)
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
      float* row0 = obuf + (warp * 8 + 2 * tg) * C::OSTR + mt * 16 + gq;
      float* row1 = row0 + C::OSTR;
      row0[0] = o[mt][0] * f[0];
      row1[0] = o[mt][1] * f[1];
      row0[8] = o[mt][2] * f[0];
      row1[8] = o[mt][3] * f[1];
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
        mbar_wait_bounded_at(&full[s], (issued[s] - 1) & 1, &dummy, dl, a.status, 3, issued[s],
                             s, consumed[s]);
  }
}

// Log-sum-exp merge of the splits of one (sequence, query token, q head)
// (decode: one token per sequence): 128 threads =
// 16 dim quads x 8 split lanes per 64 output dims, so the reads of a
// split's partial are coalesced and the splits are summed in parallel. The
// grid's z dimension splits the head dimension when there are few
// (sequence, head) pairs. Split weights 2^(lse_s - M) are formed once per CTA.
template <int D>
__global__ void __launch_bounds__(128) k_decode_combine(DecodeAttnArgs a) {
  extern __shared__ float w_s[];  // [n_splits]
  __shared__ __align__(16) float red[8][64];
  __shared__ float rmax[4], rsum[4];
  // blockIdx.y = b * tokens + t: the row of (sequence b, query token t)
  const int h = blockIdx.x, bt = blockIdx.y, b = bt / a.tokens;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bf16* dst = a.out + ((int64_t)bt * a.Hq + h) * D;
  const int64_t len = a.seq_lens[b];
  if (len < a.tokens || len > a.max_len) {
    for (int d = blockIdx.z * 64 + tid; d < D; d += gridDim.z * 64)
      if (tid < 64) dst[d] = __float2bfloat16(0.f);
    return;
  }
  const int64_t n_valid = a.window > 0 ? (len < a.window ? len : (int64_t)a.window) : len;
  const int n_used = a.every_split ? a.n_splits : (int)((n_valid + a.chunk - 1) / a.chunk);
  const int64_t pr0 = ((int64_t)bt * a.Hq + h) * a.n_splits;
  float m = -INFINITY;
  for (int s = tid; s < n_used; s += 128) m = fmaxf(m, a.part_lse[pr0 + s]);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) rmax[warp] = m;
  __syncthreads();
  const float M = fmaxf(fmaxf(rmax[0], rmax[1]), fmaxf(rmax[2], rmax[3]));
  float sum = 0.f;
  for (int s = tid; s < n_used; s += 128) {
    const float w = exp2f(a.part_lse[pr0 + s] - M);
    w_s[s] = w;
    sum += w;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) rsum[warp] = sum;
  __syncthreads();
  const float inv = 1.f / ((rsum[0] + rsum[1]) + (rsum[2] + rsum[3]));
  const int q = tid & 15, sl = tid >> 4;
  for (int d0 = blockIdx.z * 64; d0 < D; d0 += gridDim.z * 64) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = sl; s < n_used; s += 8) {
      const float w = w_s[s];
      const float4 v = *reinterpret_cast<const float4*>(a.part_o + (pr0 + s) * D + d0 + q * 4);
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
    *reinterpret_cast<float4*>(&red[sl][q * 4]) = acc;
    __syncthreads();
    if (tid < 64) {
      float t = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) t += red[k][tid];
      dst[d0 + tid] = __float2bfloat16(t * inv);
    }
    __syncthreads();  // red is reused by the next 64 dims
  }
}

template <int D, int RPC, bool PAGED>
cudaError_t launch_split_as(const DecodeAttnArgs& a, int B, cudaStream_t st) {
  using C = DecCfg<D, RPC>;
  cudaError_t e = cudaFuncSetAttribute(k_decode_split<D, RPC, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM);
  if (e != cudaSuccess) return e;
  k_decode_split<D, RPC, PAGED><<<dim3(a.n_splits, a.Hkv, B), 32 * (NCW + 1), C::SMEM, st>>>(a);
  return cudaGetLastError();
}

template <int D, int RPC>
cudaError_t launch_split(const DecodeAttnArgs& a, int B, cudaStream_t st) {
  return a.page_table ? launch_split_as<D, RPC, true>(a, B, st) : launch_split_as<D, RPC, false>(a, B, st);
}

}  // namespace

// Rows per bulk copy (measured on B200, with key_of's fragment order):
// head_dim 256 copies groups of 4 rows (2 KB; the local layers of a
// 64-sequence 31B batch: 348 us at one row per copy, 226 at pairs, 185 at 4,
// 205 at 8 rows); head_dim 512 copies pairs (2 KB; that batch's global layer
// 5.20 -> 4.87 ms, 256K tokens with K = V 219 -> 210 us).
cudaError_t launch_decode_split(const DecodeAttnArgs& a, int B, int D, cudaStream_t st) {
  return D == 256 ? launch_split<256, 4>(a, B, st) : launch_split<512, 2>(a, B, st);
}

cudaError_t launch_decode_combine(const DecodeAttnArgs& a, int B, int D, cudaStream_t st) {
  // enough CTAs for about eight per SM, at most one per 64 output dims
  if (a.tokens < 1) return cudaErrorInvalidValue;
  const int pairs = a.Hq * B * a.tokens;
  const int nz = std::max(1, std::min(D / 64, (8 * 148 + pairs - 1) / pairs));
  dim3 grid(a.Hq, B * a.tokens, nz);
  const size_t smem = (size_t)a.n_splits * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;  // > 12288 splits: not planned by decode_plan
  if (D == 256)
    k_decode_combine<256><<<grid, 128, smem, st>>>(a);
  else
    k_decode_combine<512><<<grid, 128, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace hlg
