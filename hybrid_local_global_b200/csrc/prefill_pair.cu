// prefill_pair.cu -- prefill attention on CTA pairs: two 128-row query tiles
// of one (batch, q head) on two SMs that share each tcgen05 MMA
// (cta_group::2, M = 256), head_dim 256 and 512.
//
// Computes, for every query row i of a (batch, q head) and its KV head
// g = h / (Hq/Hkv) ("Gemma 4: End-to-End Architecture Walkthrough", 3a/3b):
//   out_i = sum_j softmax_j(scale <q~_i, k~_j>) v_j   over visible keys j
// where visible means j <= pos_i and, on a local layer, j > pos_i - window.
//
// Why pairs: in a 2-CTA MMA each SM supplies its own 128 rows of A (Q, or P
// from TMEM) and half of the N rows of B, so every K tile (128 keys) and V
// tile (256 output columns) is loaded and read from shared memory once per
// pair instead of once per query tile. A CTA's tile traffic halves
// (64 KB per key tile at head_dim 256, 96 KB at 512) and the TMA ring looks
// twice as far ahead.
//
// Cluster = 2 CTAs (x-adjacent), rank 0 the MMA leader. Per CTA, 192 threads:
//   warp 0     TMA producer (both CTAs): its own Q tile (D/64 boxes of 128
//              rows x 64 dims), then a ring of 32 KB stages in MMA order:
//              K_0, K_1, V_0, K_2, V_1, ... where its half of K_j is 64 keys
//              x D dims (D/256 stages) and its half of V_j is 128 keys x 128
//              output columns (one stage).
//              Both CTAs' loads of a stage complete on the leader's barrier
//              (cta_group::2 loads, no multicast), which expects both halves.
//   warp 1     TMEM owner (both CTAs); in the leader, one lane issues the
//              MMAs: S_j = Q K_j^T (M=256, N=128, K=D) into one of two
//              128-column TMEM buffers, then O += P_{j-1} V_{j-1} (M=256,
//              N=256, K=128) with P read from both CTAs' TMEM; commits arrive
//              on both CTAs' barriers.
//   warps 2-5  softmax (both CTAs), one query row per thread, as in the
//              single-CTA kernel; P_j is released to the leader's barrier.
// TMEM per CTA: O 0..255 (fp32), S/P buffers 256..383 and 384..511.
// head_dim 512 runs two pairs per query-tile pair (256 output columns
// each; the fp32 O tile of 128 x 512 would fill TMEM), each computing S.
//
// V rows past the sequence end must be finite (their P is 0, but 0 * inf is
// nan): on the one key tile that crosses the end, the MMA lane clears those
// rows in both CTAs' stages before the P.V product.
//
// Every wait is bounded by a %globaltimer deadline. On a timeout the CTA
// raises its abort flag and records GEMMA_ERR_DEVICE_TIMEOUT; the leader
// drains its MMAs, both CTAs wait for their own loads, meet at a cluster
// barrier, free TMEM and exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "pair.cuh"
#include "tc.cuh"
#include "tmap.h"

namespace hlg {

namespace {

constexpr int BM = 128, BN = 128, DV = 256;  // rows per CTA, keys per tile, output columns per pair
constexpr int KH = BN / 2;                   // keys of K per CTA
constexpr int VH = DV / 2;                   // V columns per CTA
constexpr int CHUNK_Q = BM * 128;            // Q box: 128 rows x 64 dims (16 KB)
constexpr int CHUNK_K = KH * 128;            // K box: 64 keys x 64 dims (8 KB)
constexpr int CHUNK_V = BN * 128;            // V box: 128 keys x 64 columns (16 KB)
constexpr int STAGE_B = 32768;
constexpr int ALIGN_B = 1024;
constexpr int SMEM_MAX = 232448;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_O = 0, COL_S = 256;
constexpr float RESCALE_LOG2 = 8.0f;
constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(256, BN, 0, 0);
constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(256, DV, 0, 1);
constexpr uint16_t BOTH = 0x3;

template <int NSTAGE>
struct Ctl {
  uint64_t q_full;            // leader: both CTAs' Q tiles landed
  uint64_t full[NSTAGE];      // leader: both CTAs' halves of the stage landed
  uint64_t empty[NSTAGE];     // MMAs done with the stage (both CTAs)
  uint64_t s_full[2];
  uint64_t p_ready;           // leader: 4 local + 4 peer softmax warps
  uint64_t o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int issued[NSTAGE];
  int consumed[NSTAGE];
  int q_issued, q_consumed;
};

template <int D>
struct PairCfg {
  static constexpr int Q_B = BM * D * 2;           // 64 KB / 128 KB
  static constexpr int K_STAGES = D / 256;          // stages per half K tile
  static constexpr int NV = D / DV;                 // pairs per (query-tile pair, head)
  static constexpr int NSTAGE = (SMEM_MAX - ALIGN_B - Q_B - 1024) / STAGE_B;  // 5 / 3
  static constexpr int SMEM = ALIGN_B + Q_B + NSTAGE * STAGE_B + (int)sizeof(Ctl<NSTAGE>);
  static_assert(NSTAGE >= 3 && SMEM <= SMEM_MAX, "shared memory plan");
};

struct PairArgs {
  int S, window, Hq, Hkv;
  int64_t key_cap;
  const int32_t* seq_lens_before;
  bf16* out;
  float* lse;
  int* status;
  unsigned long long wait_ns;
  int kv_token_major;  // K/V map coordinates: 0 = (d, key, head, b), 1 = (d, head, key, b)
  int key_off_window;  // 1: K/V view row = position - (pos0 - window), else = position
  int n_pairs;         // query-tile pairs per (batch, head); with head_pair: query tiles
  // paged cache (head-major views of the pool): view row = position % page_size,
  // view batch = page_table[b * pages_per_seq + position / page_size]; null: contiguous
  const int32_t* page_table;
  int page_size, pages_per_seq, n_pages;
  int head_pair;       // 1: the CTAs take q heads 2p and 2p+1 of one query tile (same KV head)
};

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t deadline, int* status, int where, int a = 0,
                                         int b = 0, int c = 0) {
  bool ok = mbar_wait_bounded_at(bar, parity, abort_flag, deadline, status, where, a, b, c);
  return __all_sync(0xffffffffu, ok);
}

// P = 2^(x - mb) over the 128 logits of one row, packed to bf16 pairs, with
// eight independent partial sums (and, if TRACK, partial maxima).
template <bool TRACK>
__device__ __forceinline__ void exp_row(const uint32_t (&r)[4][32], float mb, uint32_t (&pk)[2][32],
                                        float (&ls)[8], float (&mx)[8]) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    ls[u] = 0.f;
    if (TRACK) mx[u] = -INFINITY;
  }
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float x0 = __uint_as_float(r[i >> 4][(2 * i) & 31]);
    const float x1 = __uint_as_float(r[i >> 4][(2 * i + 1) & 31]);
    if (TRACK) mx[i & 7] = fmaxf(mx[i & 7], fmaxf(x0, x1));
    const float p0 = tc::ex2(x0 - mb), p1 = tc::ex2(x1 - mb);
    ls[i & 7] += p0 + p1;
    pk[i >> 5][i & 31] = pack_bf16x2(p0, p1);
  }
}

__device__ __forceinline__ float max8(const float (&mx)[8]) {
  return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

__device__ __forceinline__ float max_row(const uint32_t (&r)[4][32]) {
  float mx[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int e = 0; e < 32; ++e) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(r[c][e]));
  return max8(mx);
}

// Zero V rows [r0, BN) of a stage: both 64-column boxes, in this CTA (local
// stores) and in the peer (distributed shared memory), then make the writes
// visible to the tensor core's reads.
__device__ __forceinline__ void clear_v_tail_pair(uint32_t stage, int r0) {
  const uint32_t peer = pair::map_to(stage, 1);
  const uint32_t self = pair::map_to(stage, 0);
  for (int r = r0; r < BN; ++r)
    for (int c = 0; c < 2; ++c)
      for (int u = 0; u < 8; ++u) {
        const uint32_t off = (uint32_t)(c * CHUNK_V + r * 128 + u * 16);
        asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(self + off), "r"(0) : "memory");
        asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(peer + off), "r"(0) : "memory");
      }
  asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    k_prefill_pair(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const PairArgs a) {
  using Cfg = PairCfg<D>;
  constexpr int NSTAGE = Cfg::NSTAGE;
  constexpr int Q_B = Cfg::Q_B;
  extern __shared__ unsigned char sm_raw[];
  const uint32_t raw = smem_u32(sm_raw);
  const uint32_t base = (raw + ALIGN_B - 1) & ~uint32_t(ALIGN_B - 1);
  unsigned char* sm = sm_raw + (base - raw);
  const uint32_t sQ = base;
  const uint32_t sStage = base + Q_B;
  Ctl<NSTAGE>* ctl = reinterpret_cast<Ctl<NSTAGE>*>(sm + Q_B + NSTAGE * STAGE_B);
  volatile int* abort_flag = &ctl->abort;

  const uint32_t rank = pair::cta_rank();
  const bool leader = rank == 0;
  const int vh = blockIdx.y % Cfg::NV, b = blockIdx.z;
  const int pq = a.n_pairs - 1 - (int)(blockIdx.x >> 1);  // heaviest pairs first
  // query-tile pairs: rows pq0 .. pq0 + 255 of one head, rank r takes the
  // r-th 128; head pairs: rows pq0 .. pq0 + 127 of heads 2p and 2p + 1
  const int pq0 = a.head_pair ? pq * BM : pq * 2 * BM;      // first row of the pair
  const int span = a.head_pair ? BM : 2 * BM;               // rows the pair covers
  const int q0 = a.head_pair ? pq0 : pq0 + (int)rank * BM;  // first row of this CTA
  const int h = a.head_pair ? 2 * (int)(blockIdx.y / Cfg::NV) + (int)rank : (int)(blockIdx.y / Cfg::NV);
  const int g = h / (a.Hq / a.Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int64_t pos0 = a.seq_lens_before ? (int64_t)a.seq_lens_before[b] : 0;
  const int64_t n_keys = pos0 + a.S;
  // view row of a key = its position - koff (a gathered key window starts at pos0 - window)
  const int64_t koff = a.key_off_window ? pos0 - a.window : 0;
  if (pos0 < 0 || n_keys - koff > a.key_cap) return;  // reported by the RoPE kernel; same for both CTAs
  int64_t lo_first, hi_first, lo_last, hi_last;
  visible_range(pos0 + pq0, a.window, n_keys, &lo_first, &hi_first);
  visible_range(pos0 + min(pq0 + span - 1, a.S - 1), a.window, n_keys, &lo_last, &hi_last);
  const int64_t kt0 = lo_first / BN;
  const int n_tiles = (int)(hi_last / BN - kt0 + 1);

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
      ctl->issued[s] = 0;
      ctl->consumed[s] = 0;
    }
    mbar_init(&ctl->s_full[0], 1);
    mbar_init(&ctl->s_full[1], 1);
    mbar_init(&ctl->p_ready, 8);  // one arrival per softmax warp of either CTA
    mbar_init(&ctl->o_done[0], 1);
    mbar_init(&ctl->o_done[1], 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ctl->q_issued = 0;
    ctl->q_consumed = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    pair::tmem_alloc2(smem_u32(&ctl->tmem_base), TMEM_COLS);
    pair::tmem_relinquish2();
  }
  tc::fence_before_sync();
  __syncwarp();
  pair::cluster_sync();  // both CTAs' barriers exist before any remote arrive or commit
  tc::fence_after_sync();
  const uint32_t tmem = ctl->tmem_base;
  const uint64_t deadline = globaltimer_ns() + a.wait_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      // both CTAs' halves complete on the leader's barriers, which expect both
      const uint32_t q_bar = pair::map_to(smem_u32(&ctl->q_full), 0);
      if (leader) mbar_arrive_expect_tx(&ctl->q_full, 2 * Q_B);
      for (int c = 0; c < D / 64; ++c) pair::tma_load_4d_pair(sQ + c * CHUNK_Q, &tm_q, c * 64, h, q0, b, q_bar);
      ctl->q_issued = 1;
      int item = 0;
      bool ok = true;
      for (int j = 0; j <= n_tiles && ok; ++j) {
        for (int kind = 0; kind < 2 && ok; ++kind) {  // 0: K_j, 1: V_{j-1}
          if ((kind == 0 && j == n_tiles) || (kind == 1 && j == 0)) continue;
          int key0 = (int)((kt0 + j - kind) * BN - koff);  // view row
          int kb = b;                                           // view batch
          if (a.page_table) {
            // tiles never straddle a page (page_size is a multiple of 128); a
            // tile past the sequence's pages holds no visible key: any page
            const int pi = key0 / a.page_size;
            kb = pi < a.pages_per_seq ? a.page_table[(int64_t)b * a.pages_per_seq + pi] : 0;
            if (kb < 0 || kb >= a.n_pages) {
              if ((int64_t)key0 < n_keys) set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
              kb = 0;
            }
            key0 -= pi * a.page_size;
          }
          const int n_st = kind == 0 ? Cfg::K_STAGES : 1;
          for (int hs = 0; hs < n_st; ++hs, ++item) {
            const int s = item % NSTAGE;
            if (item >= NSTAGE &&
                !mbar_wait_bounded_at(&ctl->empty[s], ((item / NSTAGE) - 1) & 1, abort_flag, deadline,
                                      a.status, 31, item, s, j)) {
              ok = false;
              break;
            }
            const uint32_t dst = sStage + s * STAGE_B;
            const uint32_t bar = pair::map_to(smem_u32(&ctl->full[s]), 0);
            if (leader) mbar_arrive_expect_tx(&ctl->full[s], 2 * STAGE_B);
            ctl->issued[s] += 1;
            if (kind == 0) {
              const int k0 = key0 + (int)rank * KH;  // this CTA's 64 keys
              for (int cc = 0; cc < 4; ++cc) {
                const int d0 = (hs * 4 + cc) * 64;
                if (a.kv_token_major)
                  pair::tma_load_4d_pair(dst + cc * CHUNK_K, &tm_k, d0, g, k0, kb, bar);
                else
                  pair::tma_load_4d_pair(dst + cc * CHUNK_K, &tm_k, d0, k0, g, kb, bar);
              }
            } else {
              const int c0 = vh * DV + (int)rank * VH;  // this CTA's 128 output columns
              for (int c = 0; c < 2; ++c) {
                if (a.kv_token_major)
                  pair::tma_load_4d_pair(dst + c * CHUNK_V, &tm_v, c0 + c * 64, g, key0, kb, bar);
                else
                  pair::tma_load_4d_pair(dst + c * CHUNK_V, &tm_v, c0 + c * 64, key0, g, kb, bar);
              }
            }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader, one lane)
    if (leader && lane == 0) {
      bool ok = mbar_wait_bounded_at(&ctl->q_full, 0, abort_flag, deadline, a.status, 30, 0, 0, 0);
      if (ok) ctl->q_consumed = 1;
      int item = 0;
      for (int j = 0; j <= n_tiles && ok; ++j) {
        if (j < n_tiles) {
          const uint32_t d_s = tmem + COL_S + (uint32_t)(j & 1) * 128;
          for (int hs = 0; hs < Cfg::K_STAGES; ++hs, ++item) {
            const int s = item % NSTAGE;
            if (!mbar_wait_bounded_at(&ctl->full[s], (item / NSTAGE) & 1, abort_flag, deadline, a.status, 32,
                                      item, s, j)) {
              ok = false;
              break;
            }
            ctl->consumed[s] += 1;
            tc::fence_after_sync();
            const uint32_t st = sStage + s * STAGE_B;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t da = tc::smem_desc_sw128(sQ + (hs * 4 + cc) * CHUNK_Q + kk * 32, 16, 1024);
                const uint64_t db = tc::smem_desc_sw128(st + cc * CHUNK_K + kk * 32, 16, 1024);
                pair::mma2_ss(d_s, da, db, IDESC_S, (hs | cc | kk) != 0);
              }
            pair::commit2_mc(smem_u32(&ctl->empty[s]), BOTH);
          }
          if (!ok) break;
          pair::commit2_mc(smem_u32(&ctl->s_full[j & 1]), BOTH);
        }
        if (j >= 1) {
          if (!pair::wait_bounded_cluster(&ctl->p_ready, (j - 1) & 1, abort_flag, deadline, a.status, 34, j, 0,
                                          0)) {
            ok = false;
            break;
          }
          const uint32_t p_tm = tmem + COL_S + (uint32_t)((j - 1) & 1) * 128;
          const int s = item % NSTAGE;
          if (!mbar_wait_bounded_at(&ctl->full[s], (item / NSTAGE) & 1, abort_flag, deadline, a.status, 35,
                                    item, s, j)) {
            ok = false;
            break;
          }
          ctl->consumed[s] += 1;
          const uint32_t st = sStage + s * STAGE_B;
          const int64_t rows_valid = n_keys - (kt0 + j - 1) * BN;
          if (rows_valid < BN) clear_v_tail_pair(st, rows_valid > 0 ? (int)rows_valid : 0);
          tc::fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t db = tc::smem_desc_sw128(st + kk * 2048, CHUNK_V, 1024);
            pair::mma2_ts(tmem + COL_O, p_tm + kk * 8, db, IDESC_PV, (j - 1 > 0 || kk) ? 1u : 0u);
          }
          pair::commit2_mc(smem_u32(&ctl->empty[s]), BOTH);
          pair::commit2_mc(smem_u32(&ctl->o_done[(j - 1) & 1]), BOTH);
          ++item;
        }
      }
      // no MMA may be in flight when either CTA releases TMEM or shared memory
      pair::commit2_mc(smem_u32(&ctl->drain), BOTH);
    }
    __syncwarp();
    // the leader's MMAs read both CTAs' shared memory and write both TMEMs
    if (lane == 0) {
      volatile int never = 0;
      mbar_wait_bounded_at(&ctl->drain, 0, &never, deadline + 200000000ull, a.status, 37, 0, 0, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (both CTAs)
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tm = tmem + ((uint32_t)(wq * 32) << 16);
    const bool row_valid = q0 + row < a.S;
    const uint32_t p_ready_addr = pair::map_to(smem_u32(&ctl->p_ready), 0);
    int64_t lo, hi;
    visible_range(pos0 + (row_valid ? q0 + row : a.S - 1), a.window, n_keys, &lo, &hi);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    int pv_seen = 0;  // P.V products whose completion this thread has consumed
    for (int j = 0; j < n_tiles; ++j) {
      const int64_t kb = (kt0 + j) * BN;
      if (!wait_all(&ctl->s_full[j & 1], (j >> 1) & 1, abort_flag, deadline, a.status, 45, j)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t s_tm = tm + COL_S + (uint32_t)(j & 1) * 128;
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld32(s_tm + c * 32, r[c]);
      tc::tmem_wait_ld();
      // Logits arrive in log2 units (queries carry scale * log2 e). Keys this
      // row cannot see become -inf in place.
      if (!(kb >= lo && kb + BN - 1 <= hi)) {
        const int64_t dlo = lo - kb, dhi = hi - kb;
        const int c_lo = (int)(dlo < -1 ? -1 : dlo);
        const int c_hi = (int)(dhi > BN ? BN : dhi);
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int col = c * 32 + e;
            if (col < c_lo || col > c_hi) r[c][e] = __float_as_uint(-INFINITY);
          }
      }
      // One speculative pass against the running max; a row redoes the tile
      // only when its max moved by more than 2^8. Warps with a row that has
      // seen no key yet take the max first.
      float mx[8], ls[8];
      uint32_t pk[2][32];
      bool need;
      float alpha = 1.f;
      if (__any_sync(0xffffffffu, m_used == -INFINITY)) {
        const float m_new = fmaxf(m_used, max_row(r));
        need = m_new > m_used + RESCALE_LOG2 || (m_used == -INFINITY && m_new != -INFINITY);
        if (need) {
          alpha = (m_used == -INFINITY) ? 0.f : tc::ex2(m_used - m_new);
          l *= alpha;
          m_used = m_new;
        }
        exp_row<false>(r, m_used == -INFINITY ? 0.f : m_used, pk, ls, mx);
      } else {
        exp_row<true>(r, m_used, pk, ls, mx);
        const float m_new = fmaxf(m_used, max8(mx));
        need = m_new > m_used + RESCALE_LOG2;
        if (need) {
          alpha = tc::ex2(m_used - m_new);
          l *= alpha;
          m_used = m_new;
          exp_row<false>(r, m_used, pk, ls, mx);
        }
      }
      if (j >= 1 && __any_sync(0xffffffffu, need)) {
        // O must be stable: wait for P_{j-1} V_{j-1}
        if (pv_seen < j) {
          if (!wait_all(&ctl->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, deadline, a.status, 46, j)) {
            ok = false;
            break;
          }
          pv_seen = j;
        }
        tc::fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(tm + COL_O + c * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tc::tmem_st32(tm + COL_O + c * 32, o);
        }
        tc::tmem_wait_st();
      }
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      tc::tmem_st32(s_tm, pk[0]);
      tc::tmem_st32(s_tm + 32, pk[1]);
      // consume P_{j-1} V_{j-1} before P_{j+1} V_{j+1} can complete the next
      // phase of the same barrier (parity waits must not fall two behind)
      if (j >= 1 && pv_seen < j) {
        if (!wait_all(&ctl->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, deadline, a.status, 46, j)) {
          ok = false;
          break;
        }
        pv_seen = j;
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      // one arrival per warp: a cluster-scope release per thread costs a
      // fence each, and the warp's stores are complete after wait::st
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&ctl->p_ready);
        else
          pair::arrive_remote(p_ready_addr);
      }
    }
    if (ok)
      ok = wait_all(&ctl->o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, abort_flag, deadline,
                    a.status, 47, n_tiles);
    // Epilogue: O / l as bf16 into this CTA's Q buffer (free once the last
    // MMA is done), as the 128-byte-swizzled boxes of the output map, then
    // TMA stores of whole rows (rows past the sequence end are clipped).
    unsigned char* sO = sm;  // Q buffer
    if (ok) {
      tc::fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        tc::tmem_ld32(tm + COL_O + c * 32, o);
        tc::tmem_wait_ld();
        unsigned char* box_row = sO + (c >> 1) * CHUNK_Q + row * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(o[u * 8 + 0]) * inv, __uint_as_float(o[u * 8 + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(o[u * 8 + 2]) * inv, __uint_as_float(o[u * 8 + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(o[u * 8 + 4]) * inv, __uint_as_float(o[u * 8 + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(o[u * 8 + 6]) * inv, __uint_as_float(o[u * 8 + 7]) * inv);
          const int unit = ((c & 1) * 4 + u) ^ (row & 7);
          *reinterpret_cast<uint4*>(box_row + unit * 16) = w;
        }
      }
      if (row_valid && a.lse && vh == 0)
        a.lse[((int64_t)b * a.Hq + h) * a.S + q0 + row] =
            l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
    fence_proxy_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four softmax warps
    if (warp == 2 && lane == 0 && !*abort_flag && q0 < a.S) {
      for (int c = 0; c < DV / 64; ++c)
        tc::tma_store_4d(&tm_o, smem_u32(sO + c * CHUNK_Q), vh * DV + c * 64, h, q0, b);
      tc::bulk_commit();
      tc::bulk_wait_read0();
    }
  }

  __syncwarp();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // loads still in flight must land before shared memory is released. Both
    // CTAs' loads complete on the leader's barriers: the leader waits for the
    // phases it has armed; the peer, which has no barrier of its own to
    // watch, gives its loads a bounded 50 us.
    volatile int never = 0;
    const uint64_t dl = globaltimer_ns() + 200000000ull;
    if (leader) {
      if (ctl->q_issued && !ctl->q_consumed) mbar_wait_bounded_at(&ctl->q_full, 0, &never, dl, a.status, 49, 0, 0, 0);
      for (int s = 0; s < NSTAGE; ++s)
        if (ctl->issued[s] > ctl->consumed[s])
          mbar_wait_bounded_at(&ctl->full[s], (ctl->issued[s] - 1) & 1, &never, dl, a.status, 49,
                               ctl->issued[s], s, ctl->consumed[s]);
    } else {
      const uint64_t until = globaltimer_ns() + 50000ull;
      while (globaltimer_ns() < until) {
      }
    }
  }
  __syncwarp();
  // neither CTA leaves while the other may still arrive on its barriers
  pair::cluster_sync();
  if (warp == 1) {
    tc::fence_after_sync();
    pair::tmem_dealloc2(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
template <int D>
cudaError_t launch_pair(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                        const PairArgs& t, int B, cudaStream_t st) {
  using Cfg = PairCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(k_prefill_pair<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(2 * t.n_pairs, (t.head_pair ? t.Hq / 2 : t.Hq) * Cfg::NV, B);
  k_prefill_pair<D><<<grid, 192, Cfg::SMEM, st>>>(mq, mk, mv, mo, t);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attn_pair(const PrefillAttnArgs& a, int B, int D, int key_rows_total,
                                     int kv_token_major, int head_pair, cudaStream_t st) {
  if (D != 256 && D != 512) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mo;
  if (!make_prefill_maps(a, B, D, key_rows_total, kv_token_major, BM, KH, BN, &mq, &mk, &mv, &mo))
    return cudaErrorInvalidValue;
  PairArgs t;
  t.S = a.S;
  t.window = a.window;
  t.Hq = a.Hq;
  t.Hkv = a.Hkv;
  t.key_cap = a.key_cap;
  t.seq_lens_before = a.seq_lens_before;
  t.out = a.out;
  t.lse = a.lse;
  t.status = a.status;
  t.wait_ns = a.wait_ns;
  t.kv_token_major = kv_token_major;
  t.key_off_window = a.key_off_window;
  t.page_table = a.page_table;
  t.page_size = a.page_size;
  t.pages_per_seq = a.pages_per_seq;
  t.n_pages = a.n_pages;
  const int n_qtiles = (a.S + BM - 1) / BM;
  // head pairs need an even number of q heads per KV head (both share its K/V)
  t.head_pair = head_pair && (a.Hq / a.Hkv) % 2 == 0;
  t.n_pairs = t.head_pair ? n_qtiles : (n_qtiles + 1) / 2;
  return D == 256 ? launch_pair<256>(mq, mk, mv, mo, t, B, st) : launch_pair<512>(mq, mk, mv, mo, t, B, st);
}

}  // namespace hlg
