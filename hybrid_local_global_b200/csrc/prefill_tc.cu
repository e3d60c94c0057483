// prefill_tc.cu -- prefill attention on the 5th-generation tensor cores
// (tcgen05 MMA, TMEM accumulators, TMA-fed shared memory), head_dim 256 and
// 512.
//
// Computes, for every query row i of a (batch, q head) and its KV head
// g = h / (Hq/Hkv) ("Gemma 4: End-to-End Architecture Walkthrough", 3a/3b):
//   out_i = sum_j softmax_j(scale <q~_i, k~_j>) v_j   over visible keys j
// where visible means j <= pos_i and, on a local layer, j > pos_i - window.
//
// CTA = one 128-row query tile of one (batch, q head) and one 256-column
// half of the output (head_dim 512 uses two CTAs: the fp32 O tile of 128 x
// 512 alone would fill the 512 TMEM columns, so each CTA owns 256 output
// columns and computes S over all 512 dims); 192 threads:
//   warp 0     TMA producer: Q once (D/64 boxes of 128 rows x 64 dims), then
//              a ring of 32 KB stages in MMA order: K_0, K_1, V_0, K_2, V_1,
//              ... (a K tile = D/128 stages of 128 keys x 128 dims, a V tile
//              = 2 stages of 64 keys x 256 dims; 128-byte swizzle).
//   warp 1     TMEM owner and MMA issuer (one lane): S_j = Q K_j^T into one
//              of two 128-column TMEM buffers (M=128, N=128, K=D), then
//              O += P_{j-1} V_{j-1} (M=128, N=256, K=128) with P read from
//              TMEM; tcgen05.commit frees smem stages and signals S / O.
//   warps 2-5  softmax, one query row per thread (TMEM lane = row): load
//              S_j, mask edge tiles, online softmax in the log2 domain,
//              write P_j (bf16) over S_j's columns, rescale O in TMEM only
//              when the running max grows by more than 2^8; epilogue O / l.
// TMEM columns: O 0..255 (fp32), S/P buffers 256..383 and 384..511.
// The MMA pipe runs P_{j-1} V_{j-1} and S_{j+1} while the softmax works on
// S_j; the softmax waits for P_{j-1} V_{j-1} only before rescaling O (rare)
// and before releasing P_j, by which time it has normally completed.
//
// Tiles: key tiles [lo(first row), hi(last row)] only (window-aware
// skipping); per-element masks only on tiles that cross a row's range.
// Grid order puts the heaviest query tiles first (causal work grows with
// the tile index).
//
// Every wait is bounded by a %globaltimer deadline. On a timeout the CTA
// raises its abort flag, records GEMMA_ERR_DEVICE_TIMEOUT, waits for its
// issued MMAs (commit + bounded wait) and TMA loads, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace hlg {

namespace {

constexpr int BM = 128, BN = 128, DV = 256;  // DV: output columns per CTA
constexpr int CHUNK_B = 128 * 128;   // [128 rows][64 bf16] swizzled box
constexpr int STAGE_B = 32768;
constexpr int ALIGN_B = 1024;
constexpr int SMEM_MAX = 232448;     // opt-in dynamic shared memory per block
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_O = 0, COL_S = 256;
constexpr float RESCALE_LOG2 = 8.0f;
constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t IDESC_PV = tc::idesc_bf16_f32(128, 256, 0, 1);

template <int NSTAGE>
struct Ctl {
  uint64_t q_full;
  uint64_t full[NSTAGE];
  uint64_t empty[NSTAGE];
  uint64_t s_full[2];
  uint64_t p_ready;
  uint64_t o_done[2];  // PV_i completes phase i/2 of o_done[i % 2]
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int issued[NSTAGE];
  int consumed[NSTAGE];
  int q_issued, q_consumed;
};

template <int D>
struct TcCfg {
  static constexpr int Q_B = BM * D * 2;                 // 64 KB / 128 KB
  static constexpr int K_STAGES = D / 128;                // stages per K tile
  static constexpr int NV = D / DV;                       // CTAs per (tile, head)
  static constexpr int NSTAGE = (SMEM_MAX - ALIGN_B - Q_B - 512) / STAGE_B;  // 5 / 3
  static constexpr int SMEM = ALIGN_B + Q_B + NSTAGE * STAGE_B + (int)sizeof(Ctl<NSTAGE>);
  static_assert(NSTAGE >= 3 && SMEM <= SMEM_MAX, "shared memory plan");
};

struct TcArgs {
  int S, window, Hq, Hkv;
  int64_t key_cap;
  const int32_t* seq_lens_before;
  float scale_log2;
  bf16* out;
  float* lse;
  int* status;
  unsigned long long wait_ns;
  int kv_token_major;  // K/V map coordinates: 0 = (d, key, head, b), 1 = (d, head, key, b)
  int key_off_window;  // 1: K/V view row = position - (pos0 - window), else = position
  int n_qtiles;
  // paged cache (head-major views of the pool): view row = position % page_size,
  // view batch = page_table[b * pages_per_seq + position / page_size]; null: contiguous
  const int32_t* page_table;
  int page_size, pages_per_seq, n_pages;
  // multi-token decode (VF instances): rows (token t, q head g * G + i) = t * G + i
  // of KV head g, keys [split * chunk, +chunk) of the sequence's seq_lens[b]
  const int32_t* seq_lens;
  int tokens, chunk, n_splits;
  float* part_o;
  float* part_lse;
};

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t deadline, int* status, int where, int a = 0,
                                         int b = 0, int c = 0) {
  bool ok = mbar_wait_bounded_at(bar, parity, abort_flag, deadline, status, where, a, b, c);
  return __all_sync(0xffffffffu, ok);
}

// P = 2^(x - mb) over the 128 logits of one row, packed to bf16 pairs, with
// eight independent partial sums (and, if TRACK, partial maxima) so the
// reductions do not run down one dependency chain.
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

// VF: the multi-token decode instance (see launch_verify_attn_rows): a CTA is
// (KV head g and output half, sequence b, key split); its 128-row tile holds
// the G q heads of g for each of the `tokens` new tokens (rows past G *
// tokens see no key), and it writes fp32 partials O / l and log2-sum-exp for
// the combine instead of bf16 rows.
template <int D, bool VF>
__global__ void __launch_bounds__(192, 1)
    k_prefill_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                 const TcArgs a) {
  using Cfg = TcCfg<D>;
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

  const int G = a.Hq / a.Hkv;
  const int vh = blockIdx.x % Cfg::NV, b = blockIdx.y;
  const int h = VF ? 0 : (int)blockIdx.x / Cfg::NV;  // VF: per row, g * G + row % G
  const int g = VF ? (int)blockIdx.x / Cfg::NV : h / G;
  const int q0 = VF ? 0 : (a.n_qtiles - 1 - (int)blockIdx.z) * BM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int64_t pos0, n_keys, kt0;
  int n_tiles;
  if (VF) {
    // token t sits at position seq_lens[b] - tokens + t; this CTA reads keys
    // [split * chunk, min(+chunk, seq_lens[b]))
    n_keys = a.seq_lens[b];
    pos0 = n_keys - a.tokens;
    const int64_t k_begin = (int64_t)blockIdx.z * a.chunk;
    if (pos0 < 0 || n_keys > a.key_cap || k_begin >= n_keys) return;  // range reported by the append kernel
    const int64_t k_end = k_begin + a.chunk < n_keys ? k_begin + a.chunk : n_keys;
    kt0 = k_begin / BN;
    n_tiles = (int)((k_end - 1) / BN - kt0 + 1);
  } else {
    pos0 = a.seq_lens_before ? (int64_t)a.seq_lens_before[b] : 0;
    n_keys = pos0 + a.S;
  }
  // view row of a key = its position - koff (a gathered key window starts at pos0 - window)
  const int64_t koff = (!VF && a.key_off_window) ? pos0 - a.window : 0;
  if (!VF) {
    if (pos0 < 0 || n_keys - koff > a.key_cap) return;  // reported by the RoPE kernel
    int64_t lo_first, hi_first, lo_last, hi_last;
    visible_range(pos0 + q0, a.window, n_keys, &lo_first, &hi_first);
    visible_range(pos0 + min(q0 + BM - 1, a.S - 1), a.window, n_keys, &lo_last, &hi_last);
    kt0 = lo_first / BN;
    n_tiles = (int)(hi_last / BN - kt0 + 1);
  }

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
    mbar_init(&ctl->p_ready, 128);
    mbar_init(&ctl->o_done[0], 1);
    mbar_init(&ctl->o_done[1], 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ctl->q_issued = 0;
    ctl->q_consumed = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncwarp();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl->tmem_base;
  const uint64_t deadline = globaltimer_ns() + a.wait_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      if (VF) {
        // G heads x tokens rows; the tile's other rows are never stored
        mbar_arrive_expect_tx(&ctl->q_full, (uint32_t)(D * 2 * G * a.tokens));
        for (int c = 0; c < D / 64; ++c)
          tc::tma_load_4d(sQ + c * CHUNK_B, &tm_q, c * 64, g * G, 0, b, smem_u32(&ctl->q_full));
      } else {
        mbar_arrive_expect_tx(&ctl->q_full, Q_B);
        for (int c = 0; c < D / 64; ++c)
          tc::tma_load_4d(sQ + c * CHUNK_B, &tm_q, c * 64, h, q0, b, smem_u32(&ctl->q_full));
      }
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
          const int n_st = kind == 0 ? Cfg::K_STAGES : 2;
          for (int half = 0; half < n_st; ++half, ++item) {
            const int s = item % NSTAGE;
            if (item >= NSTAGE &&
                !mbar_wait_bounded_at(&ctl->empty[s], ((item / NSTAGE) - 1) & 1, abort_flag, deadline,
                                      a.status, 11, item, s, j)) {
              ok = false;
              break;
            }
            const uint32_t dst = sStage + s * STAGE_B;
            const uint32_t bar = smem_u32(&ctl->full[s]);
            mbar_arrive_expect_tx(&ctl->full[s], STAGE_B);
            ctl->issued[s] += 1;
            if (kind == 0) {
              for (int cc = 0; cc < 2; ++cc) {
                const int d0 = (half * 2 + cc) * 64;
                if (a.kv_token_major)
                  tc::tma_load_4d(dst + cc * CHUNK_B, &tm_k, d0, g, key0, kb, bar);
                else
                  tc::tma_load_4d(dst + cc * CHUNK_B, &tm_k, d0, key0, g, kb, bar);
              }
            } else {
              const int k0 = key0 + half * 64;
              for (int c = 0; c < 4; ++c) {
                if (a.kv_token_major)
                  tc::tma_load_4d(dst + c * 8192, &tm_v, vh * DV + c * 64, g, k0, kb, bar);
                else
                  tc::tma_load_4d(dst + c * 8192, &tm_v, vh * DV + c * 64, k0, g, kb, bar);
              }
            }
          }
        }
      }
    }
    __syncwarp();  // reconverge before the block barrier below
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = wait_all(&ctl->q_full, 0, abort_flag, deadline, a.status, 10);
    if (ok && lane == 0) ctl->q_consumed = 1;
    int item = 0;
    for (int j = 0; j <= n_tiles && ok; ++j) {
      if (j < n_tiles) {
        const uint32_t d_s = tmem + COL_S + (uint32_t)(j & 1) * 128;
        for (int half = 0; half < Cfg::K_STAGES; ++half, ++item) {
          const int s = item % NSTAGE;
          if (!wait_all(&ctl->full[s], (item / NSTAGE) & 1, abort_flag, deadline, a.status, 12, item, s, j)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            ctl->consumed[s] += 1;
            tc::fence_after_sync();
            const uint32_t st = sStage + s * STAGE_B;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t da = tc::smem_desc_sw128(sQ + (half * 2 + cc) * CHUNK_B + kk * 32, 16, 1024);
                const uint64_t db = tc::smem_desc_sw128(st + cc * CHUNK_B + kk * 32, 16, 1024);
                tc::mma_ss(d_s, da, db, IDESC_S, (half | cc | kk) != 0);
              }
            tc::commit(smem_u32(&ctl->empty[s]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc::commit(smem_u32(&ctl->s_full[j & 1]));
      }
      if (j >= 1) {
        if (!wait_all(&ctl->p_ready, (j - 1) & 1, abort_flag, deadline, a.status, 13, j)) {
          ok = false;
          break;
        }
        const int64_t tile_key0 = (kt0 + j - 1) * BN;
        const uint32_t p_tm = tmem + COL_S + (uint32_t)((j - 1) & 1) * 128;
        for (int half = 0; half < 2; ++half, ++item) {
          const int s = item % NSTAGE;
          if (!wait_all(&ctl->full[s], (item / NSTAGE) & 1, abort_flag, deadline, a.status, 14, item, s, j)) {
            ok = false;
            break;
          }
          const uint32_t st = sStage + s * STAGE_B;
          const int64_t rows_valid = n_keys - (tile_key0 + half * 64);
          if (rows_valid < 64) {
            // keys past the sequence: their P is 0, but their V rows must be finite
            const int r0 = rows_valid > 0 ? (int)rows_valid : 0;
            for (int idx = lane; idx < (64 - r0) * 4 * 8; idx += 32) {
              const int r = r0 + idx / 32, c = (idx / 8) % 4, u = idx % 8;
              *reinterpret_cast<uint4*>(sm + (st - base) + c * 8192 + r * 128 + u * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          if (lane == 0) {
            ctl->consumed[s] += 1;
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t db = tc::smem_desc_sw128(st + kk * 2048, 8192, 1024);
              tc::mma_ts(tmem + COL_O, p_tm + half * 32 + kk * 8, db, IDESC_PV,
                         (j - 1 > 0 || half || kk) ? 1u : 0u);
            }
            tc::commit(smem_u32(&ctl->empty[s]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc::commit(smem_u32(&ctl->o_done[(j - 1) & 1]));
      }
    }
    // make sure no MMA is in flight before TMEM can be released
    if (lane == 0) {
      tc::commit(smem_u32(&ctl->drain));
      volatile int never = 0;
      mbar_wait_bounded_at(&ctl->drain, 0, &never, globaltimer_ns() + 200000000ull, a.status, 18, 0, 0, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t tm = tmem + ((uint32_t)(wq * 32) << 16);
    const bool row_valid = VF ? row < G * a.tokens : q0 + row < a.S;
    int64_t lo, hi;
    if (VF) {
      // keys up to the row's token (global layer); a row past the tokens sees none
      lo = row_valid ? 0 : 1;
      hi = row_valid ? pos0 + row / G : 0;
    } else {
      visible_range(pos0 + (row_valid ? q0 + row : a.S - 1), a.window, n_keys, &lo, &hi);
    }
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    int pv_seen = 0;  // P.V products whose completion this thread has consumed
    for (int j = 0; j < n_tiles; ++j) {
      const int64_t kb = (kt0 + j) * BN;
      if (!wait_all(&ctl->s_full[j & 1], (j >> 1) & 1, abort_flag, deadline, a.status, 15, j)) {
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
      // row cannot see become -inf in place (only tiles that straddle the
      // visible range need it).
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
      // The running max m_used only moves when a tile's max exceeds it by more
      // than 2^8 (or on a row's first visible key), so P = 2^(x - m_used) is
      // computed in one pass that also takes the tile max, and redone in the
      // rare case the max moved. A warp with a row that has seen no key yet
      // takes the max first instead, since its speculation would always fail.
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
          if (!wait_all(&ctl->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, deadline, a.status, 16, j)) {
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
        if (!wait_all(&ctl->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, deadline, a.status, 16, j)) {
          ok = false;
          break;
        }
        pv_seen = j;
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      mbar_arrive(&ctl->p_ready);
    }
    if (ok)
      ok = wait_all(&ctl->o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, abort_flag, deadline,
                    a.status, 17, n_tiles);
    // Epilogue: O / l as bf16 into the Q buffer (free once the last MMA is
    // done), laid out as the 128-byte-swizzled boxes of the output map, then
    // four TMA stores. A thread owns one row, so direct stores would write
    // 16 bytes per output row per instruction; the staged copy writes whole
    // rows. Rows past the sequence end are clipped by the store.
    unsigned char* sO = sm;  // Q buffer
    if (VF) {
      // fp32 partial O / l of this split and its log2-sum-exp, for the combine
      if (ok) {
        tc::fence_after_sync();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const int t = row / G;
        const int64_t pr = (((int64_t)b * a.tokens + t) * a.Hq + g * G + row % G) * a.n_splits + blockIdx.z;
        float* dst = a.part_o + pr * D + vh * DV;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(tm + COL_O + c * 32, o);  // every lane: the load is warp-wide
          tc::tmem_wait_ld();
          if (row_valid) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<float4*>(dst + c * 32 + u * 4) =
                  make_float4(__uint_as_float(o[u * 4 + 0]) * inv, __uint_as_float(o[u * 4 + 1]) * inv,
                              __uint_as_float(o[u * 4 + 2]) * inv, __uint_as_float(o[u * 4 + 3]) * inv);
          }
        }
        if (row_valid && vh == 0) a.part_lse[pr] = l > 0.f ? m_used + __log2f(l) : -INFINITY;
      }
    } else if (ok) {
      tc::fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        tc::tmem_ld32(tm + COL_O + c * 32, o);
        tc::tmem_wait_ld();
        unsigned char* box_row = sO + (c >> 1) * CHUNK_B + row * 128;
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
    if (!VF && warp == 2 && lane == 0 && !*abort_flag) {
      for (int c = 0; c < DV / 64; ++c)
        tc::tma_store_4d(&tm_o, smem_u32(sO + c * CHUNK_B), vh * DV + c * 64, h, q0, b);
      tc::bulk_commit();
      tc::bulk_wait_read0();
    }
  }

  __syncwarp();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // loads still in flight must land before shared memory is released
    volatile int never = 0;
    const uint64_t dl = globaltimer_ns() + 200000000ull;
    if (ctl->q_issued && !ctl->q_consumed) mbar_wait_bounded_at(&ctl->q_full, 0, &never, dl, a.status, 19, 0, 0, 0);
    for (int s = 0; s < NSTAGE; ++s)
      if (ctl->issued[s] > ctl->consumed[s])
        mbar_wait_bounded_at(&ctl->full[s], (ctl->issued[s] - 1) & 1, &never, dl, a.status, 19,
                             ctl->issued[s], s, ctl->consumed[s]);
  }
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_prefill_attn_tc(const PrefillAttnArgs& a, int B, int D, int key_rows_total,
                                   int kv_token_major, cudaStream_t st) {
  if (D != 256 && D != 512) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mo;
  if (!make_prefill_maps(a, B, D, key_rows_total, kv_token_major, BM, BN, 64, &mq, &mk, &mv, &mo))
    return cudaErrorInvalidValue;
  TcArgs t;
  t.S = a.S;
  t.window = a.window;
  t.Hq = a.Hq;
  t.Hkv = a.Hkv;
  t.key_cap = a.key_cap;
  t.seq_lens_before = a.seq_lens_before;
  t.scale_log2 = a.scale_log2;
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
  t.n_qtiles = (a.S + BM - 1) / BM;
  if (D == 256) {
    using Cfg = TcCfg<256>;
    cudaError_t e =
        cudaFuncSetAttribute(k_prefill_tc<256, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hq * Cfg::NV, B, t.n_qtiles);
    k_prefill_tc<256, false><<<grid, 192, Cfg::SMEM, st>>>(mq, mk, mv, mo, t);
  } else {
    using Cfg = TcCfg<512>;
    cudaError_t e =
        cudaFuncSetAttribute(k_prefill_tc<512, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hq * Cfg::NV, B, t.n_qtiles);
    k_prefill_tc<512, false><<<grid, 192, Cfg::SMEM, st>>>(mq, mk, mv, mo, t);
  }
  return cudaGetLastError();
}

namespace {
template <int D>
cudaError_t launch_verify_as(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const TcArgs& t,
                             int B, cudaStream_t st) {
  using Cfg = TcCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(k_prefill_tc<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(t.Hkv * Cfg::NV, B, t.n_splits);
  k_prefill_tc<D, true><<<grid, 192, Cfg::SMEM, st>>>(mq, mk, mv, mq, t);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_verify_attn_rows(const VerifyAttnArgs& a, int B, int D, cudaStream_t st) {
  const int G = a.Hq / a.Hkv;
  if ((D != 256 && D != 512) || a.tokens < 1 || G * a.tokens > BM || a.chunk % BN || a.n_splits < 1)
    return cudaErrorInvalidValue;
  const uint64_t E = 2;
  CUtensorMap mq, mk, mv;
  {
    // q_rot [B][tokens][Hq][D]: a box is the G heads of one KV head for every token
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)a.Hq, (uint64_t)a.tokens, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)D * E, (uint64_t)a.Hq * D * E, (uint64_t)a.tokens * a.Hq * D * E};
    const uint32_t box[4] = {64, (uint32_t)G, (uint32_t)a.tokens, 1};
    if (!make_map_bf16_4d(&mq, a.q_rot, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    // head-major views (d, row, head, page) of the cache (a page per sequence
    // when contiguous), K boxes of 128 rows, V boxes of 64
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)a.page_size, (uint64_t)a.Hkv, (uint64_t)a.n_pages};
    const uint64_t strk[3] = {(uint64_t)a.k.stride_row * E, (uint64_t)a.k.stride_h * E, (uint64_t)a.k.stride_b * E};
    const uint64_t strv[3] = {(uint64_t)a.v.stride_row * E, (uint64_t)a.v.stride_h * E, (uint64_t)a.v.stride_b * E};
    const uint32_t bk[4] = {64, (uint32_t)BN, 1, 1}, bv[4] = {64, 64, 1, 1};
    if (!make_map_bf16_4d(&mk, a.k.ptr, dims, strk, bk) || !make_map_bf16_4d(&mv, a.v.ptr, dims, strv, bv))
      return cudaErrorInvalidValue;
  }
  TcArgs t{};
  t.S = a.tokens;
  t.window = 0;
  t.Hq = a.Hq;
  t.Hkv = a.Hkv;
  t.key_cap = a.cache_cap;
  t.seq_lens_before = nullptr;
  t.scale_log2 = 1.f;
  t.out = nullptr;
  t.lse = nullptr;
  t.status = a.status;
  t.wait_ns = a.wait_ns;
  t.kv_token_major = 0;
  t.key_off_window = 0;
  t.n_qtiles = 1;
  t.page_table = a.page_table;
  t.page_size = a.page_size;
  t.pages_per_seq = a.pages_per_seq;
  t.n_pages = a.n_pages;
  t.seq_lens = a.seq_lens;
  t.tokens = a.tokens;
  t.chunk = a.chunk;
  t.n_splits = a.n_splits;
  t.part_o = a.part_o;
  t.part_lse = a.part_lse;
  return D == 256 ? launch_verify_as<256>(mq, mk, mv, t, B, st) : launch_verify_as<512>(mq, mk, mv, t, B, st);
}

}  // namespace hlg
