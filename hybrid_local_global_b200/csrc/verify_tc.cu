// verify_tc.cu -- multi-token decode with the tensor cores: `tokens` new
// tokens per sequence (a drafter's proposals that the target model checks
// in one pass, "Gemma 4: End-to-End Architecture Walkthrough", Phase 4;
// "Gemma 4: Architecture, Training and Local Deployment", 3.4), each
// attending to the cached keys it sees and to the earlier new tokens: all
// of them on a global layer, the window before its own position on a local
// one ("Gemma 4: End-to-End Architecture Walkthrough", 3a/3b).
//
// Decode-shaped: few query rows (G q heads x tokens <= 64 per KV head)
// against many keys, so the product is taken transposed. Per tile of 128
// keys:
//   S^T = K Q^T    (M = 128 keys, N = NQ query rows, K = head_dim)
//   O^T += V^T P^T (M = 128 value dims per MMA, N = NQ, K = 128 keys)
// The query rows are the MMA's N dimension, so one CTA covers every q head
// of its KV head for all the tokens and each cached K/V byte is streamed
// once (the 128-row-tile form needs two CTAs per head at head_dim 512 and
// re-reads K). TMEM holds S^T (two buffers of NQ columns) and O^T
// (head_dim / 128 blocks of NQ columns); P^T goes through shared memory as
// the B operand of the second product, K-major. V tiles are the A operand
// read MN-major (value dims contiguous), as TMA lays them down.
//
// CTA = (KV head, sequence, split of `chunk` keys); 192 threads:
//   warp 0      TMA producer: Q once, then K_j and V_{j-1} in 32 KB stages
//               (128 keys x 128 dims) through a ring;
//   warp 1      MMA issuer (one lane) and TMEM owner;
//   warps 2..5  softmax: thread = one key of the tile (its TMEM lane), NQ
//               logits each (log2 units: the queries carry scale * log2 e).
//               Column (query) maxima are only formed when some logit
//               exceeds its column's running max by more than 2^8 (a
//               barrier reduction over the 128 threads decides); then O^T
//               and the partial sums are rescaled. Each thread keeps partial
//               column sums of its keys; they are reduced once at the end.
// Output: per query row, the split's normalised O and log2-sum-exp in the
// same layout as single-token decode, merged by launch_decode_combine; with
// a single split the normalised O goes straight to the bf16 output.
// Local layers (LOCAL) read their ring as it was before the new tokens plus
// a tail tile of the new rows (see k_verify_tc); global layers may sit in a
// paged pool (a tile's page from the page table).
//
// Every wait is bounded (%globaltimer deadline): a timeout raises the
// CTA's abort flag and records GEMMA_ERR_DEVICE_TIMEOUT; copies in flight
// are waited for (bounded) before the CTA exits.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace hlg {

namespace {

constexpr int BN = 128;             // keys per tile: the M of S^T
constexpr int CH_B = BN * 128;      // one [128 keys][64 dims] swizzled box
constexpr int STAGE_B = 2 * CH_B;   // 128 dims of a K or V tile
constexpr int ALIGN_B = 1024;
constexpr int SMEM_MAX = 232448;    // opt-in dynamic shared memory per block
constexpr float RESCALE_LOG2 = 8.0f;

template <int NSTAGE>
struct VCtl {
  uint64_t q_full;
  uint64_t full[NSTAGE];
  uint64_t empty[NSTAGE];
  uint64_t s_full[2];
  uint64_t p_ready[2];  // P^T of tile i in buffer i % 2: phase i/2 of p_ready[i % 2]
  uint64_t o_done[2];  // PV_i completes phase i/2 of o_done[i % 2]
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int issued[NSTAGE];
  int consumed[NSTAGE];
  int q_issued, q_consumed;
};

// CTAS: resident CTAs per SM. A local layer's CTA streams one ring (about 1
// MB at the 31B shape), so its prologue and epilogue weigh; two per SM with
// a 2-stage ring overlap them (measured on the 31B-shaped B64 block, k = 4:
// 208 -> 191 us per local layer). Global CTAs keep one per SM and the
// deepest ring.
template <int D, int NQ, bool LOCAL = false>
struct VCfg {
  static constexpr int CTAS = (LOCAL && D == 256 && NQ == 32) ? 2 : 1;
  static constexpr int MT = D / 128;     // K stages per tile = O^T blocks = V stages per tile
  static constexpr int Q_CH = NQ * 128;  // 64 dims of the NQ query rows
  static constexpr int Q_B = (D / 64) * Q_CH;
  static constexpr int P_CH = NQ * 128;  // 64 keys of P^T (rows = queries)
  static constexpr int P_BUF = 2 * P_CH;
  static constexpr int RED_B = 6 * NQ * 4;  // red [4][NQ], running maxima [NQ], factors [NQ]
  static constexpr int FIXED = ALIGN_B + Q_B + 2 * P_BUF + RED_B + (int)sizeof(VCtl<8>);
  static constexpr int NS_FIT = ((CTAS == 1 ? SMEM_MAX : 228 * 1024 / CTAS - 1024) - FIXED) / STAGE_B;
  static constexpr int NSTAGE = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int SMEM = ALIGN_B + NSTAGE * STAGE_B + Q_B + 2 * P_BUF + RED_B + (int)sizeof(VCtl<NSTAGE>);
  static constexpr uint32_t COL_O = 0;
  static constexpr uint32_t COL_S = MT * NQ;
  static constexpr uint32_t COLS = MT * NQ + 2 * NQ;
  static constexpr uint32_t TMEM_COLS = COLS <= 128 ? 128 : COLS <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_ST = tc::idesc_bf16_f32(128, NQ, 0, 0);  // K (K-major) x Q (K-major)
  static constexpr uint32_t IDESC_OT = tc::idesc_bf16_f32(128, NQ, 1, 0);  // V^T (MN-major) x P^T (K-major)
  static_assert(COLS <= 512, "TMEM plan");
  static_assert(NSTAGE >= (CTAS == 1 ? 3 : 2) && SMEM <= SMEM_MAX, "shared memory plan");
};

struct VArgs {
  int Hq, Hkv, tokens, chunk, n_splits;
  bf16* out;  // one split: O / l straight into [B][tokens][Hq][D] (no partials, no combine); else null
  int window;  // LOCAL: ring slots
  int64_t key_cap;
  const int32_t* page_table;  // global layers on a paged pool (see VerifyAttnArgs); else null
  int page_size, pages_per_seq, n_pages;
  const int32_t* seq_lens;
  float* part_o;
  float* part_lse;
  int* status;
  unsigned long long wait_ns;
  int drop_first_copy;  // test hook: the first K stage of unit (0, 0, 0) is never issued
};

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t deadline, int* status, int where, int a = 0,
                                         int b = 0, int c = 0) {
  bool ok = mbar_wait_bounded_at(bar, parity, abort_flag, deadline, status, where, a, b, c);
  return __all_sync(0xffffffffu, ok);
}

// OR of a predicate over the 128 softmax threads (named barrier 1).
__device__ __forceinline__ bool any128(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void sync128() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Column reduction across a warp: x[c] is this lane's value of column c;
// lane l returns the max (MAX) or sum over the 32 lanes of column l. Each
// step hands half of the remaining columns to the partner lane, so the 32
// columns take 31 shuffles in all.
template <bool MAX>
__device__ __forceinline__ float reduce_columns(float (&x)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = lane & o;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? x[i] : x[i + o];
      const float keep = up ? x[i + o] : x[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, o);
      x[i] = MAX ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return x[0];
}

// LOCAL: a local layer. The K/V maps are the ring as it was before the new
// tokens (slot s holds the latest position p < pos0 with p % window == s,
// if p >= 0); split z takes the slots [z * chunk, +chunk), and the last
// split also a tail tile of the new tokens' keys and values (tm_kt / tm_vt,
// [B][tokens][Hkv][D]). Every split writes a partial.
template <int D, int NQ, bool LOCAL>
__global__ void __launch_bounds__(192, VCfg<D, NQ, LOCAL>::CTAS)
    k_verify_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
                const __grid_constant__ CUtensorMap tm_vt, const VArgs a) {
  using C = VCfg<D, NQ, LOCAL>;
  constexpr int NSTAGE = C::NSTAGE;
  constexpr int MT = C::MT;
  extern __shared__ unsigned char sm_raw[];
  const uint32_t raw = smem_u32(sm_raw);
  const uint32_t base = (raw + ALIGN_B - 1) & ~(uint32_t)(ALIGN_B - 1);
  unsigned char* sm = sm_raw + (base - raw);
  const uint32_t sStage = base;
  const uint32_t sQ = base + NSTAGE * STAGE_B;
  const uint32_t sP = sQ + C::Q_B;
  float* red = reinterpret_cast<float*>(sm + NSTAGE * STAGE_B + C::Q_B + 2 * C::P_BUF);  // [4][NQ]
  float* m_s = red + 4 * NQ;   // running column maxima (log2 units)
  float* f_s = m_s + NQ;       // per-column factors: rescale, then 1 / sum
  VCtl<NSTAGE>* ctl = reinterpret_cast<VCtl<NSTAGE>*>(f_s + NQ);
  volatile int* abort_flag = &ctl->abort;

  const int g = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int nvalid = G * a.tokens;  // query rows: row t * G + i = (token t, q head g * G + i)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // token t sits at position pos0 + t; this CTA reads keys (global) or ring
  // slots (LOCAL) [k_begin, k_end), tile j starting at k_begin + j * BN
  const int64_t n_keys = a.seq_lens[b];
  const int64_t pos0 = n_keys - a.tokens;
  const int64_t k_begin = (int64_t)split * a.chunk;
  const int64_t k_stop = LOCAL ? (int64_t)a.window : n_keys;
  if (pos0 < 0 || (!LOCAL && n_keys > a.key_cap) || k_begin >= k_stop) {  // checked by the append kernel
    if (a.out && pos0 < 0)  // no combine will zero these rows
      for (int i = threadIdx.x; i < nvalid * D; i += blockDim.x) {
        const int n = i / D;
        a.out[(((int64_t)b * a.tokens + n / G) * a.Hq + g * G + n % G) * D + i % D] = __float2bfloat16_rn(0.f);
      }
    return;
  }
  const int64_t k_end = k_begin + a.chunk < k_stop ? k_begin + a.chunk : k_stop;
  const int n_ring = (int)((k_end - k_begin + BN - 1) / BN);
  const int n_tiles = n_ring + ((LOCAL && split == a.n_splits - 1) ? 1 : 0);  // LOCAL: + the tail tile
  // keys of a tile that hold data (V rows past them are zeroed): global,
  // up to the sequence end; ring, the slots already written
  const int64_t data_end = LOCAL ? (pos0 < a.window ? pos0 : (int64_t)a.window) : n_keys;

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
    mbar_init(&ctl->p_ready[0], 128);
    mbar_init(&ctl->p_ready[1], 128);
    mbar_init(&ctl->o_done[0], 1);
    mbar_init(&ctl->o_done[1], 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ctl->q_issued = 0;
    ctl->q_consumed = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < NQ) m_s[threadIdx.x] = -INFINITY;
  if (warp >= 2 && nvalid < NQ) {
    // query rows past nvalid: zeros (the TMA box fills rows 0..nvalid-1)
    const int t = threadIdx.x - 64, pad = NQ - nvalid;
    for (int i = t; i < (D / 64) * pad * 8; i += 128) {
      const int c = i / (pad * 8), r = nvalid + (i / 8) % pad, u = i % 8;
      *reinterpret_cast<uint4*>(sm + (sQ - base) + c * C::Q_CH + r * 128 + u * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(&ctl->tmem_base), C::TMEM_COLS);
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
      if (LOCAL) {
        tc::prefetch_tmap(&tm_kt);
        tc::prefetch_tmap(&tm_vt);
      }
      mbar_arrive_expect_tx(&ctl->q_full, (uint32_t)(D * 2 * nvalid));
      for (int c = 0; c < D / 64; ++c)
        tc::tma_load_4d(sQ + c * C::Q_CH, &tm_q, c * 64, g * G, 0, b, smem_u32(&ctl->q_full));
      ctl->q_issued = 1;
      int item = 0;
      bool ok = true;
      for (int j = 0; j <= n_tiles && ok; ++j) {
        for (int kind = 0; kind < 2 && ok; ++kind) {  // 0: K_j, 1: V_{j-1}
          if ((kind == 0 && j == n_tiles) || (kind == 1 && j == 0)) continue;
          const int jt = j - kind;
          const bool tail = LOCAL && jt == n_ring;
          const int key0 = (int)(k_begin + (int64_t)jt * BN);
          const CUtensorMap* map = tail ? (kind == 0 ? &tm_kt : &tm_vt) : (kind == 0 ? &tm_k : &tm_v);
          // view row and batch of the tile: a page of the pool (a tile never
          // straddles a page: page_size is a multiple of 128), or the sequence
          int row = key0, page = b;
          if (!LOCAL && a.page_table) {
            const int pi = key0 / a.page_size;
            page = pi < a.pages_per_seq ? a.page_table[(int64_t)b * a.pages_per_seq + pi] : 0;
            if (page < 0 || page >= a.n_pages) {  // a page outside the pool: report, read page 0
              set_status(a.status, GEMMA_ERR_DEVICE_RANGE);
              page = 0;
            }
            row = key0 - pi * a.page_size;
          }
          for (int h = 0; h < MT; ++h, ++item) {
            const int s = item % NSTAGE;
            if (item >= NSTAGE &&
                !mbar_wait_bounded_at(&ctl->empty[s], ((item / NSTAGE) - 1) & 1, abort_flag, deadline,
                                      a.status, 31, item, s, j)) {
              ok = false;
              break;
            }
            if (a.drop_first_copy && item == 0 && split == 0 && g == 0 && b == 0) continue;
            const uint32_t dst = sStage + s * STAGE_B;
            const uint32_t bar = smem_u32(&ctl->full[s]);
            mbar_arrive_expect_tx(&ctl->full[s], STAGE_B);
            ctl->issued[s] += 1;
            for (int cc = 0; cc < 2; ++cc) {
              if (tail)  // (d, head, token, b): tokens past the last are zeros
                tc::tma_load_4d(dst + cc * CH_B, map, h * 128 + cc * 64, g, 0, b, bar);
              else
                tc::tma_load_4d(dst + cc * CH_B, map, h * 128 + cc * 64, row, g, page, bar);
            }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = wait_all(&ctl->q_full, 0, abort_flag, deadline, a.status, 30);
    if (ok && lane == 0) ctl->q_consumed = 1;
    int item = 0;
    for (int j = 0; j <= n_tiles && ok; ++j) {
      if (j < n_tiles) {
        const uint32_t d_s = tmem + C::COL_S + (uint32_t)(j & 1) * NQ;
        for (int h = 0; h < MT; ++h, ++item) {
          const int s = item % NSTAGE;
          if (!wait_all(&ctl->full[s], (item / NSTAGE) & 1, abort_flag, deadline, a.status, 32, item, s, j)) {
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
                const uint64_t da = tc::smem_desc_sw128(st + cc * CH_B + kk * 32, 16, 1024);
                const uint64_t db = tc::smem_desc_sw128(sQ + (h * 2 + cc) * C::Q_CH + kk * 32, 16, 1024);
                tc::mma_ss(d_s, da, db, C::IDESC_ST, (h | cc | kk) != 0);
              }
            tc::commit(smem_u32(&ctl->empty[s]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc::commit(smem_u32(&ctl->s_full[j & 1]));
      }
      if (j >= 1) {
        // one barrier per P buffer: the softmax writes P^T of tile j + 1
        // into this buffer only after PV_{j-1}, issued below, so it arrives
        // at most one phase ahead of this wait
        if (!wait_all(&ctl->p_ready[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, deadline, a.status, 33, j)) {
          ok = false;
          break;
        }
        const int64_t rows_valid =
            (LOCAL && j - 1 == n_ring) ? BN : data_end - (k_begin + (int64_t)(j - 1) * BN);
        const uint32_t pb = sP + (uint32_t)((j - 1) & 1) * C::P_BUF;
        for (int m = 0; m < MT; ++m, ++item) {
          const int s = item % NSTAGE;
          if (!wait_all(&ctl->full[s], (item / NSTAGE) & 1, abort_flag, deadline, a.status, 34, item, s, j)) {
            ok = false;
            break;
          }
          const uint32_t st = sStage + s * STAGE_B;
          if (rows_valid < BN) {
            // keys past the sequence: their P is 0, but their V rows must be finite
            const int r0 = rows_valid > 0 ? (int)rows_valid : 0;
            for (int idx = lane; idx < (BN - r0) * 16; idx += 32) {
              const int r = r0 + idx / 16, cc = (idx / 8) & 1, u = idx & 7;
              *reinterpret_cast<uint4*>(sm + (st - base) + cc * CH_B + r * 128 + u * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          if (lane == 0) {
            ctl->consumed[s] += 1;
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              // V^T: 128 dims (two 64-dim boxes CH_B apart) x 16 keys; P^T: NQ rows x 16 keys
              const uint64_t da = tc::smem_desc_sw128(st + kk * 2048, CH_B, 1024);
              const uint64_t db = tc::smem_desc_sw128(pb + (kk >> 2) * C::P_CH + (kk & 3) * 32, 16, 1024);
              tc::mma_ss(tmem + C::COL_O + m * NQ, da, db, C::IDESC_OT, (j - 1 > 0 || kk) ? 1u : 0u);
            }
            tc::commit(smem_u32(&ctl->empty[s]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc::commit(smem_u32(&ctl->o_done[(j - 1) & 1]));
      }
    }
    // no MMA may be in flight when TMEM is released
    if (lane == 0) {
      tc::commit(smem_u32(&ctl->drain));
      volatile int never = 0;
      mbar_wait_bounded_at(&ctl->drain, 0, &never, globaltimer_ns() + 200000000ull, a.status, 38, 0, 0, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int kl = q4 * 32 + lane;  // this thread's key of the tile = its TMEM lane
    const uint32_t tm = tmem + ((uint32_t)(q4 * 32) << 16);
    float l[NQ];  // this thread's partial column sums
#pragma unroll
    for (int n = 0; n < NQ; ++n) l[n] = 0.f;
    // The running maxima live in shared memory (m_s, the same for every
    // thread; written by thread kl for column kl between barriers). The four
    // warps pass the same named barriers in the same order whatever their
    // waits return: a failed wait marks the thread bad, and the vote at the
    // top of the next tile ends the loop for all of them together.
    bool ok = true, bad = false;
    int pv_seen = 0;  // PV_0 .. PV_{pv_seen-1} are known complete
    for (int j = 0; j < n_tiles; ++j) {
      if (!bad && !wait_all(&ctl->s_full[j & 1], (j >> 1) & 1, abort_flag, deadline, a.status, 35, j)) bad = true;
      if (any128(bad)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float v[NQ];
      {
        uint32_t r[NQ / 32][32];
#pragma unroll
        for (int c = 0; c < NQ / 32; ++c) tc::tmem_ld32(tm + C::COL_S + (uint32_t)(j & 1) * NQ + c * 32, r[c]);
        tc::tmem_wait_ld();
#pragma unroll
        for (int n = 0; n < NQ; ++n) v[n] = __uint_as_float(r[n / 32][n % 32]);
      }
      // visible rows [n_lo, n_hi) for this thread's key. Global, and the
      // tail tile: row t * G + i sees keys up to pos0 + t. Ring: token t sees
      // the positions after pos0 + t - window, so slot s, at distance
      // d = (pos0 - 1 - s) mod window below pos0, is seen by tokens
      // t <= window - 2 - d (none if the slot is unwritten or past the ring).
      // Rows past nvalid see nothing.
      int n_lo = 0, n_hi = nvalid;
      if (LOCAL && j < n_ring) {
        const int64_t slot = k_begin + (int64_t)j * BN + kl;
        const int64_t d = (pos0 - 1 - slot) % a.window;
        const int64_t dd = d < 0 ? d + a.window : d;
        const bool written = slot < a.window && dd <= pos0 - 1;
        const int64_t t_max1 = a.window - 1 - dd;  // tokens 0 .. t_max1 - 1 see the slot
        n_hi = !written ? 0 : t_max1 >= a.tokens ? nvalid : (int)t_max1 * G;
      } else {
        const int64_t dk = LOCAL ? (int64_t)kl : k_begin + (int64_t)j * BN + kl - pos0;
        n_lo = dk <= 0 ? 0 : dk >= a.tokens ? NQ : (int)dk * G;
      }
      if (n_lo > 0 || n_hi < NQ) {
#pragma unroll
        for (int n = 0; n < NQ; ++n)
          if (n < n_lo || n >= n_hi) v[n] = -INFINITY;
      }
      bool need = false;
#pragma unroll
      for (int n = 0; n < NQ; n += 4) {
        const float4 m4 = *reinterpret_cast<const float4*>(m_s + n);
        need |= (v[n] > m4.x + RESCALE_LOG2) | (v[n + 1] > m4.y + RESCALE_LOG2) |
                (v[n + 2] > m4.z + RESCALE_LOG2) | (v[n + 3] > m4.w + RESCALE_LOG2);
      }
      if (any128(need)) {
        // column maxima of the tile; thread kl < NQ then moves column kl's maximum
#pragma unroll
        for (int c = 0; c < NQ / 32; ++c) {
          float x[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = v[c * 32 + e];
          red[q4 * NQ + c * 32 + lane] = reduce_columns<true>(x, lane);
        }
        sync128();
        bool moved = false;
        if (kl < NQ) {
          const float tmax = fmaxf(fmaxf(red[kl], red[NQ + kl]), fmaxf(red[2 * NQ + kl], red[3 * NQ + kl]));
          const float mold = m_s[kl], mnew = fmaxf(mold, tmax);
          f_s[kl] = mold == -INFINITY ? 0.f : tc::ex2(mold - mnew);
          m_s[kl] = mnew;
          moved = mold != -INFINITY && mnew != mold;
        }
        moved = any128(moved);  // also publishes m_s and f_s
#pragma unroll
        for (int n = 0; n < NQ; ++n) l[n] *= f_s[n];
        if (moved && j >= 1) {
          // O^T must hold PV_{j-1} before it is rescaled
          if (pv_seen < j) {
            if (wait_all(&ctl->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, deadline, a.status, 36, j))
              pv_seen = j;
            else
              bad = true;
          }
          if (!bad) {
            tc::fence_after_sync();
#pragma unroll 1
            for (int m = 0; m < MT; ++m)
#pragma unroll
              for (int c = 0; c < NQ / 32; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(tm + C::COL_O + m * NQ + c * 32, o);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f_s[c * 32 + e]);
                tc::tmem_st32(tm + C::COL_O + m * NQ + c * 32, o);
              }
            tc::tmem_wait_st();
          }
        }
      }
      // P buffer j & 1 is free once PV_{j-2} is done
      if (!bad && j >= 2 && pv_seen < j - 1) {
        if (wait_all(&ctl->o_done[j & 1], ((j - 2) >> 1) & 1, abort_flag, deadline, a.status, 37, j))
          pv_seen = j - 1;
        else
          bad = true;
      }
      if (bad) continue;  // no arrival: the issuer's bounded wait sees the abort
      // P^T row n (query), key kl: 128-byte rows of 64 keys, 16-byte units swizzled by n % 8
      unsigned char* prow = sm + (sP - base) + (j & 1) * C::P_BUF + (kl >> 6) * C::P_CH + (kl & 7) * 2;
      const int unit = (kl & 63) >> 3;
#pragma unroll
      for (int n = 0; n < NQ; n += 4) {
        const float4 m4 = *reinterpret_cast<const float4*>(m_s + n);
        const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float p = tc::ex2(v[n + u] - (mm[u] == -INFINITY ? 0.f : mm[u]));
          l[n + u] += p;
          *reinterpret_cast<bf16*>(prow + (n + u) * 128 + ((unit ^ ((n + u) & 7)) << 4)) = __float2bfloat16_rn(p);
        }
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&ctl->p_ready[j & 1]);
    }
    {
      const bool fin = ok && !bad &&
                       wait_all(&ctl->o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, abort_flag, deadline,
                                a.status, 39, n_tiles);
      ok = !any128(!fin);
    }
    if (ok) {
      tc::fence_after_sync();
      // column sums over the 128 keys; thread kl < nvalid finishes column kl
#pragma unroll
      for (int c = 0; c < NQ / 32; ++c) {
        float x[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = l[c * 32 + e];
        red[q4 * NQ + c * 32 + lane] = reduce_columns<false>(x, lane);
      }
      sync128();
      const int64_t row0 = (int64_t)b * a.tokens;
      if (kl < NQ) {
        const float L = (red[kl] + red[NQ + kl]) + (red[2 * NQ + kl] + red[3 * NQ + kl]);
        f_s[kl] = L > 0.f ? 1.f / L : 0.f;
        if (kl < nvalid && !a.out) {
          const int64_t pr = ((row0 + kl / G) * a.Hq + g * G + kl % G) * a.n_splits + split;
          a.part_lse[pr] = L > 0.f ? m_s[kl] + __log2f(L) : -INFINITY;
        }
      }
      sync128();
      // O^T / sum: this thread's TMEM lane is value dim m * 128 + kl of block m
#pragma unroll 1
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int c = 0; c < NQ / 32; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(tm + C::COL_O + m * NQ + c * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int n = c * 32 + e;
            if (n < nvalid) {
              const int64_t hr = (row0 + n / G) * a.Hq + g * G + n % G;  // output row
              if (a.out)
                a.out[hr * D + m * 128 + kl] = __float2bfloat16_rn(__uint_as_float(o[e]) * f_s[n]);
              else
                a.part_o[(hr * a.n_splits + split) * D + m * 128 + kl] = __uint_as_float(o[e]) * f_s[n];
            }
          }
        }
    }
  }

  __syncwarp();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // loads still in flight must land before shared memory is released
    volatile int never = 0;
    const uint64_t dl = globaltimer_ns() + 200000000ull;
    if (ctl->q_issued && !ctl->q_consumed) mbar_wait_bounded_at(&ctl->q_full, 0, &never, dl, a.status, 40, 0, 0, 0);
    for (int s = 0; s < NSTAGE; ++s)
      if (ctl->issued[s] > ctl->consumed[s])
        mbar_wait_bounded_at(&ctl->full[s], (ctl->issued[s] - 1) & 1, &never, dl, a.status, 40, ctl->issued[s], s,
                             ctl->consumed[s]);
  }
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, int NQ, bool LOCAL>
cudaError_t launch_as(const CUtensorMap (&m)[5], const VArgs& v, int B, cudaStream_t st) {
  using C = VCfg<D, NQ, LOCAL>;
  cudaError_t e =
      cudaFuncSetAttribute(k_verify_tc<D, NQ, LOCAL>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  k_verify_tc<D, NQ, LOCAL><<<dim3(v.Hkv, B, v.n_splits), 192, C::SMEM, st>>>(m[0], m[1], m[2], m[3], m[4], v);
  return cudaGetLastError();
}

template <int D, int NQ>
cudaError_t launch_nq(const CUtensorMap (&m)[5], const VArgs& v, int B, cudaStream_t st) {
  return v.window > 0 ? launch_as<D, NQ, true>(m, v, B, st) : launch_as<D, NQ, false>(m, v, B, st);
}

}  // namespace

int verify_tc_rows(int Hq, int Hkv, int tokens, int D) {
  const int nq = (Hq / Hkv) * tokens;
  if (D != 256 && D != 512) return 0;
  return nq <= 32 ? 32 : nq <= 64 ? 64 : 0;
}

cudaError_t launch_verify_attn_tc(const VerifyAttnArgs& a, int B, int D, cudaStream_t st) {
  const int G = a.Hq / a.Hkv;
  const int NQ = verify_tc_rows(a.Hq, a.Hkv, a.tokens, D);
  if (NQ == 0 && a.window == 0) return launch_verify_attn_rows(a, B, D, st);  // more than 64 query rows
  if (NQ == 0 || a.tokens < 1 || a.chunk % BN || a.n_splits < 1 || G * a.tokens > NQ) return cudaErrorInvalidValue;
  if (a.window > 0 && (a.tokens > BN || !a.k_tail || !a.v_tail || a.cache_cap != a.window))
    return cudaErrorInvalidValue;
  const uint64_t E = 2;
  CUtensorMap maps[5];
  CUtensorMap &mq = maps[0], &mk = maps[1], &mv = maps[2];
  {
    // q_rot [B][tokens][Hq][D]: a box is the G heads of one KV head for every token
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)a.Hq, (uint64_t)a.tokens, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)D * E, (uint64_t)a.Hq * D * E, (uint64_t)a.tokens * a.Hq * D * E};
    const uint32_t box[4] = {64, (uint32_t)G, (uint32_t)a.tokens, 1};
    if (!make_map_bf16_4d(&mq, a.q_rot, dims, str, box)) return cudaErrorInvalidValue;
  }
  if (a.window > 0 && a.page_table) return cudaErrorInvalidValue;  // rings are not paged
  {
    // head-major views (d, row, head, page) of the cache (a page per
    // sequence when contiguous); boxes of 64 dims x 128 rows
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)a.page_size, (uint64_t)a.Hkv, (uint64_t)a.n_pages};
    const uint64_t strk[3] = {(uint64_t)a.k.stride_row * E, (uint64_t)a.k.stride_h * E, (uint64_t)a.k.stride_b * E};
    const uint64_t strv[3] = {(uint64_t)a.v.stride_row * E, (uint64_t)a.v.stride_h * E, (uint64_t)a.v.stride_b * E};
    const uint32_t box[4] = {64, (uint32_t)BN, 1, 1};
    if (!make_map_bf16_4d(&mk, a.k.ptr, dims, strk, box) || !make_map_bf16_4d(&mv, a.v.ptr, dims, strv, box))
      return cudaErrorInvalidValue;
  }
  if (a.window > 0) {
    // the new tokens' rows (d, head, token, b); boxes of 64 dims x 128 tokens
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)a.Hkv, (uint64_t)a.tokens, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)D * E, (uint64_t)a.Hkv * D * E, (uint64_t)a.tokens * a.Hkv * D * E};
    const uint32_t box[4] = {64, 1, (uint32_t)BN, 1};
    if (!make_map_bf16_4d(&maps[3], a.k_tail, dims, str, box) || !make_map_bf16_4d(&maps[4], a.v_tail, dims, str, box))
      return cudaErrorInvalidValue;
  } else {
    maps[3] = mk;
    maps[4] = mv;
  }
  VArgs v{};
  v.out = a.out;
  v.window = a.window;
  v.page_table = a.page_table;
  v.page_size = a.page_size;
  v.pages_per_seq = a.pages_per_seq;
  v.n_pages = a.n_pages;
  v.Hq = a.Hq;
  v.Hkv = a.Hkv;
  v.tokens = a.tokens;
  v.chunk = a.chunk;
  v.n_splits = a.n_splits;
  v.key_cap = a.cache_cap;
  v.seq_lens = a.seq_lens;
  v.part_o = a.part_o;
  v.part_lse = a.part_lse;
  v.status = a.status;
  v.wait_ns = a.wait_ns;
  v.drop_first_copy = a.drop_first_copy;
  if (D == 256) return NQ == 32 ? launch_nq<256, 32>(maps, v, B, st) : launch_nq<256, 64>(maps, v, B, st);
  return NQ == 32 ? launch_nq<512, 32>(maps, v, B, st) : launch_nq<512, 64>(maps, v, B, st);
}

}  // namespace hlg
