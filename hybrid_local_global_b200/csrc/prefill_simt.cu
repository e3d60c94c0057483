// prefill_simt.cu -- first CUDA prefill attention (CUDA cores, fp32).
//
// out[b, i, h] = sum_j softmax_j(scale * <q~_i, k~_j>) v_j over the keys j
// visible to query i ("Gemma 4: End-to-End Architecture Walkthrough", 3a:
// window-limited on local layers, all preceding keys on global ones), KV
// head g = h / (Hq / Hkv) (3b: grouped-query attention). Online softmax in
// the log2 domain, fp32 throughout.
//
// CTA = 32 query rows of one (batch, q head); 8 warps x 4 rows; 32-key tiles
// staged in shared memory; lane j scores key j, then the warp accumulates
// P.V with lane l owning 8 (D=256) or 16 (D=512) output columns.
#include "common.cuh"
#include "kernels.h"

namespace hlg {

namespace {

constexpr int BM = 32, BN = 32, NWARP = 8, RPW = BM / NWARP;

template <int D>
__global__ void __launch_bounds__(256) k_prefill_attn_simt(PrefillAttnArgs a) {
  constexpr int KSTR = D + 8;   // padded K row (elements): conflict-free 16-byte reads
  constexpr int NC = D / 256;   // 8-column chunks per lane
  extern __shared__ __align__(16) unsigned char smem_raw[];
  bf16* qs = reinterpret_cast<bf16*>(smem_raw);
  bf16* ks = qs + BM * D;
  bf16* vs = ks + BN * KSTR;

  const int b = blockIdx.z, h = blockIdx.y, q0 = blockIdx.x * BM;
  const int g = h / (a.Hq / a.Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t pos0 = a.seq_lens_before ? (int64_t)a.seq_lens_before[b] : 0;
  const int64_t n_keys = pos0 + a.S;
  if (pos0 < 0 || n_keys > a.key_cap) return;  // reported by the RoPE kernel

  for (int idx = threadIdx.x; idx < BM * D / 8; idx += blockDim.x) {
    int r = idx / (D / 8), c = (idx % (D / 8)) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (q0 + r < a.S)
      v = *reinterpret_cast<const uint4*>(a.q_rot + (((int64_t)b * a.S + q0 + r) * a.Hq + h) * D + c);
    *reinterpret_cast<uint4*>(qs + r * D + c) = v;
  }

  int64_t lo_r[RPW], hi_r[RPW];
  float m[RPW], l[RPW], o[RPW][NC * 8];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    int row = q0 + warp * RPW + r;
    int64_t pos = pos0 + (row < a.S ? row : a.S - 1);
    visible_range(pos, a.window, n_keys, &lo_r[r], &hi_r[r]);
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int c = 0; c < NC * 8; ++c) o[r][c] = 0.f;
  }
  int64_t cta_lo, cta_hi;
  visible_range(pos0 + q0, a.window, n_keys, &cta_lo, &cta_hi);
  {
    int64_t l2, h2;
    visible_range(pos0 + min(q0 + BM - 1, a.S - 1), a.window, n_keys, &l2, &h2);
    cta_hi = h2;
  }

  for (int64_t kt = (cta_lo / BN) * BN; kt <= cta_hi; kt += BN) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < BN * D / 8; idx += blockDim.x) {
      int j = idx / (D / 8), c = (idx % (D / 8)) * 8;
      int64_t key = kt + j;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (key < n_keys) {
        kv = *reinterpret_cast<const uint4*>(a.k.ptr + b * a.k.stride_b + key * a.k.stride_row +
                                             g * a.k.stride_h + c);
        vv = *reinterpret_cast<const uint4*>(a.v.ptr + b * a.v.stride_b + key * a.v.stride_row +
                                             g * a.v.stride_h + c);
      }
      *reinterpret_cast<uint4*>(ks + j * KSTR + c) = kv;
      *reinterpret_cast<uint4*>(vs + j * D + c) = vv;
    }
    __syncthreads();

    // scores: lane scores key kt + lane for the warp's 4 rows
    float acc[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) acc[r] = 0.f;
    const bf16* krow = ks + lane * KSTR;
    for (int c = 0; c < D; c += 8) {
      uint4 kk = *reinterpret_cast<const uint4*>(krow + c);
      float2 k0 = unpack_bf16x2(kk.x), k1 = unpack_bf16x2(kk.y), k2 = unpack_bf16x2(kk.z),
             k3 = unpack_bf16x2(kk.w);
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        uint4 qq = *reinterpret_cast<const uint4*>(qs + (warp * RPW + r) * D + c);
        float2 x0 = unpack_bf16x2(qq.x), x1 = unpack_bf16x2(qq.y), x2 = unpack_bf16x2(qq.z),
               x3 = unpack_bf16x2(qq.w);
        acc[r] += x0.x * k0.x + x0.y * k0.y + x1.x * k1.x + x1.y * k1.y + x2.x * k2.x +
                  x2.y * k2.y + x3.x * k3.x + x3.y * k3.y;
      }
    }
    float p[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      int64_t key = kt + lane;
      float s = (key >= lo_r[r] && key <= hi_r[r]) ? acc[r] * a.scale_log2 : -INFINITY;
      float tmax = s;
#pragma unroll
      for (int off = 16; off; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      float m_new = fmaxf(m[r], tmax);
      float base = (m_new == -INFINITY) ? 0.f : m_new;
      float alpha = exp2f(m[r] - base);
      p[r] = exp2f(s - base);
      float psum = p[r];
#pragma unroll
      for (int off = 16; off; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      l[r] = l[r] * alpha + psum;
      m[r] = m_new;
#pragma unroll
      for (int c = 0; c < NC * 8; ++c) o[r][c] *= alpha;
    }
    for (int j = 0; j < BN; ++j) {
      float pj[RPW];
#pragma unroll
      for (int r = 0; r < RPW; ++r) pj[r] = __shfl_sync(0xffffffffu, p[r], j);
#pragma unroll
      for (int cc = 0; cc < NC; ++cc) {
        uint4 vv = *reinterpret_cast<const uint4*>(vs + j * D + cc * 256 + lane * 8);
        float2 v0 = unpack_bf16x2(vv.x), v1 = unpack_bf16x2(vv.y), v2 = unpack_bf16x2(vv.z),
               v3 = unpack_bf16x2(vv.w);
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          float* oo = &o[r][cc * 8];
          oo[0] += pj[r] * v0.x; oo[1] += pj[r] * v0.y;
          oo[2] += pj[r] * v1.x; oo[3] += pj[r] * v1.y;
          oo[4] += pj[r] * v2.x; oo[5] += pj[r] * v2.y;
          oo[6] += pj[r] * v3.x; oo[7] += pj[r] * v3.y;
        }
      }
    }
  }

#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    int row = q0 + warp * RPW + r;
    if (row >= a.S) continue;
    float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
    bf16* dst = a.out + (((int64_t)b * a.S + row) * a.Hq + h) * D;
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) {
      const float* oo = &o[r][cc * 8];
      uint4 w = make_uint4(pack_bf16x2(oo[0] * inv, oo[1] * inv), pack_bf16x2(oo[2] * inv, oo[3] * inv),
                           pack_bf16x2(oo[4] * inv, oo[5] * inv), pack_bf16x2(oo[6] * inv, oo[7] * inv));
      *reinterpret_cast<uint4*>(dst + cc * 256 + lane * 8) = w;
    }
    if (a.lse && lane == 0)
      a.lse[((int64_t)b * a.Hq + h) * a.S + row] =
          l[r] > 0.f ? (m[r] + log2f(l[r])) * 0.69314718055994530942f : -INFINITY;
  }
}

__global__ void k_visible_ranges(const int32_t* seq_lens_before, int S, int window, int32_t* out) {
  const int b = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= S) return;
  const int64_t pos0 = seq_lens_before ? (int64_t)seq_lens_before[b] : 0;
  int64_t lo, hi;
  int64_t cnt = visible_range(pos0 + i, window, pos0 + S, &lo, &hi);
  int32_t* o = out + ((int64_t)b * S + i) * 3;
  o[0] = (int32_t)lo;
  o[1] = (int32_t)hi;
  o[2] = (int32_t)cnt;
}

}  // namespace

cudaError_t launch_prefill_attn(const PrefillAttnArgs& a, int B, int D, cudaStream_t st) {
  dim3 grid((a.S + BM - 1) / BM, a.Hq, B);
  if (D == 256) {
    size_t sm = (size_t)(BM * 256 + BN * (256 + 8) + BN * 256) * 2;
    cudaFuncSetAttribute(k_prefill_attn_simt<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_prefill_attn_simt<256><<<grid, NWARP * 32, sm, st>>>(a);
  } else {
    size_t sm = (size_t)(BM * 512 + BN * (512 + 8) + BN * 512) * 2;
    cudaFuncSetAttribute(k_prefill_attn_simt<512>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_prefill_attn_simt<512><<<grid, NWARP * 32, sm, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_visible_ranges(const int32_t* seq_lens_before, int B, int S, int window,
                                  int32_t* ranges, cudaStream_t st) {
  if (S <= 0 || B <= 0) return cudaSuccess;
  dim3 grid((S + 127) / 128, B);
  k_visible_ranges<<<grid, 128, 0, st>>>(seq_lens_before, S, window, ranges);
  return cudaGetLastError();
}

}  // namespace hlg
