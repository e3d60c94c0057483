// tmap.cu -- host-side TMA tensor maps (prefill attention, int8 decode).
#include <cudaTypedefs.h>

#include <mutex>

#include "tmap.h"

namespace hlg {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_4d(CUtensorMap* m, CUtensorMapDataType type, const void* ptr, const uint64_t dims[4],
                 const uint64_t strides[3], const uint32_t box[4]) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gs[3] = {strides[0], strides[1], strides[2]};
  cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, type, 4, const_cast<void*>(ptr), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool make_map_bf16_4d(CUtensorMap* m, const void* ptr, const uint64_t dims[4], const uint64_t strides[3],
                      const uint32_t box[4]) {
  return make_map_4d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, dims, strides, box);
}

bool make_map_u8_4d(CUtensorMap* m, const void* ptr, const uint64_t dims[4], const uint64_t strides[3],
                    const uint32_t box[4]) {
  return make_map_4d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, ptr, dims, strides, box);
}

bool make_prefill_maps(const PrefillAttnArgs& a, int B, int D, int key_rows_total, int kv_token_major,
                       uint32_t q_rows, uint32_t k_rows, uint32_t v_rows, CUtensorMap* mq, CUtensorMap* mk,
                       CUtensorMap* mv, CUtensorMap* mo) {
  const uint64_t E = 2;
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)a.Hq, (uint64_t)a.S, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)D * E, (uint64_t)a.Hq * D * E, (uint64_t)a.S * a.Hq * D * E};
    const uint32_t box[4] = {64, 1, q_rows, 1};
    if (!make_map_bf16_4d(mq, a.q_rot, dims, str, box)) return false;
    if (!make_map_bf16_4d(mo, a.out, dims, str, box)) return false;
  }
  if (kv_token_major) {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)a.Hkv, (uint64_t)key_rows_total, (uint64_t)B};
    const uint64_t strk[3] = {(uint64_t)a.k.stride_h * E, (uint64_t)a.k.stride_row * E,
                              (uint64_t)a.k.stride_b * E};
    const uint64_t strv[3] = {(uint64_t)a.v.stride_h * E, (uint64_t)a.v.stride_row * E,
                              (uint64_t)a.v.stride_b * E};
    const uint32_t bk[4] = {64, 1, k_rows, 1}, bv[4] = {64, 1, v_rows, 1};
    return make_map_bf16_4d(mk, a.k.ptr, dims, strk, bk) && make_map_bf16_4d(mv, a.v.ptr, dims, strv, bv);
  }
  // head-major views are cache views: pages of key_rows_total rows (a
  // contiguous cache is n_pages = B pages of its capacity)
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)key_rows_total, (uint64_t)a.Hkv,
                            (uint64_t)(a.n_pages > 0 ? a.n_pages : B)};
  const uint64_t strk[3] = {(uint64_t)a.k.stride_row * E, (uint64_t)a.k.stride_h * E,
                            (uint64_t)a.k.stride_b * E};
  const uint64_t strv[3] = {(uint64_t)a.v.stride_row * E, (uint64_t)a.v.stride_h * E,
                            (uint64_t)a.v.stride_b * E};
  const uint32_t bk[4] = {64, k_rows, 1, 1}, bv[4] = {64, v_rows, 1, 1};
  return make_map_bf16_4d(mk, a.k.ptr, dims, strk, bk) && make_map_bf16_4d(mv, a.v.ptr, dims, strv, bv);
}

}  // namespace hlg
