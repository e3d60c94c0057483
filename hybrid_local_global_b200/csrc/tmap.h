// tmap.h -- host-side TMA tensor maps (prefill attention, int8 decode).
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "kernels.h"

namespace hlg {

// bf16 4-D map, dims innermost first, strides in bytes for dims 1..3,
// box[4], 128-byte swizzle, out-of-range elements read as zero. False when
// the driver entry point is missing or rejects the layout.
bool make_map_bf16_4d(CUtensorMap* m, const void* ptr, const uint64_t dims[4], const uint64_t strides[3],
                      const uint32_t box[4]);
// The same for a uint8 tensor (int8 KV codes); box[0] <= 128 bytes.
bool make_map_u8_4d(CUtensorMap* m, const void* ptr, const uint64_t dims[4], const uint64_t strides[3],
                    const uint32_t box[4]);

// The four maps of one prefill attention launch:
//   q, o  [B][S][Hq][D], box 64 dims x 1 head x q_rows x 1;
//   k     the K view, box 64 dims x k_rows keys;
//   v     the V view, box 64 dims x v_rows keys;
// the K/V views are [B][rows][Hkv][D] (kv_token_major) or [pages][Hkv][rows][D]
// (a cache: a.n_pages pages of key_rows_total rows; n_pages = B when contiguous).
bool make_prefill_maps(const PrefillAttnArgs& a, int B, int D, int key_rows_total, int kv_token_major,
                       uint32_t q_rows, uint32_t k_rows, uint32_t v_rows, CUtensorMap* mq, CUtensorMap* mk,
                       CUtensorMap* mv, CUtensorMap* mo);

}  // namespace hlg
