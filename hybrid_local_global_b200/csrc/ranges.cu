// ranges.cu -- debug view of the mask logic: the inclusive range and count of
// key positions each prefill query sees, from the same visible_range()
// the attention kernels use to choose key tiles and mask edge tiles.
#include "common.cuh"
#include "kernels.h"

namespace hlg {

namespace {

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

cudaError_t launch_visible_ranges(const int32_t* seq_lens_before, int B, int S, int window,
                                  int32_t* ranges, cudaStream_t st) {
  if (S <= 0 || B <= 0) return cudaSuccess;
  dim3 grid((S + 127) / 128, B);
  k_visible_ranges<<<grid, 128, 0, st>>>(seq_lens_before, S, window, ranges);
  return cudaGetLastError();
}

}  // namespace hlg
