// common.cuh -- device helpers shared by the kernels of libgemma_attn.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gemma_attn.h"

namespace hlg {

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------------------
// Visibility rule ("Gemma 4: End-to-End Architecture Walkthrough", 3a): the
// query at absolute position pos sees key j iff j <= pos and, on a local
// layer, j > pos - window. Keys 0..n_keys-1 exist. Writes the inclusive
// range and returns its size (0 when empty). Used by every kernel that
// decides which keys a query reads, and by gemma_attn_visible_ranges.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t visible_range(int64_t pos, int window,
                                                          int64_t n_keys, int64_t* lo,
                                                          int64_t* hi) {
  int64_t a = (window > 0 && pos - window + 1 > 0) ? pos - window + 1 : 0;
  int64_t b = pos < n_keys - 1 ? pos : n_keys - 1;
  *lo = a;
  *hi = b;
  return b >= a ? b - a + 1 : 0;
}

// Cache addressing. A layer's cache is a pool of pages [n_pages][Hkv][ps][D];
// position (or ring slot) p of sequence b lives at row p % ps of page
// table[b * pps + p / ps]. A contiguous cache [B][Hkv][cap][D] is the case
// table == null: page b, ps = cap. Returns the row index into the pool
// (in units of D elements), or -1 when the page index is outside the pool.
// Positions are below the int capacity, so pages take 32-bit division; a
// contiguous cache takes none (this sits on the decode producer's path).
__host__ __device__ __forceinline__ int64_t cache_row(const int32_t* table, int pps, int ps, int n_pages,
                                                      int Hkv, int b, int h, int64_t p) {
  if (!table) return ((int64_t)b * Hkv + h) * ps + p;
  const int pi = (int)p / ps;
  const int64_t page = table[(int64_t)b * pps + pi];
  if (page < 0 || page >= n_pages) return -1;
  return (page * Hkv + h) * ps + ((int)p - pi * ps);
}

// Number of rotated pairs under (p-)RoPE: floor(rope_frac * head_dim / 2).
__host__ __forceinline__ int rope_rotated_pairs(int head_dim, float rope_frac) {
  double v = (double)rope_frac * (double)(head_dim / 2);
  int n = (int)v;
  if ((double)n > v) --n;
  return n;
}

// ---------------------------------------------------------------------------
// Device status word: kernels record failures here instead of trapping.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// mbarrier (shared::cta) helpers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Device status block: one per device, owned by the library (api.cu). The
// `int* status` every kernel receives points at its first member.
struct DevStatus {
  int status;                   // first failure code since the last sync_status
  int timeout_claim;            // set by the first bounded wait that gave up
  unsigned long long info[8];   // {1, where, a, b, c, barrier word, block id, parity}
};

__device__ __forceinline__ void record_timeout(int* status, uint64_t* bar, uint32_t parity, int where,
                                               int a, int b, int c) {
  if (!status) return;
  DevStatus* d = reinterpret_cast<DevStatus*>(status);
  if (atomicCAS(&d->timeout_claim, 0, 1) == 0) {
    unsigned long long word;
    asm volatile("ld.shared.b64 %0, [%1];" : "=l"(word) : "r"((uint32_t)__cvta_generic_to_shared(bar)));
    d->info[0] = 1;
    d->info[1] = (unsigned long long)(long long)where;
    d->info[2] = (unsigned long long)(long long)a;
    d->info[3] = (unsigned long long)(long long)b;
    d->info[4] = (unsigned long long)(long long)c;
    d->info[5] = word;
    d->info[6] = (unsigned long long)blockIdx.x | ((unsigned long long)blockIdx.y << 20) |
                 ((unsigned long long)blockIdx.z << 40);
    d->info[7] = parity;
  }
}

// Bounded wait: polls until the phase with `parity` completes, until another
// thread of the CTA raised *abort, or until deadline_ns of %globaltimer has
// passed; on the deadline it raises *abort and records TIMEOUT. Returns true
// only when the phase completed.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded_at(uint64_t* bar, uint32_t parity,
                                                     volatile int* abort_flag, uint64_t deadline_ns,
                                                     int* status, int where, int a, int b, int c) {
  // a phase that has already completed: the non-blocking test answers
  // sooner than try_wait (measured on the MMA issue path)
  if (mbar_test_wait(bar, parity)) return true;
  uint32_t it = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++it & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() > deadline_ns) {
        *abort_flag = 1;
        set_status(status, GEMMA_ERR_DEVICE_TIMEOUT);
        record_timeout(status, bar, parity, where, a, b, c);
        return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag,
                                                  uint64_t deadline_ns, int* status) {
  return mbar_wait_bounded_at(bar, parity, abort_flag, deadline_ns, status, -1, 0, 0, 0);
}

// 1-D bulk copy global -> shared, completion signalled as tx bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// bf16 packing helpers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

}  // namespace hlg
