// Device-side helpers shared by the libflux kernels (sm_100a).
//
// * SA visibility arithmetic: the key-block ranges of the streaming pattern (sink
//   blocks plus a local window of blocks, Table 6 / Figure 1 of the Flux Attention
//   paper), used by the prefill tile scheduler, the decode split planner and
//   flux_sa_block_ranges alike, so that one function defines the block indices.
// * mbarrier / bulk-copy wrappers (inline PTX) with bounded waits: a wait that runs
//   past its time limit records FLUX_DEVICE_TIMEOUT in the status word and returns
//   false instead of spinning forever or trapping.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace flux {

constexpr unsigned kStatusCapacity = 0x1u;
constexpr unsigned kStatusTimeout = 0x2u;
constexpr unsigned kStatusBadLength = 0x4u;

// A pipeline wait gives up after this long (nanoseconds of %globaltimer).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// ------------------------------------------------------------------ SA geometry

// Visible key blocks of query block qb: [0, sink_end) U [win_begin, win_end).
// When the window reaches back to the sink the two merge and sink_end = 0.
struct BlockRanges {
  int sink_end, win_begin, win_end;
};

__host__ __device__ __forceinline__ BlockRanges sa_key_blocks(int qb, int n_sink_blocks,
                                                              int n_win_blocks) {
  int win_begin = qb - n_win_blocks + 1;
  if (win_begin < 0) win_begin = 0;
  int sink_end = n_sink_blocks < qb + 1 ? n_sink_blocks : qb + 1;
  BlockRanges r;
  if (win_begin <= sink_end) {
    r.sink_end = 0;
    r.win_begin = 0;
  } else {
    r.sink_end = sink_end;
    r.win_begin = win_begin;
  }
  r.win_end = qb + 1;
  return r;
}

// Visible keys of query position t as two half-open position ranges
// [lo0, hi0) U [lo1, hi1) (lo0 = 0; the first range may be empty).
struct KeyRanges {
  int lo0, hi0, lo1, hi1;
};

__host__ __device__ __forceinline__ KeyRanges visible_key_ranges(int t, bool fa, int block,
                                                                 int sink, int window) {
  KeyRanges r;
  r.lo0 = 0;
  if (fa) {
    r.hi0 = 0;
    r.lo1 = 0;
    r.hi1 = t + 1;
    return r;
  }
  BlockRanges br = sa_key_blocks(t / block, sink / block, window / block);
  r.hi0 = br.sink_end * block;
  r.lo1 = br.win_begin * block;
  r.hi1 = t + 1;
  return r;
}

__device__ __forceinline__ bool route_is_fa(const uint32_t* fa_mask, int mask_words, int b,
                                            int layer) {
  uint32_t w = __ldg(fa_mask + (size_t)b * mask_words + (layer >> 5));
  return (w >> (layer & 31)) & 1u;
}

// ------------------------------------------------------------------ small utilities

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void bf16x8_to_float(const uint4& v, float (&f)[8]) {
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xffff0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xffff0000u);
  f[4] = __uint_as_float(v.z << 16);
  f[5] = __uint_as_float(v.z & 0xffff0000u);
  f[6] = __uint_as_float(v.w << 16);
  f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false (and sets
// the timeout bit) if it does not within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* status) {
#pragma unroll 1
  for (int i = 0; i < 16; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}

// ------------------------------------------------------------------ bulk copies

// 1-D bulk copy global -> shared (this CTA), completing on an mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void named_barrier_sync(int id, int n_threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n_threads) : "memory");
}

}  // namespace flux
