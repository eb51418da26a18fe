// Device-side helpers shared by the libflux kernels (sm_100a).
//
// * SA visibility arithmetic: the key-block ranges of the streaming pattern (sink
//   blocks plus a local window of blocks, Table 6 / Figure 1 of the Flux Attention
//   paper).  sa_key_blocks is the one definition of the block indices; every other
//   use goes through it: visible_key_ranges (one query row: the decode split planner
//   and the prefill per-key mask), visible_key_ranges_rows (the union over a tile of
//   query rows: the prefill tile scheduler and its mask test) and flux_sa_block_ranges.
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
constexpr unsigned kStatusRingRoute = 0x8u;
constexpr unsigned kStatusLayout = 0x10u;
constexpr unsigned kStatusBounds = 0x20u;

// Bounds guards of the checked build (compiled with FLUX_CHECKED: libflux_checked.so).
// A guard whose condition fails records kStatusBounds in the status word and the access
// it guards is skipped; nothing traps.  In the plain build FLUX_IN_BOUNDS(...) is the
// constant true, the condition is not even evaluated, and the access runs as the
// host-side argument checks and the kernel's own logic allow.
#ifdef FLUX_CHECKED
#define FLUX_IN_BOUNDS(cond, status) ::flux::bounds_ok((cond), (status))
#else
#define FLUX_IN_BOUNDS(cond, status) true
#endif

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

// Visible keys of the query rows [t_min, t_max] taken together, as
// [0, hi0) U [lo1, t_max + 1).  Every key j in [t_min, t_max] is visible from row j
// itself (its own block is in its window), so only keys below t_min need a rule: the
// window start of a row never decreases with t, and a row whose window reaches back to
// the sink (lo1 == 0) makes every earlier row do the same, so the union is the first
// row's window joined with the last row's sink range.
__host__ __device__ __forceinline__ KeyRanges visible_key_ranges_rows(int t_min, int t_max, bool fa,
                                                                      int block, int sink,
                                                                      int window) {
  const KeyRanges first = visible_key_ranges(t_min, fa, block, sink, window);
  const KeyRanges last = visible_key_ranges(t_max, fa, block, sink, window);
  KeyRanges r;
  r.lo0 = 0;
  r.hi0 = first.lo1 == 0 ? 0 : last.hi0;
  r.lo1 = first.lo1;
  r.hi1 = t_max + 1;
  return r;
}

__device__ __forceinline__ bool route_is_fa(const uint32_t* fa_mask, int mask_words, int b,
                                            int layer) {
  uint32_t w = __ldg(fa_mask + (size_t)b * mask_words + (layer >> 5));
  return (w >> (layer & 31)) & 1u;
}

// ------------------------------------------------------------------ small utilities

__device__ __forceinline__ bool bounds_ok(bool cond, unsigned* status) {
  if (!cond) atomicOr(status, kStatusBounds);
  return cond;
}

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

// ------------------------------------------------------------------ packed fp32x2 (sm_100)

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for a pair of x <= 8 on the FMA pipe instead of the MUFU unit.  Argument
// reduction x = j + f with j = round(x) (the 1.5 * 2^23 rounding constant) and
// f in [-1/2, 1/2]; 2^f by a cubic whose coefficients were fitted here to 2^f on
// [-1/2, 1/2] by iteratively reweighted least squares on the relative error (Lawson's
// minimax algorithm), maximum relative error 7.5e-5 in fp32; 2^j is added to the
// exponent field.  x is clamped at -125 so that the result stays a normal number:
// inputs below that (masked keys) give 2^-125 instead of 0, which no bf16 P or fp32
// row sum can tell apart from 0 in a row that has a visible key.
__device__ __forceinline__ uint64_t exp2_poly_f2(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  const uint64_t round_c = f2_pack(12582912.f, 12582912.f);
  const uint64_t xc = f2_pack(x0, x1);
  const uint64_t t = f2_add(xc, round_c);              // low bits hold round(x)
  const uint64_t j = f2_add(t, f2_pack(-12582912.f, -12582912.f));
  const uint64_t f = f2_add(xc, j ^ 0x8000000080000000ull);  // x - round(x)
  uint64_t p = f2_fma(f2_pack(0.0551716685f, 0.0551716685f), f, f2_pack(0.2426111400f, 0.2426111400f));
  p = f2_fma(p, f, f2_pack(0.6932609677f, 0.6932609677f));
  p = f2_fma(p, f, f2_pack(0.9999280572f, 0.9999280572f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  return f2_pack(__int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23)),
                 __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23)));
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
// the timeout bit) if it does not within limit_ns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* status,
                                          unsigned long long limit_ns = kWaitLimitNs) {
#pragma unroll 1
  for (int i = 0; i < 16; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) {
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

// ------------------------------------------------------------------ dependent launch

// A kernel launched with programmatic stream serialisation may start while the
// kernel before it on the stream is still running.  pdl_wait() blocks until that
// kernel has completed and its memory is visible (a no-op for a normal launch);
// every such kernel calls it before touching global memory.  pdl_trigger() lets the
// next kernel on the stream be launched early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace flux
