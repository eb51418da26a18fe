// Split-KV flash-decode for both routes of Flux Attention (Table 3: decode reuses the
// prefill route; Table 6: SA = sink + local window of KV blocks), sm_100a.
//
// One query token per sequence attends the keys of its route: FA reads the whole
// cache [0, seq_len), SA reads only the sink rows and the window rows.  Decode is
// bound by HBM bandwidth, so the kernel is built around moving K/V bytes, and one
// call is one kernel launch:
//
//  * the visible keys of each (sequence, KV head) pair are cut into 128-key stages;
//    all pairs' stages, laid end to end, are dealt to the persistent grid (one CTA
//    per SM) as equal contiguous ranges, so every CTA streams the same number of
//    stages (FA and SA pairs, ragged lengths alike) and closes a partial result only
//    where its range crosses a pair boundary -- one to three times per CTA at large
//    batch, instead of once per fixed-size split.  When there are no more pairs than
//    CTAs and streaming the longest pair whole costs less than splitting plus merging
//    (a streaming-rate model, below), each CTA takes one pair whole instead;
//  * one producer lane streams each piece's K and V rows -- contiguous in the
//    [B][Hkv][cap][d] cache -- into a 3-stage ring of 128-key stages with 1-D bulk
//    copies (cp.async.bulk, no cluster), completing on mbarriers; the group's query
//    rows ride along with the first stage of every piece;
//  * 8 consumer warps (16 keys each per stage) read the stage with 128-bit shared
//    loads: 8 lanes cover one key row (16 B each), 4 rows per warp instruction, all
//    G = Hq/Hkv query heads of the group at once, with packed fp32x2 FMAs; the q.k
//    partial sums are reduced across the 8 lanes with a transposing butterfly (each
//    level hands half of the remaining head sums to the partner lane);
//  * online softmax in the log2 domain per head; P.V accumulates in fp32 registers;
//  * a piece that covers its whole pair normalises and writes the bf16 output itself;
//    the pieces of a split pair write (running max, running sum, unnormalised
//    accumulator) per head to the workspace, and the CTA that finishes the pair's last
//    piece (an arrival counter in the workspace) merges them and writes the output;
//  * the appending variant (flux_decode_append) also takes the step's new K/V row:
//    the pair's newest key is streamed from k_new / v_new instead of the cache, the
//    CTA that holds it writes the row into the cache, and the last CTA to finish
//    reading the lengths (a second arrival counter) advances seq_len.
//
// The arrival counters live at fixed offsets at the start of the workspace, so they
// do not move with the geometry; every call leaves them at zero, and a workspace only
// has to be zero-filled once, before its first call.
#include <math.h>

#include <mutex>

#include "../../include/flux.h"
#include "flux_device.cuh"
#include "flux_internal.h"

// Scratch for flux_decode_static: the split partials and arrival counters that
// flux_decode keeps in the caller's workspace, held instead in a fixed array inside
// the library image.  Every GPU that loads the library reserves these bytes until the
// process exits; like every __device__ array without an initialiser it starts zeroed,
// which is the state the arrival counters need.  In host code this name is only a
// host-side stand-in: its device address comes from cudaGetSymbolAddress (see
// static_scratch_address below).
static __device__ __align__(256) unsigned char g_decode_static_scratch[FLUX_DECODE_STATIC_SCRATCH_BYTES];

namespace flux {
namespace {

constexpr int kStageKeys = kDecStageKeys;
constexpr int kMaxStages = 3;
constexpr int kConsumerWarps = 8;
// Three warpgroups: two of consumers (warps 0-7) and one whose first lane is the
// producer.  A block of 384 threads launches with 168 registers per thread (three
// warps per SM sub-partition); the producer warpgroup then gives most of its registers
// back (setmaxnreg.dec to kProducerRegs) and the consumers take them
// (setmaxnreg.inc to kConsumerRegs): 256 x 232 + 128 x 40 = 64512 = 384 x 168, the
// registers the block was launched with, so the increase never waits.  With 168 the
// consumers spilled.
constexpr int kThreads = 384;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 40;
constexpr int kConsumerRegs = 232;
static_assert(kConsumerThreads * kConsumerRegs + (kThreads - kConsumerThreads) * kProducerRegs <=
                  kThreads * kLaunchRegs,
              "register split above the launch allocation");
constexpr int kKeysPerWarp = kStageKeys / kConsumerWarps;  // 16 keys per warp per stage
constexpr int kPasses = kKeysPerWarp / 4;                  // 4 keys per warp instruction
static_assert(kPasses == 4, "the tile maximum below is written for 4 passes");
constexpr uint32_t kRouteFa = 0x80000000u;  // route bit of a per-sequence info word

struct DecodeArgs {
  const uint32_t* fa_mask;
  int mask_words, layer;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* k_new;  // appending variant: [B][1][Hkv][D]; otherwise null
  const uint16_t* v_new;
  int32_t* seq_len;       // written only by the appending variant
  int batch, capacity, hkv, block, sink, window;
  float scale_log2;  // log2(e) / sqrt(d)
  int ring_rows;     // 0: contiguous cache; > 0: SA ring cache of sink + ring_rows rows
  int rows;          // physical rows per (sequence, KV head)
  unsigned* ws_ctr;  // [kDecCtaCounters] split-pair arrivals, then the length arrival
  float* ws_acc;     // [B][Hkv][kDecMaxSplits][G][D]
  float2* ws_ml;     // [B][Hkv][kDecMaxSplits][G] = (max, sum)
  uint16_t* o;
  unsigned* status;
};

// The visible keys of a decode query at position T - 1 (T keys in the sequence,
// counting the appended one), flattened in position order and laid out in up to three
// physically contiguous pieces: [0, len0) (sink, or everything in a contiguous
// cache's merged case), then [start1, start1 + len1) and [start2, start2 + len2) (the
// window; two pieces when it wraps around a ring cache).
struct Plan {
  int n_vis, stages;
  int len0, start1, len1, start2;
};

__device__ __forceinline__ Plan make_plan(const DecodeArgs& a, int T, bool fa) {
  Plan p{0, 0, 0, 0, 0, 0};
  if (T <= 0) return p;
  const KeyRanges r = visible_key_ranges(T - 1, fa, a.block, a.sink, a.window);
  if (a.ring_rows == 0) {
    p.len0 = r.hi0 - r.lo0;
    p.start1 = r.lo1;
    p.len1 = r.hi1 - r.lo1;
  } else {
    // positions below the sink stay in place; position q >= sink lives in slot
    // sink + (q - sink) mod ring_rows
    const int R = a.ring_rows;
    if (r.lo1 == 0) {  // the window reaches key 0: keys [0, T), and T - sink <= window <= R
      p.len0 = min(T, a.sink);
      p.start1 = a.sink;
      p.len1 = max(0, T - a.sink);
    } else {
      p.len0 = r.hi0;
      const int L = r.hi1 - r.lo1;
      const int s0 = (r.lo1 - a.sink) % R;
      p.start1 = a.sink + s0;
      p.len1 = min(L, R - s0);
      p.start2 = a.sink;
    }
  }
  p.n_vis = (r.hi0 - r.lo0) + (r.hi1 - r.lo1);
  p.stages = (p.n_vis + kDecStageKeys - 1) / kDecStageKeys;
  return p;
}

// Physical row of position t (the appended key's destination).
__device__ __forceinline__ int physical_row(const DecodeArgs& a, int t) {
  if (a.ring_rows == 0 || t < a.sink) return t;
  return a.sink + (t - a.sink) % a.ring_rows;
}

// One CTA's piece of one pair: the pair's stages [k0, k1) (virtual keys [v0, v1)).
// split numbers the CTAs that share the pair, n_split counts them; first_cta is the
// CTA holding split 0 (it indexes the pair's arrival counter).
struct Item {
  int b, kvh, split, n_split, first_cta;
  int v0, v1;
  int seg_end;  // global stage index where this piece ends
  Plan p;
};

// The stage ranges: the pairs' stages laid end to end (sequence-major, then KV head),
// prefix[b] = stages of all pairs of sequences before b; CTA c owns global stages
// [c * per, (c + 1) * per).  per is at least ceil(max pair stages / 62), so a pair
// meets at most 63 <= kDecMaxSplits CTAs.
__device__ __forceinline__ int stages_per_cta(int total, int max_pair_stages) {
  const int even = (total + int(gridDim.x) - 1) / int(gridDim.x);
  const int cap = (max_pair_stages + kDecMaxSplits - 3) / (kDecMaxSplits - 2);
  return max(1, max(even, cap));
}

// Streaming-rate model the planner uses to choose between two ways of dealing the
// stages (constants measured on B200):
//  * split: equal contiguous stage ranges over the whole grid (above); pairs longer
//    than a range are cut, and their partial results are merged at the end;
//  * whole pairs: CTA p streams pair p from first key to last and writes the final
//    output itself; no partials, nothing to merge.
// A stage costs stage_bytes / kHbmBytesPerNs for every CTA streaming at the same time
// (HBM is shared), but at least stage_bytes / kCtaBytesPerNs (the rate one CTA's
// consumer warps sustain on their own); merging split partials adds about kMergeNs
// (partial writes, the arrival and the merging CTA's dependent reads).  Whole pairs
// win when the longest pair streams, at that rate, in less time than the even split
// plus the merge: e.g. 16 sequences at 32K context on the SA route (128 pairs of 17
// stages), not on the FA route or at 8 sequences.
constexpr float kHbmBytesPerNs = 6400.f;
constexpr float kCtaBytesPerNs = 48.f;
constexpr float kMergeNs = 3000.f;

__device__ __forceinline__ bool whole_pairs_pay(int total, int max_pair_stages, int n_pairs,
                                                int grid, float stage_bytes) {
  if (n_pairs > grid || max_pair_stages == 0) return false;
  const float solo = stage_bytes / kCtaBytesPerNs;
  const float t_pairs =
      float(max_pair_stages) * fmaxf(solo, float(n_pairs) * stage_bytes / kHbmBytesPerNs);
  const int per = stages_per_cta(total, max_pair_stages);
  const float t_split = float(per) * fmaxf(solo, float(grid) * stage_bytes / kHbmBytesPerNs) +
                        (per < max_pair_stages ? kMergeNs : 0.f);
  return t_pairs < t_split;
}

// Per-sequence word kept in shared memory: keys attended (T, counting an appended
// key; 0 = nothing to attend) | kRouteFa.  The kernel reads seq_len from global memory
// once, in its prologue: the appending variant rewrites it while the grid runs.
__device__ __forceinline__ Plan plan_of(const DecodeArgs& a, uint32_t info) {
  return make_plan(a, int(info & ~kRouteFa), (info & kRouteFa) != 0u);
}

// The piece that starts at global stage s of a range ending at end.
__device__ __forceinline__ Item item_at(const DecodeArgs& a, const int* prefix,
                                        const uint32_t* info, int s, int end, int per) {
  int lo = 0, hi = a.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= s) lo = mid; else hi = mid;
  }
  Item it;
  it.b = lo;
  it.p = plan_of(a, info[lo]);
  const int ns = it.p.stages;
  const int r = s - prefix[lo];
  it.kvh = r / ns;
  const int pair0 = prefix[lo] + it.kvh * ns;
  const int pair1 = pair0 + ns;
  it.seg_end = min(end, pair1);
  it.first_cta = pair0 / per;
  it.split = s / per - it.first_cta;
  it.n_split = (pair1 - 1) / per - it.first_cta + 1;
  it.v0 = (s - pair0) * kDecStageKeys;
  it.v1 = min(it.p.n_vis, (it.seg_end - pair0) * kDecStageKeys);
  return it;
}

// Stages cover consecutive virtual keys of the item, whatever physical pieces they
// come from, so a key's stage row (and hence the arithmetic) depends only on its place
// in the position order: a ring cache and a contiguous cache give identical results,
// and so do an appended key streamed from k_new and the same key read from the cache.
__device__ __forceinline__ int item_stages(const Item& it) {
  return (it.v1 - it.v0 + kStageKeys - 1) / kStageKeys;
}

__device__ __forceinline__ int stage_keys(const Item& it, int k) {
  return min(kStageKeys, it.v1 - it.v0 - k * kStageKeys);
}

// Physical runs of stage k: up to three (first physical row, count, stage row) triples
// read from the cache.  With an appended key (the pair's last virtual key, position
// T - 1) in the stage, that key is left out of the runs and new_dst is its stage row
// (it comes from k_new / v_new); otherwise new_dst = -1.
__device__ __forceinline__ int stage_runs(const Item& it, int k, bool append, int (&row)[3],
                                          int (&cnt)[3], int (&dst)[3], int& new_dst) {
  const int vs = it.v0 + k * kStageKeys;
  int ve = min(it.v1, vs + kStageKeys);
  new_dst = -1;
  if (append && ve == it.p.n_vis) {
    new_dst = ve - 1 - vs;
    --ve;
  }
  const int len2 = it.p.n_vis - it.p.len0 - it.p.len1;
  const int pvs[3] = {0, it.p.len0, it.p.len0 + it.p.len1};
  const int pln[3] = {it.p.len0, it.p.len1, len2};
  const int pst[3] = {0, it.p.start1, it.p.start2};
  int n = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int a0 = max(vs, pvs[i]);
    const int a1 = min(ve, pvs[i] + pln[i]);
    if (a1 > a0) {
      row[n] = pst[i] + (a0 - pvs[i]);
      cnt[n] = a1 - a0;
      dst[n] = a0 - vs;
      ++n;
    }
  }
  return n;
}

__device__ __forceinline__ uint4 lds128(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_addr(p)));
  return v;
}

// Sum G per-lane values over the 8 lanes of a key group (lane bits 0..2) so that each
// lane ends with the full sum of one value: head (c >> (3 - log2 G)), c = lane & 7.
// Each butterfly level hands half of the remaining values to the partner lane.
template <int G>
__device__ __forceinline__ float group_reduce(float (&v)[G], int lane) {
  if constexpr (G == 8) {
    const bool u2 = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = u2 ? v[i] : v[i + 4];
      const float keep = u2 ? v[i + 4] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    const bool u1 = lane & 2;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = u1 ? v[i] : v[i + 2];
      const float keep = u1 ? v[i + 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    const bool u0 = lane & 1;
    const float send = u0 ? v[0] : v[1];
    const float keep = u0 ? v[1] : v[0];
    return keep + __shfl_xor_sync(0xffffffffu, send, 1);
  } else if constexpr (G == 4) {
    const bool u2 = lane & 4;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = u2 ? v[i] : v[i + 2];
      const float keep = u2 ? v[i + 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    const bool u1 = lane & 2;
    const float send = u1 ? v[0] : v[1];
    const float keep = u1 ? v[1] : v[0];
    float r = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    return r + __shfl_xor_sync(0xffffffffu, r, 1);
  } else if constexpr (G == 2) {
    const bool u2 = lane & 4;
    const float send = u2 ? v[0] : v[1];
    const float keep = u2 ? v[1] : v[0];
    float r = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    return r + __shfl_xor_sync(0xffffffffu, r, 1);
  } else {
    float r = v[0];
    r += __shfl_xor_sync(0xffffffffu, r, 4);
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    return r + __shfl_xor_sync(0xffffffffu, r, 1);
  }
}

// bf16 pair (one 32-bit word) -> the two values as an fp32 pair, exactly.
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <int D, int G, int S>
struct DecodeSmemLayout {
  static constexpr int kStages = S;
  static constexpr size_t kv_stage = size_t(kStageKeys) * D;  // elements per stage
  static constexpr size_t q_slot = size_t(G) * D;              // elements per q slot
  static constexpr size_t off_k = 0;
  static constexpr size_t off_v = off_k + kStages * kv_stage * 2;
  static constexpr size_t off_q = off_v + kStages * kv_stage * 2;
  // P of the stage; the merge reuses it as float2 [kDecMaxSplits][G] (same size)
  static constexpr size_t off_p = off_q + kStages * q_slot * 2;
  static_assert(kConsumerWarps * kKeysPerWarp * 4 == kDecMaxSplits * 8, "merge scratch");
  static constexpr size_t off_acc = off_p + kConsumerWarps * kKeysPerWarp * G * 4;
  static constexpr size_t off_m = off_acc + size_t(kConsumerWarps) * G * D * 4;
  static constexpr size_t off_l = off_m + kConsumerWarps * G * 4;
  static constexpr size_t off_bar = (off_l + kConsumerWarps * G * 4 + 15) / 16 * 16;
  static constexpr size_t off_wmax = off_bar + 2 * kStages * 8;  // int per warp, 2 flags
  static constexpr size_t off_prefix = off_wmax + 16 * 4;
  static constexpr size_t off_info(int batch) { return off_prefix + size_t(batch + 1) * 4; }
  static constexpr size_t bytes(int batch) { return off_info(batch) + size_t(batch) * 4; }
};

// As many stages (up to 3) as fit in the 227 KB of a CTA with 1024-sequence tables:
// 3 for every geometry except d = 128 with 8 query heads per KV head.
template <int D, int G>
using DecodeSmem = DecodeSmemLayout<
    D, G, (DecodeSmemLayout<D, G, kMaxStages>::bytes(kDecMaxBatch) <= 227 * 1024) ? kMaxStages : 2>;

template <int D, int G, bool APPEND>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeArgs a) {
  using L = DecodeSmem<D, G>;
  constexpr int kStages = L::kStages;
  constexpr int NCH = D / 64;          // 16-byte chunks of a row per lane
  constexpr int GB = (G == 1) ? 0 : (G == 2) ? 1 : (G == 4) ? 2 : 3;
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* sK = reinterpret_cast<uint16_t*>(smem + L::off_k);
  uint16_t* sV = reinterpret_cast<uint16_t*>(smem + L::off_v);
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem + L::off_q);
  float* sP = reinterpret_cast<float*>(smem + L::off_p);
  float* sAcc = reinterpret_cast<float*>(smem + L::off_acc);
  float* sM = reinterpret_cast<float*>(smem + L::off_m);
  float* sL = reinterpret_cast<float*>(smem + L::off_l);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  int* prefix = reinterpret_cast<int*>(smem + L::off_prefix);
  uint32_t* info = reinterpret_cast<uint32_t*>(smem + L::off_info(a.batch));
  int* wmax = reinterpret_cast<int*>(smem + L::off_wmax);  // [0..11] warp maxima, [13, 15] flags

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + kStages);
  const int n_pairs = a.batch * a.hkv;
  pdl_trigger();  // the next kernel on the stream may be scheduled; it waits for this grid
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kConsumerWarps);
    }
    fence_barrier_init();
  }
  pdl_wait();  // seq_len, the caches and q may come from earlier kernels

  // Prologue: each sequence's length is read once; keys attended, route, stage counts,
  // then an exclusive scan (warp 0) and the largest pair.
  int my_max = 0;
  for (int b = tid; b < a.batch; b += kThreads) {
    const int T0 = a.seq_len[b];
    const bool fa = route_is_fa(a.fa_mask, a.mask_words, b, a.layer);
    const bool valid = T0 >= 0 && T0 <= a.capacity;
    const bool ring_fa = a.ring_rows > 0 && fa;  // a ring cache only holds what SA reads
    int T = 0;
    if (valid && !ring_fa) {
      if (!APPEND) {
        T = T0;
      } else if (T0 < a.capacity) {
        T = T0 + 1;
      } else if (blockIdx.x == 0) {
        atomicOr(a.status, kStatusCapacity);
      }
    }
    if (blockIdx.x == 0) {
      if (!valid) atomicOr(a.status, kStatusBadLength);
      if (ring_fa && (T0 > 0 || APPEND)) atomicOr(a.status, kStatusRingRoute);
    }
    info[b] = uint32_t(T) | (fa ? kRouteFa : 0u);
    const Plan p = make_plan(a, T, fa);
    prefix[b + 1] = a.hkv * p.stages;
    my_max = max(my_max, p.stages);
  }
  my_max = __reduce_max_sync(0xffffffffu, my_max);
  if (lane == 0) wmax[warp] = my_max;
  __syncthreads();
  if (warp == 0) {
    int running = 0;
    for (int base = 0; base < a.batch; base += 32) {
      const int i = base + lane;
      int v = (i < a.batch) ? prefix[i + 1] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += y;
      }
      if (i < a.batch) prefix[i + 1] = v + running;
      running += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) prefix[0] = 0;
    int m = 0;
    for (int w = 0; w < kThreads / 32; ++w) m = max(m, wmax[w]);
    if (lane == 0) wmax[15] = m;
  }
  __syncthreads();
  // sequences with nothing to attend get zeros, shared out over the grid
  for (int b = blockIdx.x; b < a.batch; b += gridDim.x) {
    if ((info[b] & ~kRouteFa) == 0u) {
      uint16_t* ob = a.o + size_t(b) * a.hkv * G * D;
      for (int i = tid; i < a.hkv * G * D; i += kThreads) ob[i] = 0;
    }
  }
  const int total = prefix[a.batch];
  int per, range0, range1;
  if (whole_pairs_pay(total, wmax[15], n_pairs, int(gridDim.x),
                      float(kStageKeys) * D * 2 * 2)) {
    // CTA p takes pair p whole: one item, split 0 of 1 (per larger than any range)
    per = 1 << 30;
    range0 = range1 = 0;
    if (int(blockIdx.x) < n_pairs) {
      const int b = int(blockIdx.x) / a.hkv, kvh = int(blockIdx.x) % a.hkv;
      const int ns = (prefix[b + 1] - prefix[b]) / a.hkv;
      range0 = prefix[b] + kvh * ns;
      range1 = range0 + ns;
    }
  } else {
    per = stages_per_cta(total, wmax[15]);
    range0 = min(total, int(blockIdx.x) * per);
    range1 = min(total, range0 + per);
  }
  const size_t row_elems = D;

  if (warp >= kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (APPEND && warp == kConsumerWarps + 1) {
      // Off the consumers' path: every thread of this CTA has read its lengths (before
      // the first barrier); the last CTA to arrive advances them (no CTA of this grid
      // reads seq_len again) and re-zeroes the counter.
      unsigned last = 0u;
      if (lane == 0) {
        last = atomicAdd(a.ws_ctr + kDecCtaCounters - 1, 1u) == gridDim.x - 1;
        if (last) a.ws_ctr[kDecCtaCounters - 1] = 0u;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        for (int b = lane; b < a.batch; b += 32) {
          const int T = int(info[b] & ~kRouteFa);
          if (T > 0) a.seq_len[b] = T;
        }
      }
    }
    if (warp == kConsumerWarps && lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int g = 0;
      bool ok = true;
      for (int sg = range0; sg < range1 && ok;) {
        const Item it = item_at(a, prefix, info, sg, range1, per);
        sg = it.seg_end;
        const size_t head_off = (size_t(it.b) * a.hkv + it.kvh) * a.rows * row_elems;
        const size_t pair_row = (size_t(it.b) * a.hkv + it.kvh) * D;  // q group / new row
        const int ns = item_stages(it);
        for (int k = 0; k < ns; ++k, ++g) {
          int row[3], cnt[3], dst[3], new_dst;
          const int runs = stage_runs(it, k, APPEND, row, cnt, dst, new_dst);
          const int st = g % kStages;
          const uint32_t ph = (g / kStages) & 1;
          if (!mbar_wait(empty0 + 8 * st, ph ^ 1, a.status)) { ok = false; break; }
          const uint32_t bytes = uint32_t(stage_keys(it, k)) * D * 2;
          const uint32_t qbytes = (k == 0) ? uint32_t(G * D * 2) : 0u;
          mbar_arrive_expect_tx(full0 + 8 * st, 2 * bytes + qbytes);
          if (k == 0 && FLUX_IN_BOUNDS(it.b < a.batch && it.kvh < a.hkv, a.status))
            bulk_g2s(smem_addr(sQ + st * L::q_slot), a.q + pair_row * G, qbytes, full0 + 8 * st, pol);
          for (int r = 0; r < runs; ++r) {
            const uint32_t rb = uint32_t(cnt[r]) * D * 2;
            const size_t src = head_off + size_t(row[r]) * row_elems;
            // (a skipped copy leaves its stage short: the consumers' wait then times out)
            if (!FLUX_IN_BOUNDS(row[r] >= 0 && row[r] + cnt[r] <= a.rows && dst[r] >= 0 &&
                                    dst[r] + cnt[r] <= kStageKeys,
                                a.status))
              continue;
            bulk_g2s(smem_addr(sK + st * L::kv_stage + size_t(dst[r]) * D), a.k + src, rb,
                     full0 + 8 * st, pol);
            bulk_g2s(smem_addr(sV + st * L::kv_stage + size_t(dst[r]) * D), a.v + src, rb,
                     full0 + 8 * st, pol);
          }
          if (APPEND && new_dst >= 0 && FLUX_IN_BOUNDS(new_dst < kStageKeys, a.status)) {
            bulk_g2s(smem_addr(sK + st * L::kv_stage + size_t(new_dst) * D), a.k_new + pair_row,
                     D * 2, full0 + 8 * st, pol);
            bulk_g2s(smem_addr(sV + st * L::kv_stage + size_t(new_dst) * D), a.v_new + pair_row,
                     D * 2, full0 + 8 * st, pol);
          }
        }
      }
      // never leave the CTA with copies in flight: wait for each stage's last fill
      for (int s = 0; s < kStages; ++s) {
        const int last = (g - 1 - s) >= 0 ? ((g - 1 - s) / kStages) * kStages + s : -1;
        if (last >= 0) mbar_wait(full0 + 8 * s, (last / kStages) & 1, a.status);
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsumerRegs));
  const int key_sub = lane >> 3;           // which of the 4 rows of a warp instruction
  const int c = lane & 7;                  // 16-byte chunk within the row
  const int hl = c >> (3 - GB);            // head this lane holds after group_reduce
  const bool owner = (c & ((1 << (3 - GB)) - 1)) == 0;
  const int group_lane0 = lane & 24;
  int* flag = wmax + 13;                   // merge flag, shared by the consumer warps
  int g = 0;
  bool ok = true;
  for (int sg = range0; sg < range1;) {
    const Item it = item_at(a, prefix, info, sg, range1, per);
    sg = it.seg_end;
    const int pair = it.b * a.hkv + it.kvh;
    uint64_t q2[G][4 * NCH];   // pre-scaled query pairs of this lane's 8*NCH dims
    uint64_t acc[G][4 * NCH];  // P.V pairs of this lane's dims
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 4 * NCH; ++i) acc[h][i] = 0ull;
    float m_run = -INFINITY, l_run = 0.f;

    const int ns = ok ? item_stages(it) : 0;
    for (int k = 0; k < ns; ++k, ++g) {
      const int n = stage_keys(it, k);
      const int st = g % kStages;
      const uint32_t ph = (g / kStages) & 1;
      if (!mbar_wait(full0 + 8 * st, ph, a.status)) { ok = false; break; }
      if (k == 0) {
        const uint64_t sc = f2_pack(a.scale_log2, a.scale_log2);
        const uint16_t* qs = sQ + st * L::q_slot;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            const uint4 raw = lds128(qs + h * D + ch * 64 + c * 8);
            q2[h][ch * 4 + 0] = f2_mul(bf16x2_to_f2(raw.x), sc);
            q2[h][ch * 4 + 1] = f2_mul(bf16x2_to_f2(raw.y), sc);
            q2[h][ch * 4 + 2] = f2_mul(bf16x2_to_f2(raw.z), sc);
            q2[h][ch * 4 + 3] = f2_mul(bf16x2_to_f2(raw.w), sc);
          }
      }
      const uint16_t* Ks = sK + st * L::kv_stage;
      const uint16_t* Vs = sV + st * L::kv_stage;

      float s[kPasses];
#pragma unroll
      for (int p = 0; p < kPasses; ++p) {
        const int key = warp * kKeysPerWarp + p * 4 + key_sub;
        // two accumulation chains per head (even / odd words) halve the dependent FMAs
        uint64_t dot2[G], dot2b[G];
#pragma unroll
        for (int h = 0; h < G; ++h) dot2[h] = dot2b[h] = 0ull;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          const uint4 raw = lds128(Ks + key * D + ch * 64 + c * 8);
          const uint64_t k0 = bf16x2_to_f2(raw.x), k1 = bf16x2_to_f2(raw.y);
          const uint64_t k2 = bf16x2_to_f2(raw.z), k3 = bf16x2_to_f2(raw.w);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            dot2[h] = f2_fma(q2[h][ch * 4 + 0], k0, dot2[h]);
            dot2b[h] = f2_fma(q2[h][ch * 4 + 1], k1, dot2b[h]);
            dot2[h] = f2_fma(q2[h][ch * 4 + 2], k2, dot2[h]);
            dot2b[h] = f2_fma(q2[h][ch * 4 + 3], k3, dot2b[h]);
          }
        }
        float dot[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float lo, hi;
          f2_unpack(f2_add(dot2[h], dot2b[h]), lo, hi);
          dot[h] = lo + hi;
        }
        const float r = group_reduce<G>(dot, lane);
        s[p] = (key < n) ? r : -INFINITY;
      }
      float mt = fmax3(s[0], s[1], s[2]);
      mt = fmaxf(mt, s[3]);
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
      const float m_new = fmaxf(m_run, mt);
      if (__any_sync(0xffffffffu, m_new > m_run)) {
        const float alpha = (m_new > m_run) ? ex2_mufu(m_run - m_new) : 1.f;
        l_run *= alpha;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float ah = __shfl_sync(0xffffffffu, alpha, group_lane0 | (h << (3 - GB)));
          const uint64_t ah2 = f2_pack(ah, ah);
#pragma unroll
          for (int i = 0; i < 4 * NCH; ++i) acc[h][i] = f2_mul(acc[h][i], ah2);
        }
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float* Pw = sP + warp * kKeysPerWarp * G;
#pragma unroll
      for (int p = 0; p < kPasses; ++p) {
        const float pr = ex2_mufu(s[p] - m_use);
        l_run += pr;
        if (owner) Pw[(p * 4 + key_sub) * G + hl] = pr;
      }
      __syncwarp();
#pragma unroll
      for (int p = 0; p < kPasses; ++p) {
        const int key = warp * kKeysPerWarp + p * 4 + key_sub;
        if (key < n) {
          uint64_t pw2[G];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float pw = Pw[(p * 4 + key_sub) * G + h];
            pw2[h] = f2_pack(pw, pw);
          }
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            const uint4 raw = lds128(Vs + key * D + ch * 64 + c * 8);
            const uint64_t v0 = bf16x2_to_f2(raw.x), v1 = bf16x2_to_f2(raw.y);
            const uint64_t v2 = bf16x2_to_f2(raw.z), v3 = bf16x2_to_f2(raw.w);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              acc[h][ch * 4 + 0] = f2_fma(pw2[h], v0, acc[h][ch * 4 + 0]);
              acc[h][ch * 4 + 1] = f2_fma(pw2[h], v1, acc[h][ch * 4 + 1]);
              acc[h][ch * 4 + 2] = f2_fma(pw2[h], v2, acc[h][ch * 4 + 2]);
              acc[h][ch * 4 + 3] = f2_fma(pw2[h], v3, acc[h][ch * 4 + 3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
    }
    // A piece whose pipeline wait timed out still takes part in its pair's arrival
    // below (its partial is garbage, the status word says so), so the counters return
    // to zero as in every call.

    // reduce the 4 row groups of the warp, then the 8 warps through shared memory
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 4 * NCH; ++i) {
        float lo, hi;
        f2_unpack(acc[h][i], lo, hi);
        lo += __shfl_xor_sync(0xffffffffu, lo, 8);
        hi += __shfl_xor_sync(0xffffffffu, hi, 8);
        lo += __shfl_xor_sync(0xffffffffu, lo, 16);
        hi += __shfl_xor_sync(0xffffffffu, hi, 16);
        acc[h][i] = f2_pack(lo, hi);
      }
    if (key_sub == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          float f[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) f2_unpack(acc[h][ch * 4 + i], f[2 * i], f[2 * i + 1]);
          float4* dst = reinterpret_cast<float4*>(sAcc + (warp * G + h) * D + ch * 64 + c * 8);
          dst[0] = make_float4(f[0], f[1], f[2], f[3]);
          dst[1] = make_float4(f[4], f[5], f[6], f[7]);
        }
      if (owner) {
        sM[warp * G + hl] = m_run;
        sL[warp * G + hl] = l_run;
      }
    }
    named_barrier_sync(1, kConsumerThreads);
    uint16_t* out = a.o + size_t(pair) * G * D;
    const size_t rec0 = size_t(pair) * kDecMaxSplits;
    for (int i = tid; i < G * D; i += kConsumerThreads) {
      const int h = i / D, e = i % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sM[w * G + h]);
      float av = 0.f, lv = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = sM[w * G + h];
        const float f = (mw == -INFINITY) ? 0.f : ex2_mufu(mw - M);
        av = fmaf(f, sAcc[(w * G + h) * D + e], av);
        lv = fmaf(f, sL[w * G + h], lv);
      }
      if (it.n_split == 1) {
        const float inv = (lv > 0.f) ? 1.f / lv : 0.f;
        const __nv_bfloat16 hb = __float2bfloat16_rn(inv * av);
        out[i] = *reinterpret_cast<const uint16_t*>(&hb);
      } else {
        if (FLUX_IN_BOUNDS(it.split < kDecMaxSplits, a.status)) {
          a.ws_acc[(rec0 + it.split) * G * D + i] = av;
          if (e == 0) a.ws_ml[(rec0 + it.split) * G + h] = make_float2(M, lv);
        }
      }
    }
    const int new_row = physical_row(a, it.p.n_vis == 0 ? 0 : int(info[it.b] & ~kRouteFa) - 1);
    if (APPEND && it.v1 == it.p.n_vis &&
        FLUX_IN_BOUNDS(new_row >= 0 && new_row < a.rows, a.status)) {
      // this piece holds the pair's newest key: write its row into the cache
      const size_t dst = ((size_t(it.b) * a.hkv + it.kvh) * a.rows + new_row) * D;
      const size_t src = size_t(pair) * D;
      for (int i = tid; i < 2 * D / 8; i += kConsumerThreads) {
        const bool is_v = i >= D / 8;
        const int ch = is_v ? i - D / 8 : i;
        const uint4 x = __ldg(reinterpret_cast<const uint4*>((is_v ? a.v_new : a.k_new) + src) + ch);
        // the appending entry points take the caches as writable buffers
        reinterpret_cast<uint4*>(const_cast<uint16_t*>(is_v ? a.v : a.k) + dst)[ch] = x;
      }
    }
    if (it.n_split > 1 && FLUX_IN_BOUNDS(it.first_cta < kDecCtaCounters - 1 &&
                                             it.n_split <= kDecMaxSplits,
                                         a.status)) {
      // publish this piece's partial, then count it; the pair's last piece merges
      __threadfence();
      named_barrier_sync(1, kConsumerThreads);
      if (tid == 0) {
        const unsigned old = atomicAdd(a.ws_ctr + it.first_cta, 1u);
        const bool last = old == unsigned(it.n_split - 1);
        if (last) a.ws_ctr[it.first_cta] = 0u;  // back to zero for the next call
        *flag = last;
      }
      named_barrier_sync(1, kConsumerThreads);
      if (*flag) {
        __threadfence();
        const int nsp = it.n_split;
        float2* wml = reinterpret_cast<float2*>(sP);  // [kDecMaxSplits][G]: (max, sum)
        for (int i = tid; i < nsp * G; i += kConsumerThreads) wml[i] = __ldcg(a.ws_ml + rec0 * G + i);
        named_barrier_sync(1, kConsumerThreads);
        if (warp < G) {
          // one warp per query head: splits over the lanes; weights 2^(m_s - M) / L
          const int h = warp;
          float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
          if (lane < nsp) { m0 = wml[lane * G + h].x; l0 = wml[lane * G + h].y; }
          if (lane + 32 < nsp) { m1 = wml[(lane + 32) * G + h].x; l1 = wml[(lane + 32) * G + h].y; }
          float M = fmaxf(m0, m1);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
          const float f0 = (lane < nsp && m0 != -INFINITY) ? ex2_mufu(m0 - M) : 0.f;
          const float f1 = (lane + 32 < nsp && m1 != -INFINITY) ? ex2_mufu(m1 - M) : 0.f;
          float lv = f0 * l0 + f1 * l1;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) lv += __shfl_xor_sync(0xffffffffu, lv, off);
          const float inv = (lv > 0.f) ? 1.f / lv : 0.f;
          __syncwarp();
          if (lane < nsp) wml[lane * G + h].x = f0 * inv;
          if (lane + 32 < nsp) wml[(lane + 32) * G + h].x = f1 * inv;
        }
        named_barrier_sync(1, kConsumerThreads);
        for (int i = tid; i < G * D; i += kConsumerThreads) {
          const int h = i / D;
          const float* src = a.ws_acc + rec0 * G * D + i;
          float av0 = 0.f, av1 = 0.f;
          int sp = 0;
          for (; sp + 2 <= nsp; sp += 2) {
            av0 = fmaf(wml[sp * G + h].x, __ldcg(src + size_t(sp) * G * D), av0);
            av1 = fmaf(wml[(sp + 1) * G + h].x, __ldcg(src + size_t(sp + 1) * G * D), av1);
          }
          if (sp < nsp) av0 = fmaf(wml[sp * G + h].x, __ldcg(src + size_t(sp) * G * D), av0);
          const __nv_bfloat16 hb = __float2bfloat16_rn(av0 + av1);
          out[i] = *reinterpret_cast<const uint16_t*>(&hb);
        }
      }
    }
    named_barrier_sync(1, kConsumerThreads);  // sAcc, sM, sL, sP free for the next item
  }
}

template <int D, int G, bool APPEND>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  using L = DecodeSmem<D, G>;
  const size_t smem = L::bytes(a.batch);
  // the attribute is per device; set it (to the largest size any batch needs) once.
  // Host threads may make their first call on a device concurrently: the flag is
  // read and written under a lock.
  static std::mutex attr_mutex;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(attr_mutex);
    if (!attr_set[dev]) {
      err = cudaFuncSetAttribute(decode_kernel<D, G, APPEND>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(L::bytes(kDecMaxBatch)));
      if (err != cudaSuccess) return err;
      attr_set[dev] = true;
    }
  }
  const int grid = device_sm_count();
  if (grid > kDecCtaCounters - 1) return cudaErrorInvalidConfiguration;
  return launch_pdl(decode_kernel<D, G, APPEND>, dim3(grid), dim3(kThreads), smem, stream, a);
}

constexpr int kMaxDevices = 64;
std::mutex g_static_mutex;
void* g_static_address[kMaxDevices] = {};

// Device address of the static scratch on the current device.  Looked up once per
// device (with that device current) on its first use and cached.
cudaError_t static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_address[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_decode_static_scratch);
    if (err != cudaSuccess) return err;
    g_static_address[dev] = p;
  }
  *out = g_static_address[dev];
  return cudaSuccess;
}

}  // namespace

size_t decode_workspace_bytes(const AttnGeom& g, int batch) {
  const int G = g.hq / g.hkv;
  const size_t recs = size_t(batch) * g.hkv * kDecMaxSplits * G;
  const size_t acc = (recs * g.head_dim * 4 + 255) / 256 * 256;
  return kDecCounterBytes + acc + recs * 8;
}

cudaError_t launch_decode(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                          const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                          const uint16_t* k_new, const uint16_t* v_new, int32_t* seq_len,
                          int batch, int capacity, int ring_rows, uint16_t* o, void* workspace,
                          unsigned* status, cudaStream_t stream) {
  const int G = g.hq / g.hkv;
  DecodeArgs a;
  a.fa_mask = fa_mask;
  a.mask_words = g.mask_words;
  a.layer = layer;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.k_new = k_new;
  a.v_new = v_new;
  a.seq_len = seq_len;
  a.batch = batch;
  a.ring_rows = ring_rows;
  a.rows = ring_rows > 0 ? g.sink + ring_rows : capacity;
  a.capacity = ring_rows > 0 ? 0x7fffffff : capacity;  // a ring never runs out of rows
  a.hkv = g.hkv;
  a.block = g.block;
  a.sink = g.sink;
  a.window = g.window;
  a.scale_log2 = float(1.4426950408889634 / sqrt(double(g.head_dim)));
  const size_t recs = size_t(batch) * g.hkv * kDecMaxSplits * G;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.ws_ctr = reinterpret_cast<unsigned*>(ws);
  a.ws_acc = reinterpret_cast<float*>(ws + kDecCounterBytes);
  const size_t acc_bytes = (recs * g.head_dim * 4 + 255) / 256 * 256;
  a.ws_ml = reinterpret_cast<float2*>(ws + kDecCounterBytes + acc_bytes);
  a.o = o;
  a.status = status;
  const bool append = k_new != nullptr;
#define FLUX_DECODE_CASE(DD, GG)                                                   \
  if (g.head_dim == DD && G == GG)                                                 \
    return append ? launch_decode_t<DD, GG, true>(a, stream)                       \
                  : launch_decode_t<DD, GG, false>(a, stream);
  FLUX_DECODE_CASE(128, 1)
  FLUX_DECODE_CASE(128, 2)
  FLUX_DECODE_CASE(128, 4)
  FLUX_DECODE_CASE(128, 8)
  FLUX_DECODE_CASE(64, 1)
  FLUX_DECODE_CASE(64, 2)
  FLUX_DECODE_CASE(64, 4)
  FLUX_DECODE_CASE(64, 8)
#undef FLUX_DECODE_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_static(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                                 const uint16_t* q, const uint16_t* k_cache,
                                 const uint16_t* v_cache, const int32_t* seq_len, int batch,
                                 int capacity, uint16_t* o, unsigned* status,
                                 cudaStream_t stream) {
  // The array starts zeroed and every call leaves its arrival counters at zero; the
  // partial records need no clearing (each is written before it is read).
  void* scratch = nullptr;
  const cudaError_t err = static_scratch_address(&scratch);
  if (err != cudaSuccess) return err;
  return launch_decode(g, layer, fa_mask, q, k_cache, v_cache, nullptr, nullptr,
                       const_cast<int32_t*>(seq_len), batch, capacity, 0, o, scratch, status,
                       stream);
}

}  // namespace flux
