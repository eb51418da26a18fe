// Split-KV flash-decode for both routes of Flux Attention (Table 3: decode reuses the
// prefill route; Table 6: SA = sink + local window of KV blocks), sm_100a.
//
// One query token per sequence attends the keys of its route: FA reads the whole
// cache [0, seq_len), SA reads only the sink rows and the window rows.  Decode is
// bound by HBM bandwidth, so the kernel is built around moving K/V bytes:
//
//  * the visible keys of each (sequence, KV head) pair are cut into 128-key stages;
//    all pairs' stages, laid end to end, are dealt to the persistent grid (one CTA
//    per SM) as equal contiguous ranges, so every CTA streams the same number of
//    stages (FA and SA pairs, ragged lengths alike) and closes a partial result only
//    where its range crosses a pair boundary -- one to three times per CTA at large
//    batch, instead of once per fixed-size split;
//  * one producer lane streams each split's K and V rows -- contiguous in the
//    [B][Hkv][cap][d] cache -- into a 3-stage ring of 128-key stages with 1-D bulk
//    copies (cp.async.bulk, no cluster), completing on mbarriers; the group's query
//    rows ride along with the first stage of every split;
//  * 8 consumer warps (16 keys each per stage) read the stage with 128-bit shared
//    loads: 8 lanes cover one key row (16 B each), 4 rows per warp instruction, all
//    G = Hq/Hkv query heads of the group at once, with packed fp32x2 FMAs; the q.k
//    partial sums are reduced across the 8 lanes with a transposing butterfly (each
//    level hands half of the remaining head sums to the partner lane);
//  * online softmax in the log2 domain per head; P.V accumulates in fp32 registers;
//  * each item writes (running max, running sum, unnormalised accumulator) per head
//    to the caller's workspace; a combine kernel merges the splits and writes bf16.
#include <math.h>

#include <mutex>

#include "../../include/flux.h"
#include "flux_device.cuh"
#include "flux_internal.h"

// Scratch for flux_decode_static: the split partials that flux_decode keeps in the
// caller's workspace, held instead in a fixed array inside the library image.  Every
// GPU that loads the library reserves these bytes until the process exits.  In host
// code this name is only a host-side stand-in: its device address comes from
// cudaGetSymbolAddress (see static_scratch_address below).
static __device__ __align__(256) unsigned char g_decode_static_scratch[FLUX_DECODE_STATIC_SCRATCH_BYTES];

namespace flux {
namespace {

constexpr int kStageKeys = kDecStageKeys;
constexpr int kMaxStages = 3;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kKeysPerWarp = kStageKeys / kConsumerWarps;  // 16 keys per warp per stage
constexpr int kPasses = kKeysPerWarp / 4;                  // 4 keys per warp instruction
static_assert(kPasses == 4, "the tile maximum below is written for 4 passes");

struct DecodeArgs {
  const uint32_t* fa_mask;
  int mask_words, layer;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* seq_len;
  int batch, capacity, hkv, block, sink, window;
  float scale_log2;  // log2(e) / sqrt(d)
  int ring_rows;     // 0: contiguous cache; > 0: SA ring cache of sink + ring_rows rows
  int rows;          // physical rows per (sequence, KV head)
  float* ws_acc;     // [B][Hkv][kDecMaxSplits][G][D]
  float2* ws_ml;     // [B][Hkv][kDecMaxSplits][G] = (max, sum)
  int* ws_nsplit;    // [B][Hkv]: partial results written for the pair
  uint16_t* o;
  unsigned* status;
};

// The visible keys of sequence b's decode query, flattened in position order and laid
// out in up to three physically contiguous pieces: [0, len0) (sink, or everything in a
// contiguous cache's merged case), then [start1, start1 + len1) and
// [start2, start2 + len2) (the window; two pieces when it wraps around a ring cache).
struct Plan {
  int n_vis, stages;
  int len0, start1, len1, start2;
};

__device__ __forceinline__ Plan make_plan(const DecodeArgs& a, int b) {
  Plan p{0, 0, 0, 0, 0, 0};
  const int T = a.seq_len[b];
  if (T <= 0 || T > a.capacity) return p;
  const bool fa = route_is_fa(a.fa_mask, a.mask_words, b, a.layer);
  if (a.ring_rows > 0 && fa) return p;  // a ring cache only holds what SA reads
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

// One CTA's piece of one pair: the pair's stages [k0, k1) (virtual keys [v0, v1)).
// split numbers the CTAs that share the pair, n_split counts them.
struct Item {
  int b, kvh, split, n_split;
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

// The piece that starts at global stage s of a range ending at end.
__device__ __forceinline__ Item item_at(const DecodeArgs& a, const int* prefix, int s, int end,
                                        int per) {
  int lo = 0, hi = a.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= s) lo = mid; else hi = mid;
  }
  Item it;
  it.b = lo;
  it.p = make_plan(a, lo);
  const int ns = it.p.stages;
  const int r = s - prefix[lo];
  it.kvh = r / ns;
  const int pair0 = prefix[lo] + it.kvh * ns;
  const int pair1 = pair0 + ns;
  it.seg_end = min(end, pair1);
  it.split = s / per - pair0 / per;
  it.n_split = (pair1 - 1) / per - pair0 / per + 1;
  it.v0 = (s - pair0) * kDecStageKeys;
  it.v1 = min(it.p.n_vis, (it.seg_end - pair0) * kDecStageKeys);
  return it;
}

// Stages cover consecutive virtual keys of the item, whatever physical pieces they
// come from, so a key's stage row (and hence the arithmetic) depends only on its place
// in the position order: a ring cache and a contiguous cache give identical results.
__device__ __forceinline__ int item_stages(const Item& it) {
  return (it.v1 - it.v0 + kStageKeys - 1) / kStageKeys;
}

__device__ __forceinline__ int stage_keys(const Item& it, int k) {
  return min(kStageKeys, it.v1 - it.v0 - k * kStageKeys);
}

// Physical runs of stage k: up to three (first physical row, count, stage row) triples.
__device__ __forceinline__ int stage_runs(const Item& it, int k, int (&row)[3], int (&cnt)[3],
                                          int (&dst)[3]) {
  const int vs = it.v0 + k * kStageKeys;
  const int ve = min(it.v1, vs + kStageKeys);
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
  static constexpr size_t off_p = off_q + kStages * q_slot * 2;                  // float
  static constexpr size_t off_acc = off_p + kConsumerWarps * kKeysPerWarp * G * 4;
  static constexpr size_t off_m = off_acc + size_t(kConsumerWarps) * G * D * 4;
  static constexpr size_t off_l = off_m + kConsumerWarps * G * 4;
  static constexpr size_t off_bar = (off_l + kConsumerWarps * G * 4 + 15) / 16 * 16;
  static constexpr size_t off_wmax = off_bar + 2 * kStages * 8;  // int per warp
  static constexpr size_t off_prefix = off_wmax + 16 * 4;
  static size_t bytes(int batch) { return off_prefix + size_t(batch + 1) * 4; }
};

// As many stages (up to 3) as fit in 220 KB of shared memory with a 1024-sequence
// length table: 3 for every geometry except d = 128 with 8 query heads per KV head.
template <int D, int G>
using DecodeSmem = DecodeSmemLayout<
    D, G, (DecodeSmemLayout<D, G, kMaxStages>::off_prefix + 4100 <= 220 * 1024) ? kMaxStages : 2>;

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1) decode_split_kernel(const DecodeArgs a) {
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
  int* wmax = reinterpret_cast<int*>(smem + L::off_wmax);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + kStages);
  pdl_trigger();  // the combine kernel may be scheduled now; it waits for this grid
  pdl_wait();     // seq_len, the caches and the workspace come from earlier kernels

  // per-sequence stage counts, then an exclusive scan (warp 0) and the largest pair
  int my_max = 0;
  for (int b = tid; b < a.batch; b += kThreads) {
    const Plan p = make_plan(a, b);
    prefix[b + 1] = a.hkv * p.stages;
    my_max = max(my_max, p.stages);
    const int T = a.seq_len[b];
    if ((T < 0 || T > a.capacity) && blockIdx.x == 0) atomicOr(a.status, kStatusBadLength);
    if (a.ring_rows > 0 && T > 0 && blockIdx.x == 0 &&
        route_is_fa(a.fa_mask, a.mask_words, b, a.layer))
      atomicOr(a.status, kStatusRingRoute);
  }
  my_max = __reduce_max_sync(0xffffffffu, my_max);
  if (lane == 0) wmax[warp] = my_max;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kConsumerWarps);
    }
    fence_barrier_init();
  }
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
  const int total = prefix[a.batch];
  const int per = stages_per_cta(total, wmax[15]);
  const int range0 = min(total, int(blockIdx.x) * per);
  const int range1 = min(total, range0 + per);
  const size_t row_elems = D;

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int g = 0;
      bool ok = true;
      for (int sg = range0; sg < range1 && ok;) {
        const Item it = item_at(a, prefix, sg, range1, per);
        sg = it.seg_end;
        const size_t head_off = (size_t(it.b) * a.hkv + it.kvh) * a.rows * row_elems;
        const uint16_t* qsrc = a.q + (size_t(it.b) * a.hkv * G + size_t(it.kvh) * G) * D;
        const int ns = item_stages(it);
        for (int k = 0; k < ns; ++k, ++g) {
          int row[3], cnt[3], dst[3];
          const int runs = stage_runs(it, k, row, cnt, dst);
          const int st = g % kStages;
          const uint32_t ph = (g / kStages) & 1;
          if (!mbar_wait(empty0 + 8 * st, ph ^ 1, a.status)) { ok = false; break; }
          const uint32_t bytes = uint32_t(stage_keys(it, k)) * D * 2;
          const uint32_t qbytes = (k == 0) ? uint32_t(G * D * 2) : 0u;
          mbar_arrive_expect_tx(full0 + 8 * st, 2 * bytes + qbytes);
          if (k == 0) bulk_g2s(smem_addr(sQ + st * L::q_slot), qsrc, qbytes, full0 + 8 * st, pol);
          for (int r = 0; r < runs; ++r) {
            const uint32_t rb = uint32_t(cnt[r]) * D * 2;
            const size_t src = head_off + size_t(row[r]) * row_elems;
            bulk_g2s(smem_addr(sK + st * L::kv_stage + size_t(dst[r]) * D), a.k + src, rb,
                     full0 + 8 * st, pol);
            bulk_g2s(smem_addr(sV + st * L::kv_stage + size_t(dst[r]) * D), a.v + src, rb,
                     full0 + 8 * st, pol);
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
  const int key_sub = lane >> 3;           // which of the 4 rows of a warp instruction
  const int c = lane & 7;                  // 16-byte chunk within the row
  const int hl = c >> (3 - GB);            // head this lane holds after group_reduce
  const bool owner = (c & ((1 << (3 - GB)) - 1)) == 0;
  const int group_lane0 = lane & 24;
  int g = 0;
  bool ok = true;
  for (int sg = range0; sg < range1 && ok;) {
    const Item it = item_at(a, prefix, sg, range1, per);
    sg = it.seg_end;
    uint64_t q2[G][4 * NCH];   // pre-scaled query pairs of this lane's 8*NCH dims
    uint64_t acc[G][4 * NCH];  // P.V pairs of this lane's dims
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 4 * NCH; ++i) acc[h][i] = 0ull;
    float m_run = -INFINITY, l_run = 0.f;

    const int ns = item_stages(it);
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
        uint64_t dot2[G];
#pragma unroll
        for (int h = 0; h < G; ++h) dot2[h] = 0ull;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          const uint4 raw = lds128(Ks + key * D + ch * 64 + c * 8);
          const uint64_t k0 = bf16x2_to_f2(raw.x), k1 = bf16x2_to_f2(raw.y);
          const uint64_t k2 = bf16x2_to_f2(raw.z), k3 = bf16x2_to_f2(raw.w);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            dot2[h] = f2_fma(q2[h][ch * 4 + 0], k0, dot2[h]);
            dot2[h] = f2_fma(q2[h][ch * 4 + 1], k1, dot2[h]);
            dot2[h] = f2_fma(q2[h][ch * 4 + 2], k2, dot2[h]);
            dot2[h] = f2_fma(q2[h][ch * 4 + 3], k3, dot2[h]);
          }
        }
        float dot[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float lo, hi;
          f2_unpack(dot2[h], lo, hi);
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
    if (!ok) break;

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
    named_barrier_sync(1, kConsumerWarps * 32);
    const size_t rec = (size_t(it.b) * a.hkv + it.kvh) * kDecMaxSplits + it.split;
    if (tid == 0 && it.split == 0) a.ws_nsplit[size_t(it.b) * a.hkv + it.kvh] = it.n_split;
    for (int i = tid; i < G * D; i += kConsumerWarps * 32) {
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
      a.ws_acc[(rec * G + h) * D + e] = av;
      if (e == 0) a.ws_ml[rec * G + h] = make_float2(M, lv);
    }
    named_barrier_sync(1, kConsumerWarps * 32);
  }
}

// Merge the split partials of one (sequence, KV head): weights 2^(m_s - M) / L are
// computed once per (split, head) in shared memory, then the partial accumulators are
// read coalesced along d.
template <int D, int G>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeArgs a) {
  __shared__ float wgt[kDecMaxSplits][G];
  pdl_trigger();
  pdl_wait();  // the split kernel's partials
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int n_split = make_plan(a, b).n_vis > 0 ? a.ws_nsplit[size_t(b) * a.hkv + kvh] : 0;
  const size_t rec0 = (size_t(b) * a.hkv + kvh) * kDecMaxSplits;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (warp < G) {
    // one warp per query head of the group: splits spread over the lanes
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    if (lane < n_split) {
      const float2 ml = a.ws_ml[(rec0 + lane) * G + warp];
      m0 = ml.x; l0 = ml.y;
    }
    if (lane + 32 < n_split) {
      const float2 ml = a.ws_ml[(rec0 + lane + 32) * G + warp];
      m1 = ml.x; l1 = ml.y;
    }
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float f0 = (lane < n_split) ? ex2_mufu(m0 - M) : 0.f;
    const float f1 = (lane + 32 < n_split) ? ex2_mufu(m1 - M) : 0.f;
    float lv = f0 * l0 + f1 * l1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lv += __shfl_xor_sync(0xffffffffu, lv, off);
    const float inv = (lv > 0.f) ? 1.f / lv : 0.f;
    if (lane < n_split) wgt[lane][warp] = f0 * inv;
    if (lane + 32 < n_split) wgt[lane + 32][warp] = f1 * inv;
  }
  __syncthreads();
  uint16_t* out = a.o + (size_t(b) * a.hkv * G + size_t(kvh) * G) * D;
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int gi = i / D, e = i % D;
    const float* src = a.ws_acc + (rec0 * G + gi) * D + e;
    float av0 = 0.f, av1 = 0.f, av2 = 0.f, av3 = 0.f;
    int s = 0;
    for (; s + 4 <= n_split; s += 4) {
      av0 = fmaf(wgt[s][gi], src[size_t(s) * G * D], av0);
      av1 = fmaf(wgt[s + 1][gi], src[size_t(s + 1) * G * D], av1);
      av2 = fmaf(wgt[s + 2][gi], src[size_t(s + 2) * G * D], av2);
      av3 = fmaf(wgt[s + 3][gi], src[size_t(s + 3) * G * D], av3);
    }
    for (; s < n_split; ++s) av0 = fmaf(wgt[s][gi], src[size_t(s) * G * D], av0);
    const __nv_bfloat16 hb = __float2bfloat16_rn((av0 + av1) + (av2 + av3));
    out[gi * D + e] = *reinterpret_cast<const uint16_t*>(&hb);
  }
}

template <int D, int G>
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
      err = cudaFuncSetAttribute(decode_split_kernel<D, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(L::bytes(kDecMaxBatch)));
      if (err != cudaSuccess) return err;
      attr_set[dev] = true;
    }
  }
  err = launch_pdl(decode_split_kernel<D, G>, dim3(device_sm_count()), dim3(kThreads), smem,
                   stream, a);
  if (err != cudaSuccess) return err;
  return launch_pdl(decode_combine_kernel<D, G>, dim3(a.hkv, a.batch), dim3(256), 0, stream, a);
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
  return acc + recs * 8 + size_t(batch) * g.hkv * 4;
}

cudaError_t launch_decode(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                          const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                          const int32_t* seq_len, int batch, int capacity, int ring_rows,
                          uint16_t* o, void* workspace, unsigned* status, cudaStream_t stream) {
  const int G = g.hq / g.hkv;
  DecodeArgs a;
  a.fa_mask = fa_mask;
  a.mask_words = g.mask_words;
  a.layer = layer;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
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
  a.ws_acc = static_cast<float*>(workspace);
  const size_t acc_bytes = (recs * g.head_dim * 4 + 255) / 256 * 256;
  a.ws_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + acc_bytes);
  a.ws_nsplit = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + acc_bytes + recs * 8);
  a.o = o;
  a.status = status;
#define FLUX_DECODE_CASE(DD, GG) \
  if (g.head_dim == DD && G == GG) return launch_decode_t<DD, GG>(a, stream);
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
  // The split kernel writes every partial record the combine kernel reads, so the
  // scratch needs no clearing between calls.
  void* scratch = nullptr;
  const cudaError_t err = static_scratch_address(&scratch);
  if (err != cudaSuccess) return err;
  return launch_decode(g, layer, fa_mask, q, k_cache, v_cache, seq_len, batch, capacity, 0, o,
                       scratch, status, stream);
}

}  // namespace flux
