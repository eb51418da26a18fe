// Split-KV flash-decode for both routes of Flux Attention (Table 3: decode reuses the
// prefill route; Table 6: SA = sink + local window of KV blocks), sm_100a.
//
// One query token per sequence attends the keys of its route: FA reads the whole
// cache [0, seq_len), SA reads only the sink rows and the window rows.  Decode is
// bound by HBM bandwidth, so the kernel is built around moving K/V bytes:
//
//  * the visible keys of each (sequence, KV head) are cut into at most 64 splits of
//    >= 128 keys; a persistent grid (one CTA per SM) walks the (sequence, KV head,
//    split) items round-robin, so SA layers launch no idle CTAs;
//  * one producer lane streams each split's K and V rows -- contiguous in the
//    [B][Hkv][cap][d] cache -- into a 4-stage shared-memory ring with 1-D bulk copies
//    (cp.async.bulk, no cluster), completing on mbarriers;
//  * 8 consumer warps read the stage with 128-bit shared loads: 8 lanes cover one
//    key row (16 B each), 4 rows per warp instruction, all G = Hq/Hkv query heads of
//    the group at once; the q.k partial sums are reduced across the 8 lanes with a
//    transposing butterfly (G values in log2(G)+... shuffles instead of G*3);
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

constexpr int kStageKeys = 64;
constexpr int kStages = 4;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kKeysPerWarp = kStageKeys / kConsumerWarps;  // 8 keys per warp per stage
constexpr int kPasses = kKeysPerWarp / 4;                  // 4 keys per warp instruction

struct DecodeArgs {
  const uint32_t* fa_mask;
  int mask_words, layer;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* seq_len;
  int batch, capacity, hkv, block, sink, window;
  float scale_log2;  // log2(e) / sqrt(d)
  float* ws_acc;     // [B][Hkv][kDecMaxSplits][G][D]
  float2* ws_ml;     // [B][Hkv][kDecMaxSplits][G] = (max, sum)
  uint16_t* o;
  unsigned* status;
};

// The visible keys of sequence b's decode query, flattened: virtual key v maps to
// position v when v < len0, else to lo1 + (v - len0).
struct Plan {
  int len0, lo1, n_vis, n_split, chunk;
};

__device__ __forceinline__ Plan make_plan(const DecodeArgs& a, int b) {
  Plan p{0, 0, 0, 0, 1};
  const int T = a.seq_len[b];
  if (T <= 0 || T > a.capacity) return p;
  const bool fa = route_is_fa(a.fa_mask, a.mask_words, b, a.layer);
  const KeyRanges r = visible_key_ranges(T - 1, fa, a.block, a.sink, a.window);
  p.len0 = r.hi0 - r.lo0;
  p.lo1 = r.lo1;
  p.n_vis = p.len0 + (r.hi1 - r.lo1);
  const int s = (p.n_vis + kDecMinChunk - 1) / kDecMinChunk;
  p.n_split = s < kDecMaxSplits ? s : kDecMaxSplits;
  p.chunk = (p.n_vis + p.n_split - 1) / p.n_split;
  return p;
}

struct Item {
  int b, kvh, split;
  int a0, na;  // first piece: positions [a0, a0 + na)
  int b0, nb;  // second piece: positions [b0, b0 + nb)
};

// Item idx of the flattened (sequence, KV head, split) list; prefix[b] counts the
// items of sequences before b.
__device__ __forceinline__ Item item_at(const DecodeArgs& a, const int* prefix, int idx) {
  int lo = 0, hi = a.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= idx) lo = mid; else hi = mid;
  }
  Item it;
  it.b = lo;
  const Plan p = make_plan(a, lo);
  const int r = idx - prefix[lo];
  it.kvh = r / p.n_split;
  it.split = r % p.n_split;
  const int v0 = it.split * p.chunk;
  const int v1 = min(p.n_vis, v0 + p.chunk);
  const int ea = min(v1, p.len0);
  it.a0 = v0;
  it.na = max(0, ea - v0);
  const int sb = max(v0, p.len0);
  it.b0 = p.lo1 + (sb - p.len0);
  it.nb = max(0, v1 - sb);
  return it;
}

__device__ __forceinline__ int item_stages(const Item& it) {
  return (it.na + kStageKeys - 1) / kStageKeys + (it.nb + kStageKeys - 1) / kStageKeys;
}

// Stage k of an item: first key position and key count.
__device__ __forceinline__ void item_stage(const Item& it, int k, int& pos, int& n) {
  const int sa = (it.na + kStageKeys - 1) / kStageKeys;
  if (k < sa) {
    pos = it.a0 + k * kStageKeys;
    n = min(kStageKeys, it.na - k * kStageKeys);
  } else {
    const int kk = k - sa;
    pos = it.b0 + kk * kStageKeys;
    n = min(kStageKeys, it.nb - kk * kStageKeys);
  }
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

template <int D, int G>
struct DecodeSmem {
  static constexpr size_t kv_stage = size_t(kStageKeys) * D;  // elements per stage
  static constexpr size_t off_k = 0;
  static constexpr size_t off_v = off_k + kStages * kv_stage * 2;
  static constexpr size_t off_p = off_v + kStages * kv_stage * 2;               // float
  static constexpr size_t off_acc = off_p + kConsumerWarps * kKeysPerWarp * G * 4;
  static constexpr size_t off_m = off_acc + size_t(kConsumerWarps) * G * D * 4;
  static constexpr size_t off_l = off_m + kConsumerWarps * G * 4;
  static constexpr size_t off_bar = (off_l + kConsumerWarps * G * 4 + 15) / 16 * 16;
  static constexpr size_t off_prefix = off_bar + 2 * kStages * 8;
  static size_t bytes(int batch) { return off_prefix + size_t(batch + 1) * 4; }
};

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1) decode_split_kernel(const DecodeArgs a) {
  using L = DecodeSmem<D, G>;
  constexpr int NCH = D / 64;          // 16-byte chunks of a row per lane
  constexpr int GB = (G == 1) ? 0 : (G == 2) ? 1 : (G == 4) ? 2 : 3;
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* sK = reinterpret_cast<uint16_t*>(smem + L::off_k);
  uint16_t* sV = reinterpret_cast<uint16_t*>(smem + L::off_v);
  float* sP = reinterpret_cast<float*>(smem + L::off_p);
  float* sAcc = reinterpret_cast<float*>(smem + L::off_acc);
  float* sM = reinterpret_cast<float*>(smem + L::off_m);
  float* sL = reinterpret_cast<float*>(smem + L::off_l);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  int* prefix = reinterpret_cast<int*>(smem + L::off_prefix);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + kStages);

  // per-sequence item counts, then an exclusive scan (warp 0)
  for (int b = tid; b < a.batch; b += kThreads) {
    const Plan p = make_plan(a, b);
    prefix[b + 1] = a.hkv * p.n_split;
    const int T = a.seq_len[b];
    if ((T < 0 || T > a.capacity) && blockIdx.x == 0) atomicOr(a.status, kStatusBadLength);
  }
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
  }
  __syncthreads();
  const int total = prefix[a.batch];
  const size_t row_elems = D;

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int g = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
        const Item it = item_at(a, prefix, idx);
        const size_t head_off = (size_t(it.b) * a.hkv + it.kvh) * a.capacity * row_elems;
        const int ns = item_stages(it);
        for (int k = 0; k < ns; ++k, ++g) {
          int pos, n;
          item_stage(it, k, pos, n);
          const int st = g % kStages;
          const uint32_t ph = (g / kStages) & 1;
          if (!mbar_wait(empty0 + 8 * st, ph ^ 1, a.status)) { ok = false; break; }
          const uint32_t bytes = uint32_t(n) * D * 2;
          mbar_arrive_expect_tx(full0 + 8 * st, 2 * bytes);
          bulk_g2s(smem_addr(sK + st * L::kv_stage), a.k + head_off + size_t(pos) * row_elems,
                   bytes, full0 + 8 * st, pol);
          bulk_g2s(smem_addr(sV + st * L::kv_stage), a.v + head_off + size_t(pos) * row_elems,
                   bytes, full0 + 8 * st, pol);
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
  for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
    const Item it = item_at(a, prefix, idx);
    float qf[G][8 * NCH];
    {
      const uint16_t* qp = a.q + (size_t(it.b) * a.hkv * G + size_t(it.kvh) * G) * D;
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qp + h * D + ch * 64 + c * 8));
          float f[8];
          bf16x8_to_float(raw, f);
#pragma unroll
          for (int e = 0; e < 8; ++e) qf[h][ch * 8 + e] = f[e] * a.scale_log2;
        }
    }
    float acc[G][8 * NCH];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8 * NCH; ++e) acc[h][e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    const int ns = item_stages(it);
    for (int k = 0; k < ns; ++k, ++g) {
      int pos, n;
      item_stage(it, k, pos, n);
      const int st = g % kStages;
      const uint32_t ph = (g / kStages) & 1;
      if (!mbar_wait(full0 + 8 * st, ph, a.status)) { ok = false; break; }
      const uint16_t* Ks = sK + st * L::kv_stage;
      const uint16_t* Vs = sV + st * L::kv_stage;

      float s[kPasses];
#pragma unroll
      for (int p = 0; p < kPasses; ++p) {
        const int key = warp * kKeysPerWarp + p * 4 + key_sub;
        float dot[G];
#pragma unroll
        for (int h = 0; h < G; ++h) dot[h] = 0.f;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          const uint4 raw = lds128(Ks + key * D + ch * 64 + c * 8);
          float kf[8];
          bf16x8_to_float(raw, kf);
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) dot[h] = fmaf(qf[h][ch * 8 + e], kf[e], dot[h]);
        }
        const float r = group_reduce<G>(dot, lane);
        s[p] = (key < n) ? r : -INFINITY;
      }
      float mt = s[0];
#pragma unroll
      for (int p = 1; p < kPasses; ++p) mt = fmaxf(mt, s[p]);
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
      const float m_new = fmaxf(m_run, mt);
      if (__any_sync(0xffffffffu, m_new > m_run)) {
        const float alpha = (m_new > m_run) ? fast_exp2(m_run - m_new) : 1.f;
        l_run *= alpha;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float ah = __shfl_sync(0xffffffffu, alpha, group_lane0 | (h << (3 - GB)));
#pragma unroll
          for (int e = 0; e < 8 * NCH; ++e) acc[h][e] *= ah;
        }
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float* Pw = sP + warp * kKeysPerWarp * G;
#pragma unroll
      for (int p = 0; p < kPasses; ++p) {
        const float pr = fast_exp2(s[p] - m_use);
        l_run += pr;
        if (owner) Pw[(p * 4 + key_sub) * G + hl] = pr;
      }
      __syncwarp();
#pragma unroll
      for (int p = 0; p < kPasses; ++p) {
        const int key = warp * kKeysPerWarp + p * 4 + key_sub;
        if (key < n) {
          float pw[G];
#pragma unroll
          for (int h = 0; h < G; ++h) pw[h] = Pw[(p * 4 + key_sub) * G + h];
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            const uint4 raw = lds128(Vs + key * D + ch * 64 + c * 8);
            float vf[8];
            bf16x8_to_float(raw, vf);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[h][ch * 8 + e] = fmaf(pw[h], vf[e], acc[h][ch * 8 + e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
    }
    if (!ok) break;

    // reduce the 4 row groups of the warp, then the 8 warps through shared memory
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8 * NCH; ++e) {
        acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], 8);
        acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], 16);
      }
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
    if (key_sub == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          float4* dst = reinterpret_cast<float4*>(sAcc + (warp * G + h) * D + ch * 64 + c * 8);
          dst[0] = make_float4(acc[h][ch * 8 + 0], acc[h][ch * 8 + 1], acc[h][ch * 8 + 2],
                               acc[h][ch * 8 + 3]);
          dst[1] = make_float4(acc[h][ch * 8 + 4], acc[h][ch * 8 + 5], acc[h][ch * 8 + 6],
                               acc[h][ch * 8 + 7]);
        }
      if (owner) {
        sM[warp * G + hl] = m_run;
        sL[warp * G + hl] = l_run;
      }
    }
    named_barrier_sync(1, kConsumerWarps * 32);
    const size_t rec = (size_t(it.b) * a.hkv + it.kvh) * kDecMaxSplits + it.split;
    for (int i = tid; i < G * D; i += kConsumerWarps * 32) {
      const int h = i / D, e = i % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sM[w * G + h]);
      float av = 0.f, lv = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = sM[w * G + h];
        const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
        av = fmaf(f, sAcc[(w * G + h) * D + e], av);
        lv = fmaf(f, sL[w * G + h], lv);
      }
      a.ws_acc[(rec * G + h) * D + e] = av;
      if (e == 0) a.ws_ml[rec * G + h] = make_float2(M, lv);
    }
    named_barrier_sync(1, kConsumerWarps * 32);
  }
}

template <int D, int G>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeArgs a) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int kvh = h / G, gi = h % G;
  const Plan p = make_plan(a, b);
  uint16_t* out = a.o + (size_t(b) * a.hkv * G + h) * D;
  const size_t rec0 = (size_t(b) * a.hkv + kvh) * kDecMaxSplits;
  float M = -INFINITY;
  for (int s = 0; s < p.n_split; ++s) M = fmaxf(M, a.ws_ml[(rec0 + s) * G + gi].x);
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float lv = 0.f, av = 0.f;
    for (int s = 0; s < p.n_split; ++s) {
      const float2 ml = a.ws_ml[(rec0 + s) * G + gi];
      const float f = fast_exp2(ml.x - M);
      lv = fmaf(f, ml.y, lv);
      av = fmaf(f, a.ws_acc[((rec0 + s) * G + gi) * D + e], av);
    }
    const float r = (p.n_split > 0) ? av / lv : 0.f;
    const __nv_bfloat16 hb = __float2bfloat16_rn(r);
    out[e] = *reinterpret_cast<const uint16_t*>(&hb);
  }
}

template <int D, int G>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  using L = DecodeSmem<D, G>;
  const size_t smem = L::bytes(a.batch);
  cudaError_t err = cudaFuncSetAttribute(decode_split_kernel<D, G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return err;
  const int max_items = a.batch * a.hkv * kDecMaxSplits;
  const int grid = min(max_items, device_sm_count());
  decode_split_kernel<D, G><<<grid, kThreads, smem, stream>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  decode_combine_kernel<D, G><<<dim3(a.hkv * G, a.batch), 128, 0, stream>>>(a);
  return cudaGetLastError();
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
  return acc + recs * 8;
}

cudaError_t launch_decode(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                          const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                          const int32_t* seq_len, int batch, int capacity, uint16_t* o,
                          void* workspace, unsigned* status, cudaStream_t stream) {
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
  a.capacity = capacity;
  a.hkv = g.hkv;
  a.block = g.block;
  a.sink = g.sink;
  a.window = g.window;
  a.scale_log2 = float(1.4426950408889634 / sqrt(double(g.head_dim)));
  const size_t recs = size_t(batch) * g.hkv * kDecMaxSplits * G;
  a.ws_acc = static_cast<float*>(workspace);
  a.ws_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) +
                                      (recs * g.head_dim * 4 + 255) / 256 * 256);
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
  return launch_decode(g, layer, fa_mask, q, k_cache, v_cache, seq_len, batch, capacity, o,
                       scratch, status, stream);
}

}  // namespace flux
