// Causal GQA flash-attention prefill on the 5th-generation tensor cores (sm_100a),
// for both routes of Flux Attention: Full Attention visits every KV tile up to the
// diagonal, streaming Sparse Attention (Table 6: attention-sink blocks plus a local
// window of blocks) visits only the sink tiles and the window tiles.  The route is
// read on the device from the layer's bit of the router's mask (Figure 2).
//
// One CTA computes one 128-query tile of one query head.  Roles (352 threads):
//   warps 0-7  softmax, two warpgroups that ping-pong over the KV tiles: warpgroup g
//              (g = 0, 1) takes the tiles j = g, g + 2, g + 4, ...  Thread = one
//              query row.  For its tile it reads the row of S = Q K^T from tensor
//              memory (tcgen05.ld), masks boundary tiles, runs the online softmax in
//              registers (log2 domain; its own stale row maximum, raised only when
//              the new maximum exceeds it by more than 2^8, and then its O is
//              rescaled in tensor memory) and writes P as bf16 into its own P buffer
//              in shared memory (128-byte swizzle, K-major: the A operand of P.V).
//              As soon as the row of S has been read it releases the S buffer, so
//              S_{j+2} runs on the tensor cores while the exponentials of tile j are
//              still being computed.  The exponentials are taken against the current
//              maximum in the same pass that finds the tile maximum; only a warp with a
//              row whose maximum jumped re-reads the tile.  Each warpgroup accumulates
//              its own O; at the end the two partial (max, sum, O) are merged per row,
//              normalised and stored.
//   warps 8-9  TMA producers (cp.async.bulk.tensor, 128-byte swizzle, no cluster, no
//              multicast): warp 8 the Q tile once and K tiles into a ring (2 stages at
//              d = 128, 3 at d = 64) released as soon as each tile's S MMAs complete;
//              warp 9 V tiles into a 2-stage ring released by the P.V MMAs.
//   warp 10    MMA issuer (one thread) with two streams per warpgroup: S_j = Q K_j^T
//              (A, B from shared memory) into the S buffer of warpgroup j % 2 once that
//              buffer is released and K_j has landed, and O_{j%2} += P_j V_j (P_j from
//              the warpgroup's P buffer, V_j an MN-major operand) once P_j is written;
//              completion is signalled with tcgen05.commit on mbarriers, the P buffer
//              is released by the commit after P_j V_j.  The warp also allocates and
//              frees the 512 tensor-memory columns (S0 | S1 | O0 | O1).
// Keeping P in tensor memory over S (the earlier design) forced S_{j+2} to wait for
// P_j V_j; with P in shared memory the 8K-token FA launch went from 0.574 to 0.550 ms.
//
// Every mbarrier wait is bounded: on time-out the thread records FLUX_DEVICE_TIMEOUT
// and leaves its loop; all roles meet at the final barrier, the producers first wait
// for their copies in flight, the MMA thread for its MMAs, and the tensor memory is
// always freed.
#include <cuda.h>
#include <math.h>

#include "flux_device.cuh"
#include "flux_internal.h"
#include "tc_sm100.cuh"

namespace flux {
namespace {

constexpr int BM = 128;  // query rows per tile (MMA M)
constexpr int BN = 128;  // keys per KV tile (MMA N of Q K^T, MMA K of P V)
// K tiles are released as soon as their S MMA completes, V tiles when their P.V MMA
// completes.  With P in shared memory (two 32 KB buffers) d = 128 fits 2 + 2 stages in
// the 227 KB of a CTA; d = 64 keeps 3 K stages.
template <int D> constexpr int kKSt = D == 128 ? 2 : 3;
constexpr int kVStages = 2;
constexpr int kSoftmaxThreads = 256;
constexpr int kKProducerWarp = 8;
constexpr int kVProducerWarp = 9;
constexpr int kMmaWarp = 10;
constexpr int kThreads = 352;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;           // O_g accumulator columns [256 + 128 g, + D)
constexpr uint32_t kSubBytes = 128 * 128;  // one 64-column swizzled sub-tile of 128 rows
constexpr uint32_t kPBytes = 2 * kSubBytes;  // P tile: 128 rows x 128 keys bf16
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Of every 8 exponential pairs of a softmax row, this many go to the MUFU unit and the
// rest to the polynomial on the FMA pipe.  Measured on B200 (Llama shape, 32K prompt):
// 8/8 -> 8.09 ms, 6/8 -> 8.45 ms, 5/8 -> 8.70 ms: the softmax warps are bound by issue
// and latency, not by MUFU throughput, so every exponential stays on MUFU.
constexpr int kMufuPairsPer8 = 8;

template <int D>
struct Smem {
  static constexpr int NCH = D / 64;
  static constexpr uint32_t tile = NCH * kSubBytes;  // Q tile or one K / V tile
  static constexpr uint32_t off_q = 0;
  static constexpr int KS = kKSt<D>;
  static constexpr uint32_t off_k = off_q + tile;
  static constexpr uint32_t off_v = off_k + KS * tile;
  static constexpr uint32_t off_p = off_v + kVStages * tile;  // P of warpgroup g at + g kPBytes
  static constexpr uint32_t off_ms = off_p + 2 * kPBytes;     // float [2][128] row maxima
  static constexpr uint32_t off_ls = off_ms + 2 * 128 * 4;      // float [2][128] row sums
  static constexpr uint32_t off_bar = off_ls + 2 * 128 * 4;
  // q_full | k_full[KS] | k_empty[KS] | v_full[2] | v_empty[2] | s_full[2] | p_full[2] |
  // s_free[2] | p_free[2] | o_final | mma_idle
  static constexpr int n_bars = 1 + 2 * KS + 2 * kVStages + 2 + 2 + 2 + 2 + 2;
  static constexpr uint32_t off_tmem = off_bar + n_bars * 8;
  static constexpr uint32_t used = off_tmem + 16;
  // The dynamic shared memory starts 1024-byte aligned (checked by the kernel, which
  // reports FLUX_DEVICE_LAYOUT otherwise), so no alignment slack is reserved: the d = 128
  // layout needs 226 KB of the 227 KB a CTA may have.  At least 116 KB, so that a second
  // CTA (which would need its own 512 tensor-memory columns) never shares the SM.
  static constexpr uint32_t bytes = used > 118784 ? used : 118784;
};

struct PrefillArgs {
  const uint32_t* fa_mask;
  int mask_words, layer;
  const int32_t* seq_len;
  int capacity, n_q, hq, hkv, block, sink, window, n_mtiles;
  float scale_log2;
  uint16_t* o;
  unsigned* status;
};

// ------------------------------------------------------------------ tile schedule

// KV tiles of one query tile: tile index j < n0 is key tile j (the sink tiles); the
// rest are key tiles w0 + (j - n0) (the window, up to the diagonal).  For FA n0 = 0
// and w0 = 0.  Built from the union of the tile's rows' visible keys
// (visible_key_ranges_rows, the shared SA definition), rounded out to whole tiles: a
// tile is visited iff it holds a key that some row of the query tile sees.
struct TilePlan {
  int n0, w0, n_tiles;
  int t_min, t_max;   // absolute positions of the tile's first and last real query
  int gap0, gap1;     // keys [gap0, gap1) are hidden from the last row (empty for FA)
};

__device__ __forceinline__ TilePlan plan_tiles(const PrefillArgs& a, bool fa, int t_min, int t_max) {
  TilePlan p;
  p.t_min = t_min;
  p.t_max = t_max;
  const int last = t_max / BN;
  const KeyRanges u = visible_key_ranges_rows(t_min, t_max, fa, a.block, a.sink, a.window);
  // The rows' sink/window gaps grow with t, so the last row's gap covers every row's.
  const KeyRanges lr = visible_key_ranges(t_max, fa, a.block, a.sink, a.window);
  p.gap0 = lr.hi0;
  p.gap1 = lr.lo1;
  const int n_sink_tiles = (u.hi0 + BN - 1) / BN;
  const int w0 = u.lo1 / BN;
  if (w0 <= n_sink_tiles) {  // FA, or the window reaches back to the sink tiles
    p.n0 = 0;
    p.w0 = 0;
    p.n_tiles = last + 1;
  } else {
    p.n0 = n_sink_tiles;
    p.w0 = w0;
    p.n_tiles = n_sink_tiles + (last + 1 - w0);
  }
  return p;
}

__device__ __forceinline__ int tile_key0(const TilePlan& p, int j) {
  return (j < p.n0 ? j : p.w0 + (j - p.n0)) * BN;
}

// True when some (query, key) pair of the tile is not visible: a key past the first
// row (causal diagonal, valid length), or a key in the last row's sink/window gap.
__device__ __forceinline__ bool tile_needs_mask(const TilePlan& p, int k0) {
  if (k0 + BN - 1 > p.t_min) return true;
  return k0 < p.gap1 && k0 + BN > p.gap0;
}

// The plan of query tile m_tile of sequence b, as the prefill kernel computes it.
// ok = false for a sequence whose length is out of range (nothing is computed).
__device__ __forceinline__ TilePlan plan_for(const PrefillArgs& a, int b, int m_tile, int& rows,
                                             int& q_start, bool& ok) {
  const int seq = a.seq_len[b];
  ok = seq >= a.n_q && seq <= a.capacity;
  q_start = seq - a.n_q;
  const int row0 = m_tile * BM;
  rows = min(BM, a.n_q - row0);
  const bool fa = route_is_fa(a.fa_mask, a.mask_words, b, a.layer);
  return plan_tiles(a, fa, q_start + row0, q_start + row0 + rows - 1);
}

// ------------------------------------------------------------------ the kernel

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillArgs a) {
  using L = Smem<D>;
  constexpr int NCH = L::NCH;
  constexpr int KS = L::KS;
  constexpr int DH = D / 2;  // O columns per softmax warpgroup
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  if (raw_addr & 1023u) {  // the swizzled TMA tiles need 1024-byte alignment
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
      atomicOr(a.status, kStatusLayout);
    return;
  }
  const uint32_t base = raw_addr;
  uint8_t* smem = smem_raw;

  const uint32_t sQ = base + L::off_q;
  const uint32_t sK = base + L::off_k;
  const uint32_t sV = base + L::off_v;
  float* ms = reinterpret_cast<float*>(smem + L::off_ms);
  float* ls = reinterpret_cast<float*>(smem + L::off_ls);
  const uint32_t bar0 = base + L::off_bar;
  const uint32_t bar_q = bar0;
  const uint32_t bar_kfull = bar0 + 8;                        // + 8 * K stage
  const uint32_t bar_kempty = bar_kfull + 8 * KS;
  const uint32_t bar_vfull = bar_kempty + 8 * KS;       // + 8 * V stage
  const uint32_t bar_vempty = bar_vfull + 8 * kVStages;
  const uint32_t bar_sfull = bar_vempty + 8 * kVStages;       // + 8 * warpgroup
  const uint32_t bar_pfull = bar_sfull + 16;                  // + 8 * warpgroup
  const uint32_t bar_sfree = bar_pfull + 16;   // + 8 * warpgroup: S read, buffer reusable
  const uint32_t bar_pfree = bar_sfree + 16;   // + 8 * warpgroup: P.V done, P buffer free
  const uint32_t bar_ofinal = bar_pfree + 16;
  const uint32_t sP = base + L::off_p;
  const uint32_t bar_idle = bar_ofinal + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::off_tmem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x;
  const int m_tile = a.n_mtiles - 1 - int(blockIdx.y);  // longest causal rows first
  const int b = blockIdx.z;
  const int kvh = h / (a.hq / a.hkv);

  int rows, q_start;
  bool len_ok;
  const TilePlan plan = plan_for(a, b, m_tile, rows, q_start, len_ok);
  if (!len_ok) {
    if (tid == 0 && h == 0 && blockIdx.y == 0) atomicOr(a.status, kStatusBadLength);
    return;
  }
  const int seq = q_start + a.n_q;
  const int row0 = m_tile * BM;                    // first query index of the tile
  const bool fa = route_is_fa(a.fa_mask, a.mask_words, b, a.layer);

  // The K producer thread initialises the barriers and issues the Q tile and the first
  // K tiles at once, while the MMA warp allocates tensor memory: the loads are in
  // flight before the CTA-wide barrier instead of after it.
  const bool k_thread = (tid == kKProducerWarp * 32);
  const int kv_row = b * a.hkv + kvh;
  int k_pre = 0;  // K tiles issued before the barrier
  if (k_thread) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(bar_kfull + 8 * s, 1);
      mbar_init(bar_kempty + 8 * s, 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar_vfull + 8 * s, 1);
      mbar_init(bar_vempty + 8 * s, 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar_sfull + 8 * g, 1);
      mbar_init(bar_pfull + 8 * g, 4);
      mbar_init(bar_sfree + 8 * g, 4);
      mbar_init(bar_pfree + 8 * g, 1);
    }
    mbar_init(bar_ofinal, 1);
    mbar_init(bar_idle, 1);
    fence_barrier_init();
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    mbar_arrive_expect_tx(bar_q, L::tile);
    for (int c = 0; c < NCH; ++c) tma_load_4d(sQ + c * kSubBytes, &tmQ, c * 64, h, row0, b, bar_q);
    k_pre = plan.n_tiles < KS ? plan.n_tiles : KS;
    for (int j = 0; j < k_pre; ++j) {
      const int k0 = tile_key0(plan, j);
      mbar_arrive_expect_tx(bar_kfull + 8 * j, L::tile);
      for (int c = 0; c < NCH; ++c)
        tma_load_3d(sK + j * L::tile + c * kSubBytes, &tmK, c * 64, k0, kv_row, bar_kfull + 8 * j);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kKProducerWarp || warp == kVProducerWarp) {
    // ---------------------------------------------------------------- TMA producers
    // warp 8 loads Q and the K ring, warp 9 the V ring; each waits only on its own
    // ring's release barriers, so K runs up to three tiles ahead of the MMAs.
    if (lane == 0) {
      const bool is_k = (warp == kKProducerWarp);
      const int n_st = is_k ? KS : kVStages;
      const uint32_t full = is_k ? bar_kfull : bar_vfull;
      const uint32_t empty = is_k ? bar_kempty : bar_vempty;
      const uint32_t ring = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      if (!is_k) prefetch_tmap(map);
      // Q and the first K tiles were issued before the CTA barrier
      int issued = is_k ? k_pre : 0;
      for (int j = issued; j < plan.n_tiles; ++j) {
        const int st = j % n_st;
        const uint32_t ph = (j / n_st) & 1;
        if (!mbar_wait(empty + 8 * st, ph ^ 1, a.status)) break;
        const int k0 = tile_key0(plan, j);
        mbar_arrive_expect_tx(full + 8 * st, L::tile);
        for (int c = 0; c < NCH; ++c)
          tma_load_3d(ring + st * L::tile + c * kSubBytes, map, c * 64, k0, kv_row, full + 8 * st);
        ++issued;
      }
      // wait for the copies in flight before the CTA may exit
      if (is_k) mbar_wait(bar_q, 0, a.status);
      for (int j = (issued > n_st ? issued - n_st : 0); j < issued; ++j)
        mbar_wait(full + 8 * (j % n_st), (j / n_st) & 1, a.status);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc(BM, BN, false, false);
      constexpr uint32_t idesc_o = make_idesc(BM, D, false, true);
      bool ok = mbar_wait(bar_q, 0, a.status);
      // S_j = Q K_j^T into the S buffer of warpgroup j % 2 (its K stage has landed)
      auto issue_s = [&](int j) {
        const int st = j % KS;
        tc_fence_after();
        const uint32_t kb = sK + st * L::tile;
        const uint32_t sbuf = tmem + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSubBytes + (kk & 3) * 32;
          mma_bf16(sbuf, sw128_desc(sQ + off, 16, 1024), sw128_desc(kb + off, 16, 1024), idesc_s,
                   kk > 0);
        }
        mma_commit(bar_sfull + 8 * (j & 1));
        mma_commit(bar_kempty + 8 * st);
      };
      const int n = plan.n_tiles;
      for (int j = 0; ok && j < 2 && j < n; ++j) {
        ok = mbar_wait(bar_kfull + 8 * (j % KS), (j / KS) & 1, a.status);
        if (ok) issue_s(j);
      }
      // Two independent streams per warpgroup g: S_{j+2} as soon as the softmax has read
      // S_j out of tensor memory (s_free) and K_{j+2} has landed -- P lives in shared
      // memory, so the S buffer is free before P_j V_j runs -- and P_j V_j as soon as P_j
      // (p_full) and V_j have landed.  Polling uses the non-blocking test.
      int s_next[2] = {2, 3}, pv_next[2] = {0, 1};
      // The clock is read only after 256 idle polls in a row, never on a productive
      // pass: the loop's latency is the MMAs' reaction time.  A wait is thus bounded by
      // the limit plus 256 polls.
      unsigned idle = 0;
      unsigned long long t_idle = 0;
      while (ok && (pv_next[0] < n || pv_next[1] < n)) {
        bool progress = false;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int js = s_next[g];
          // K_js refills the slot of K_{js-KS}.  A parity test on the slot is exact only
          // once that earlier fill is known to have landed, i.e. once S_{js-KS} has been
          // issued (with KS = 3 it belongs to the other warpgroup); K_js cannot land
          // before that anyway, since S_{js-KS} has to release the slot first.  The
          // index (g + KS) & 1 is a constant of the unrolled loop (a dynamic one would put
          // s_next in local memory, on this thread's critical path).
          const int t_prev = js - KS;
          const bool prev_seen = (KS % 2 == 0) || t_prev < 0 || s_next[(g + KS) & 1] > t_prev;
          if (js < n && prev_seen && mbar_test(bar_sfree + 8 * g, ((js - 2) >> 1) & 1) &&
              mbar_test(bar_kfull + 8 * (js % KS), (js / KS) & 1)) {
            issue_s(js);
            s_next[g] = js + 2;
            progress = true;
          }
          const int j = pv_next[g];
          if (j >= n) continue;
          // V_j refills the slot of V_{j-2}, read by P_{j-2} V_{j-2} of this warpgroup,
          // already issued: the parity test is exact
          static_assert(kVStages == 2, "V slot reuse must stay within one warpgroup");
          const int st = j % kVStages;
          if (!mbar_test(bar_pfull + 8 * g, (j >> 1) & 1)) continue;
          if (!mbar_test(bar_vfull + 8 * st, (j / kVStages) & 1)) continue;
          tc_fence_after();
          const uint32_t vb = sV + st * L::tile;
          const uint32_t pb = sP + g * kPBytes;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kSubBytes + (kk & 3) * 32;
            mma_bf16(tmem + kTmemO + g * 128, sw128_desc(pb + off, 16, 1024),
                     sw128_desc(vb + kk * 16 * 128, kSubBytes, 1024), idesc_o, (j >= 2 || kk > 0));
          }
          mma_commit(bar_vempty + 8 * st);
          mma_commit(bar_pfree + 8 * g);
          pv_next[g] = j + 2;
          progress = true;
        }
        if (progress) {
          idle = 0;
        } else if ((++idle & 255u) == 0u) {
          const unsigned long long now = global_ns();
          if (idle == 256u) {
            t_idle = now;
          } else if (now - t_idle > kWaitLimitNs) {
            atomicOr(a.status, kStatusTimeout);
            ok = false;
          }
        }
      }
      // every MMA this thread issued has finished before tensor memory is freed
      mma_commit(bar_ofinal);
      mma_commit(bar_idle);
      mbar_wait(bar_idle, 0, a.status);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int g = warp >> 2;                      // warpgroup: tiles j = g (mod 2)
    const int r = (warp & 3) * 32 + lane;         // query row within the tile
    const bool real_row = r < rows;
    const int t = plan.t_min + (real_row ? r : rows - 1);
    // this row's visible keys: [0, vr.hi0) U [vr.lo1, t], the shared SA definition
    const KeyRanges vr = visible_key_ranges(t, fa, a.block, a.sink, a.window);
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t srow = tmem + g * 128 + lane_base;
    const uint32_t orow = tmem + kTmemO + g * 128 + lane_base;
    // this row of the warpgroup's P buffer (128-byte swizzle, K-major, as the MMA reads it)
    const uint32_t prow = sP + g * kPBytes + (r >> 3) * 1024 + (r & 7) * 128;
    const float c = a.scale_log2;
    float m_used = -INFINITY;  // scaled (log2) units
    float l_sum = 0.f;
    bool ok = true;
    for (int j = g; j < plan.n_tiles; j += 2) {
      if (!mbar_wait(bar_sfull + 8 * g, (j >> 1) & 1, a.status)) { ok = false; break; }
      tc_fence_after();
      const int k0 = tile_key0(plan, j);
      const bool masked = tile_needs_mask(plan, k0);
      // This row's visible key offsets i in [0, BN) of the tile: causal i <= lim, and for
      // SA outside the gap [gap0, gap1) between the sink and the window (has_gap: the
      // gap meets this tile).  The mask costs instructions on every key of a masked tile
      // (the diagonal tile of every causal row block), so the common causal-only case is
      // one compare and one select per key.
      const int lim = t - k0;
      const int gap0 = min(max(vr.hi0 - k0, 0), BN);
      const int gap1 = min(max(vr.lo1 - k0, 0), BN);
      const bool has_gap = __any_sync(0xffffffffu, gap0 < gap1);
      // Load 64 columns of the S row into s[] and apply the tile's mask.
      auto load_half = [&](uint32_t (&s)[64], int half) {
        FLUX_TMEM_LD32(srow + half * 64, s);
        {
          uint32_t* s2 = s + 32;
          FLUX_TMEM_LD32(srow + half * 64 + 32, s2);
        }
        tmem_wait_ld();
        if (masked) {
          const int lim_h = lim - half * 64;  // visible iff i <= lim_h
          if (has_gap) {
            const int g0 = gap0 - half * 64, g1 = gap1 - half * 64;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const bool vis = (i <= lim_h) & ((i < g0) | (i >= g1));
              s[i] = vis ? s[i] : 0xff800000u;  // -inf
            }
          } else if (__any_sync(0xffffffffu, lim_h < 63)) {
#pragma unroll
            for (int i = 0; i < 64; ++i) s[i] = (i <= lim_h) ? s[i] : 0xff800000u;
          }
        }
      };
      auto max_half = [&](const uint32_t (&s)[64]) -> float {
        float mx[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) mx[x] = __uint_as_float(s[x]);
#pragma unroll
        for (int i = 8; i < 64; i += 16)
#pragma unroll
          for (int x = 0; x < 8; ++x)
            mx[x] = fmax3(mx[x], __uint_as_float(s[i + x]), __uint_as_float(s[i + 8 + x]));
        return fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
      };
      // P = exp2(S * c - m) of one half as packed bf16 pairs over columns
      // [32 half, 32 half + 32) of the buffer (keys 2w, 2w + 1 in column w); returns the
      // half's row sum.  The S values there were consumed before this store.
      auto exp_half = [&](const uint32_t (&s)[64], int half, float m_use) -> float {
        const uint64_t c2 = f2_pack(c, c);
        const uint64_t nm2 = f2_pack(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[32];
#pragma unroll
        for (int w = 0; w < 32; ++w) {
          const uint64_t x2 =
              f2_fma(f2_pack(__uint_as_float(s[2 * w]), __uint_as_float(s[2 * w + 1])), c2, nm2);
          uint64_t p2;
          if ((w & 7) >= kMufuPairsPer8) {
            p2 = exp2_poly_f2(x2);  // on the FMA pipe
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(ex2_mufu(x0), ex2_mufu(x1));
          }
          acc[w & 3] = f2_add(acc[w & 3], p2);
          float p0, p1;
          f2_unpack(p2, p0, p1);
          pk[w] = pack_bf16x2(p0, p1);
        }
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          sts128(prow + half * kSubBytes + ((cc ^ (r & 7)) << 4), pk[4 * cc], pk[4 * cc + 1],
                 pk[4 * cc + 2], pk[4 * cc + 3]);
        const uint64_t sum2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        float s0, s1;
        f2_unpack(sum2, s0, s1);
        return s0 + s1;
      };
      // Fast path: exponentials against the current stale maximum, one TMEM read of S.
      // Any row of the warp whose maximum moved by more than the threshold (and the
      // first tile) sends the warp to the slow path, which recomputes the tile.
      // P_{j-2} V_{j-2} must have read this warpgroup's P buffer (and written O_g)
      // before P_j is stored or O_g rescaled; waited for once, where first needed
      bool p_free = false;
      auto wait_p_free = [&]() {
        if (!p_free) {
          if (!mbar_wait(bar_pfree + 8 * g, ((j >> 1) & 1) ^ 1, a.status)) ok = false;
          p_free = true;
        }
      };
      // S_j has been read out of tensor memory: S_{j+2} may be issued into the buffer
      auto release_s = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sfree + 8 * g);
      };
      float mrow, lpart = 0.f;
      bool slow;
      {
        uint32_t s[64];
        load_half(s, 0);
        mrow = max_half(s);
        slow = __any_sync(0xffffffffu, m_used == -INFINITY || mrow * c > m_used + kRescaleThreshold);
        if (!slow) {
          wait_p_free();
          lpart = exp_half(s, 0, m_used);
          load_half(s, 1);
          const float m1 = max_half(s);
          mrow = fmaxf(mrow, m1);
          slow = __any_sync(0xffffffffu, m1 * c > m_used + kRescaleThreshold);
          if (!slow) {
            release_s();
            lpart += exp_half(s, 1, m_used);
          }
        } else {
          load_half(s, 1);
          mrow = fmaxf(mrow, max_half(s));
        }
      }
      if (slow) {
        const float m_tile = mrow * c;
        const bool bump = (m_used == -INFINITY) ? (m_tile > -INFINITY)
                                                : (m_tile > m_used + kRescaleThreshold);
        float alpha = 1.f;
        if (bump) {
          alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - m_tile);
          m_used = m_tile;
          l_sum *= alpha;
        }
        // O_g was last written by P_{j-2} V_{j-2}: wait for it before the rescale
        wait_p_free();
        if (j >= 2 && __any_sync(0xffffffffu, bump)) {
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t ov[32];
            FLUX_TMEM_LD32(orow + q * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            FLUX_TMEM_ST32(orow + q * 32, ov);
          }
        }
        const float m_use = (m_used == -INFINITY) ? 0.f : m_used;
        lpart = 0.f;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t s[64];
          load_half(s, half);
          if (half == 1) release_s();
          lpart += exp_half(s, half, m_use);
        }
      }
      l_sum += lpart;
      tmem_wait_st();
      fence_proxy_async_smem();  // P stores, before the MMA reads them
      // keys past the valid length: zero their V rows (the cache there is unwritten)
      if (k0 + BN > seq) {
        const int st = j % kVStages;
        if (!mbar_wait(bar_vfull + 8 * st, (j / kVStages) & 1, a.status)) { ok = false; break; }
        if (k0 + r >= seq) {
#pragma unroll
          for (int cch = 0; cch < NCH; ++cch) {
            const uint32_t vrow = sV + st * L::tile + cch * kSubBytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int x = 0; x < 8; ++x) sts128(vrow + x * 16, 0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull + 8 * g);
    }
    // epilogue: merge the two warpgroups' (max, sum, O), normalise, store; warpgroup g
    // writes output columns [g D/2, (g + 1) D/2)
    ms[g * 128 + r] = m_used;
    ls[g * 128 + r] = l_sum;
    named_barrier_sync(1, kSoftmaxThreads);
    const bool two = plan.n_tiles > 1;
    const float m0 = ms[r], m1 = two ? ms[128 + r] : -INFINITY;
    const float M = fmaxf(m0, m1);
    const float a0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - M);
    const float a1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - M);
    const float inv_l = 1.f / (a0 * ls[r] + (two ? a1 * ls[128 + r] : 0.f));
    if (ok && plan.n_tiles > 0 && mbar_wait(bar_ofinal, 0, a.status)) {
      tc_fence_after();
      const float w0 = a0 * inv_l, w1 = a1 * inv_l;
      const uint32_t o0 = tmem + kTmemO + lane_base + g * DH;
      uint16_t* dst = a.o + ((size_t(b) * a.n_q + row0 + r) * a.hq + h) * D + g * DH;
#pragma unroll
      for (int q = 0; q < DH / 32; ++q) {
        uint32_t x0[32], x1[32];
        FLUX_TMEM_LD32(o0 + q * 32, x0);
        if (two) {
          FLUX_TMEM_LD32(o0 + 128 + q * 32, x1);
        }
        tmem_wait_ld();
        float f[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          f[i] = two ? fmaf(__uint_as_float(x0[i]), w0, __uint_as_float(x1[i]) * w1)
                     : __uint_as_float(x0[i]) * w0;
        if (real_row) {
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            uint4 w;
            w.x = pack_bf16x2(f[8 * x + 0], f[8 * x + 1]);
            w.y = pack_bf16x2(f[8 * x + 2], f[8 * x + 3]);
            w.z = pack_bf16x2(f[8 * x + 4], f[8 * x + 5]);
            w.w = pack_bf16x2(f[8 * x + 6], f[8 * x + 7]);
            *reinterpret_cast<uint4*>(dst + q * 32 + x * 8) = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ tile schedule query

// The KV tiles the prefill kernel visits for every query tile, computed by the same
// plan_for / tile_needs_mask calls the kernel makes (flux_prefill_tile_plan).
__global__ void __launch_bounds__(128) prefill_tile_plan_kernel(const PrefillArgs a, int32_t* tiles,
                                                                int max_tiles) {
  const int m_tile = blockIdx.x, b = blockIdx.y;
  int rows, q_start;
  bool ok;
  const TilePlan p = plan_for(a, b, m_tile, rows, q_start, ok);
  int32_t* out = tiles + (size_t(b) * a.n_mtiles + m_tile) * max_tiles;
  for (int i = threadIdx.x; i < max_tiles; i += blockDim.x) {
    int v = -1;
    if (ok && i < p.n_tiles) {
      const int k0 = tile_key0(p, i);
      v = (k0 / BN) | (tile_needs_mask(p, k0) ? int(kTilePlanMasked) : 0);
    }
    out[i] = v;
  }
  if (!ok && threadIdx.x == 0 && m_tile == 0) atomicOr(a.status, kStatusBadLength);
}

// ------------------------------------------------------------------ host side

template <int D>
cudaError_t launch_prefill_t(const AttnGeom& g, const PrefillArgs& a, const uint16_t* q,
                             const uint16_t* k_cache, const uint16_t* v_cache, int batch,
                             cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  // Q: [B][n_q][Hq][D] as 4-D (D, Hq, n_q, B); box 64 x 1 x 128 x 1
  const cuuint64_t qd[4] = {cuuint64_t(D), cuuint64_t(g.hq), cuuint64_t(a.n_q), cuuint64_t(batch)};
  const cuuint64_t qs[3] = {cuuint64_t(D) * 2, cuuint64_t(g.hq) * D * 2,
                            cuuint64_t(a.n_q) * g.hq * D * 2};
  const cuuint32_t qbox[4] = {64, 1, BM, 1};
  // K, V: [B][Hkv][cap][D] as 3-D (D, cap, B*Hkv); box 64 x 128 x 1
  const cuuint64_t kd[3] = {cuuint64_t(D), cuuint64_t(a.capacity), cuuint64_t(batch) * g.hkv};
  const cuuint64_t ks[2] = {cuuint64_t(D) * 2, cuuint64_t(a.capacity) * D * 2};
  const cuuint32_t kbox[3] = {64, BN, 1};
  if (!make_map(&mq, q, 4, qd, qs, qbox) || !make_map(&mk, k_cache, 3, kd, ks, kbox) ||
      !make_map(&mv, v_cache, 3, kd, ks, kbox))
    return cudaErrorInvalidValue;
  const uint32_t smem = Smem<D>::bytes;
  cudaError_t err =
      cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return err;
  const dim3 grid(g.hq, a.n_mtiles, batch);
  prefill_kernel<D><<<grid, kThreads, smem, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

PrefillArgs prefill_args(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                         const int32_t* seq_len, int capacity, int n_q, uint16_t* o,
                         unsigned* status) {
  PrefillArgs a;
  a.fa_mask = fa_mask;
  a.mask_words = g.mask_words;
  a.layer = layer;
  a.seq_len = seq_len;
  a.capacity = capacity;
  a.n_q = n_q;
  a.hq = g.hq;
  a.hkv = g.hkv;
  a.block = g.block;
  a.sink = g.sink;
  a.window = g.window;
  a.n_mtiles = (n_q + BM - 1) / BM;
  a.scale_log2 = float(1.4426950408889634 / sqrt(double(g.head_dim)));
  a.o = o;
  a.status = status;
  return a;
}

}  // namespace

cudaError_t launch_prefill(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                           const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                           const int32_t* seq_len, int batch, int capacity, int n_q, uint16_t* o,
                           unsigned* status, cudaStream_t stream) {
  const PrefillArgs a = prefill_args(g, layer, fa_mask, seq_len, capacity, n_q, o, status);
  if (a.n_mtiles > 65535) return cudaErrorInvalidValue;
  if (g.head_dim == 128) return launch_prefill_t<128>(g, a, q, k_cache, v_cache, batch, stream);
  if (g.head_dim == 64) return launch_prefill_t<64>(g, a, q, k_cache, v_cache, batch, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_tile_plan(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                                     const int32_t* seq_len, int batch, int capacity, int n_q,
                                     int32_t* tiles, int max_tiles, unsigned* status,
                                     cudaStream_t stream) {
  const PrefillArgs a = prefill_args(g, layer, fa_mask, seq_len, capacity, n_q, nullptr, status);
  if (a.n_mtiles > 65535) return cudaErrorInvalidValue;
  prefill_tile_plan_kernel<<<dim3(a.n_mtiles, batch), 128, 0, stream>>>(a, tiles, max_tiles);
  return cudaGetLastError();
}

}  // namespace flux
