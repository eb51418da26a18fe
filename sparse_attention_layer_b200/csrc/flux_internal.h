// Internal interface between the C-ABI layer (flux_api.cu) and the kernel files.
// Arguments arrive here already validated; launchers return a cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace flux {

struct AttnGeom {
  int n_layers, mask_words, hq, hkv, head_dim, block, sink, window;
};

// Launch with programmatic dependent launch allowed (the kernel must call pdl_wait()
// before its first global memory access): its CTAs can be scheduled while the
// previous kernel on the stream drains, hiding launch latency between the short
// kernels of a decode step.
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<A&&>(args)...);
}

// ----- decode (split-KV; split pairs are merged inside the same launch)
constexpr int kDecMaxSplits = 64;   // splits per (sequence, KV head)
constexpr int kDecStageKeys = 128;  // keys per decode pipeline stage
constexpr int kDecMaxBatch = 1024;
// Arrival counters at the start of every decode workspace: one per CTA of the grid
// (a split pair counts its pieces in the counter of the CTA holding its first piece),
// then one for the appending variant's length update; padded to 256 bytes.
constexpr int kDecCtaCounters = 1025;
constexpr size_t kDecCounterBytes = (kDecCtaCounters * 4 + 255) / 256 * 256;

size_t decode_workspace_bytes(const AttnGeom& g, int batch);

// ring_rows == 0: contiguous cache of `capacity` rows per (sequence, KV head);
// ring_rows > 0: SA ring cache of sink + ring_rows rows (capacity unused).
// k_new / v_new non-null: the appending variant (one new row per sequence, seq_len
// advanced); null: seq_len is only read.
cudaError_t launch_decode(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                          const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                          const uint16_t* k_new, const uint16_t* v_new, int32_t* seq_len,
                          int batch, int capacity, int ring_rows, uint16_t* o, void* workspace,
                          unsigned* status, cudaStream_t stream);

// Decode with the library's own file-scope scratch array instead of a caller
// workspace (flux_decode_static).  Its size is FLUX_DECODE_STATIC_SCRATCH_BYTES.
cudaError_t launch_decode_static(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                                 const uint16_t* q, const uint16_t* k_cache,
                                 const uint16_t* v_cache, const int32_t* seq_len, int batch,
                                 int capacity, uint16_t* o, unsigned* status,
                                 cudaStream_t stream);

// ----- KV append
cudaError_t launch_kv_append(const AttnGeom& g, uint16_t* k_cache, uint16_t* v_cache,
                             int32_t* seq_len, int batch, int capacity, const uint16_t* k_new,
                             const uint16_t* v_new, int n_new, unsigned* status,
                             cudaStream_t stream);

// SA ring caches: compaction from a full cache, and append
cudaError_t launch_kv_compact_ring(const AttnGeom& g, const uint16_t* k_cache,
                                   const uint16_t* v_cache, int capacity, const int32_t* seq_len,
                                   int batch, uint16_t* k_ring, uint16_t* v_ring, int ring_rows,
                                   unsigned* status, cudaStream_t stream);
cudaError_t launch_kv_append_ring(const AttnGeom& g, uint16_t* k_ring, uint16_t* v_ring,
                                  int32_t* seq_len, int batch, int ring_rows,
                                  const uint16_t* k_new, const uint16_t* v_new, int n_new,
                                  unsigned* status, cudaStream_t stream);

// ----- router
constexpr int kRouterMaxHidden = 16384;
constexpr int kRouterMaxRank = 1024;
constexpr int kRouterMaxLayers = 1024;

cudaError_t launch_route(const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                         const uint16_t* b2, int hidden, int rank, int n_layers,
                         const uint16_t* xq, int batch, int seq, int pool_len, float tau,
                         uint32_t* fa_mask, double* logits, cudaStream_t stream);

// ----- prefill (tcgen05 / TMEM / TMA)
cudaError_t launch_prefill(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                           const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                           const int32_t* seq_len, int batch, int capacity, int n_q, uint16_t* o,
                           unsigned* status, cudaStream_t stream);

// The KV tiles flux_prefill visits per query tile (flux_prefill_tile_plan); entries
// carry kTilePlanMasked when the kernel masks keys of the tile.
constexpr unsigned kTilePlanMasked = 0x40000000u;
cudaError_t launch_prefill_tile_plan(const AttnGeom& g, int layer, const uint32_t* fa_mask,
                                     const int32_t* seq_len, int batch, int capacity, int n_q,
                                     int32_t* tiles, int max_tiles, unsigned* status,
                                     cudaStream_t stream);

// ----- SA block ranges (the block indices the kernels use)
cudaError_t launch_sa_block_ranges(const AttnGeom& g, int n_qblocks, int32_t* ranges,
                                   cudaStream_t stream);

int device_sm_count();

}  // namespace flux
