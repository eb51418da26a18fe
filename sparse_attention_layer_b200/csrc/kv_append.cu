// KV-cache append for the contiguous per-layer cache [B][Hkv][cap][d] (bf16).
//
// New rows arrive token-major ([B][n][Hkv][d], the layout a QKV projection writes)
// and land head-major in the cache, so that every (sequence, KV head) keeps its keys
// in one contiguous byte range -- the property the decode bulk copies and the prefill
// TMA boxes rely on (the pages' "contiguous memory access" of layer-level routing).
//
// Large appends (prefill) take two launches: the copy reads seq_len[b] as the write
// position; the second launch advances seq_len[b], so no copy CTA can observe a
// half-updated length.  Both use programmatic dependent launch, so the second grid is
// already scheduled when the first completes.  Small appends (decode: a few rows per sequence) take one: a
// single CTA per sequence copies its rows and then advances seq_len[b] itself after a
// CTA barrier; it is launched with programmatic dependent launch, like the decode
// kernels after it.  A sequence that would pass the capacity is skipped and
// FLUX_DEVICE_CAPACITY is set.
//
// SA ring caches (decode-time KV eviction of layers routed to SA): sink rows stay in
// place and position p >= sink lives in row sink + (p - sink) mod ring_rows, so with
// ring_rows >= window every key an SA decode query can see is kept.  Compaction moves
// a prefilled full cache into that layout; the ring append writes new rows there.
#include "flux_device.cuh"
#include "flux_internal.h"

namespace flux {
namespace {

__global__ void __launch_bounds__(256) kv_append_copy_kernel(
    uint16_t* __restrict__ k_cache, uint16_t* __restrict__ v_cache,
    const int32_t* __restrict__ seq_len, int capacity, const uint16_t* __restrict__ k_new,
    const uint16_t* __restrict__ v_new, int n_new, int hkv, int chunks_per_row,
    unsigned* status) {
  pdl_trigger();  // the length update may be scheduled; it waits for this grid
  pdl_wait();     // seq_len and the new rows may come from earlier kernels
  const int b = blockIdx.y;
  const int start = seq_len[b];
  if (start < 0 || start + n_new > capacity) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, kStatusCapacity);
    return;
  }
  const long long per_seq = (long long)n_new * hkv * chunks_per_row;
  const size_t row_elems = size_t(chunks_per_row) * 8;
  const uint4* ks = reinterpret_cast<const uint4*>(k_new) + size_t(b) * per_seq;
  const uint4* vs = reinterpret_cast<const uint4*>(v_new) + size_t(b) * per_seq;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < per_seq;
       i += (long long)gridDim.x * blockDim.x) {
    const int ch = int(i % chunks_per_row);
    const long long rest = i / chunks_per_row;
    const int kvh = int(rest % hkv);
    const int tok = int(rest / hkv);
    if (!FLUX_IN_BOUNDS(start + tok < capacity, status)) continue;
    const size_t dst = ((size_t(b) * hkv + kvh) * capacity + start + tok) * row_elems + ch * 8;
    const uint4 kv = __ldg(ks + i);
    const uint4 vv = __ldg(vs + i);
    *reinterpret_cast<uint4*>(k_cache + dst) = kv;
    *reinterpret_cast<uint4*>(v_cache + dst) = vv;
  }
}

// One CTA per sequence: copy the rows, then advance the length (read by every thread
// before the barrier, written by one thread after it).
__global__ void __launch_bounds__(256) kv_append_fused_kernel(
    uint16_t* __restrict__ k_cache, uint16_t* __restrict__ v_cache, int32_t* seq_len,
    int capacity, const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
    int n_new, int hkv, int chunks_per_row, unsigned* status) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  const int start = seq_len[b];
  const bool fits = start >= 0 && start + n_new <= capacity;
  if (fits) {
    const int per_seq = n_new * hkv * chunks_per_row;
    const size_t row_elems = size_t(chunks_per_row) * 8;
    const uint4* ks = reinterpret_cast<const uint4*>(k_new) + size_t(b) * per_seq;
    const uint4* vs = reinterpret_cast<const uint4*>(v_new) + size_t(b) * per_seq;
    for (int i = threadIdx.x; i < per_seq; i += blockDim.x) {
      const int ch = i % chunks_per_row;
      const int rest = i / chunks_per_row;
      const int kvh = rest % hkv;
      const int tok = rest / hkv;
      if (!FLUX_IN_BOUNDS(start + tok < capacity, status)) continue;
      const size_t dst = ((size_t(b) * hkv + kvh) * capacity + start + tok) * row_elems + ch * 8;
      *reinterpret_cast<uint4*>(k_cache + dst) = __ldg(ks + i);
      *reinterpret_cast<uint4*>(v_cache + dst) = __ldg(vs + i);
    }
  } else if (threadIdx.x == 0) {
    atomicOr(status, kStatusCapacity);
  }
  __syncthreads();
  if (threadIdx.x == 0 && fits) seq_len[b] = start + n_new;
}

__global__ void kv_append_advance_kernel(int32_t* seq_len, int batch, int capacity, int n_new) {
  pdl_trigger();
  pdl_wait();  // every copy CTA has read its start (the copy grid has completed)
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  const int start = seq_len[b];
  if (start >= 0 && start + n_new <= capacity) seq_len[b] = start + n_new;
}

// Physical row of logical position p in an SA ring cache (sink + ring_rows rows).
__device__ __forceinline__ int ring_slot(int p, int sink, int ring_rows) {
  return p < sink ? p : sink + (p - sink) % ring_rows;
}

// Rows [seq_len[b], seq_len[b] + n_new) into their ring slots; n_new <= ring_rows, so
// the new rows never share a slot.
__global__ void __launch_bounds__(256) kv_append_ring_kernel(
    uint16_t* __restrict__ k_ring, uint16_t* __restrict__ v_ring,
    const int32_t* __restrict__ seq_len, int sink, int ring_rows,
    const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new, int n_new, int hkv,
    int chunks_per_row, unsigned* status) {
  const int b = blockIdx.y;
  const int start = seq_len[b];
  if (start < 0) return;
  const int rows = sink + ring_rows;
  const long long per_seq = (long long)n_new * hkv * chunks_per_row;
  const size_t row_elems = size_t(chunks_per_row) * 8;
  const uint4* ks = reinterpret_cast<const uint4*>(k_new) + size_t(b) * per_seq;
  const uint4* vs = reinterpret_cast<const uint4*>(v_new) + size_t(b) * per_seq;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < per_seq;
       i += (long long)gridDim.x * blockDim.x) {
    const int ch = int(i % chunks_per_row);
    const long long rest = i / chunks_per_row;
    const int kvh = int(rest % hkv);
    const int tok = int(rest / hkv);
    const int slot = ring_slot(start + tok, sink, ring_rows);
    if (!FLUX_IN_BOUNDS(slot >= 0 && slot < rows, status)) continue;
    const size_t dst = ((size_t(b) * hkv + kvh) * rows + slot) * row_elems + ch * 8;
    *reinterpret_cast<uint4*>(k_ring + dst) = __ldg(ks + i);
    *reinterpret_cast<uint4*>(v_ring + dst) = __ldg(vs + i);
  }
}

// Ring append of a few rows: one CTA per sequence, then it advances the length.
__global__ void __launch_bounds__(256) kv_append_ring_fused_kernel(
    uint16_t* __restrict__ k_ring, uint16_t* __restrict__ v_ring, int32_t* seq_len, int sink,
    int ring_rows, const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
    int n_new, int hkv, int chunks_per_row, unsigned* status) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  const int start = seq_len[b];
  if (start >= 0) {
    const int rows = sink + ring_rows;
    const int per_seq = n_new * hkv * chunks_per_row;
    const size_t row_elems = size_t(chunks_per_row) * 8;
    const uint4* ks = reinterpret_cast<const uint4*>(k_new) + size_t(b) * per_seq;
    const uint4* vs = reinterpret_cast<const uint4*>(v_new) + size_t(b) * per_seq;
    for (int i = threadIdx.x; i < per_seq; i += blockDim.x) {
      const int ch = i % chunks_per_row;
      const int rest = i / chunks_per_row;
      const int kvh = rest % hkv;
      const int tok = rest / hkv;
      const int slot = ring_slot(start + tok, sink, ring_rows);
      if (!FLUX_IN_BOUNDS(slot >= 0 && slot < rows, status)) continue;
      const size_t dst = ((size_t(b) * hkv + kvh) * rows + slot) * row_elems + ch * 8;
      *reinterpret_cast<uint4*>(k_ring + dst) = __ldg(ks + i);
      *reinterpret_cast<uint4*>(v_ring + dst) = __ldg(vs + i);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && start >= 0) seq_len[b] = start + n_new;
}

__global__ void kv_advance_unbounded_kernel(int32_t* seq_len, int batch, int n_new) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch && seq_len[b] >= 0) seq_len[b] += n_new;
}

// Retained rows of a full cache -- the sink rows and the last ring_rows positions past
// the sink -- copied to their ring slots.
__global__ void __launch_bounds__(256) kv_compact_ring_kernel(
    const uint16_t* __restrict__ k_cache, const uint16_t* __restrict__ v_cache, int capacity,
    const int32_t* __restrict__ seq_len, uint16_t* __restrict__ k_ring,
    uint16_t* __restrict__ v_ring, int sink, int ring_rows, int hkv, int chunks_per_row,
    unsigned* status) {
  const int b = blockIdx.y;
  const int T = seq_len[b];
  if (T < 0 || T > capacity) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, kStatusBadLength);
    return;
  }
  const int head = min(sink, T);
  const int tail0 = max(sink, T - ring_rows);
  const int n_ret = head + max(0, T - tail0);
  const int rows = sink + ring_rows;
  const long long total = (long long)n_ret * hkv * chunks_per_row;
  const size_t row_elems = size_t(chunks_per_row) * 8;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int ch = int(i % chunks_per_row);
    const long long rest = i / chunks_per_row;
    const int kvh = int(rest % hkv);
    const int r = int(rest / hkv);
    const int pos = r < head ? r : tail0 + (r - head);
    if (!FLUX_IN_BOUNDS(pos >= 0 && pos < capacity, status)) continue;
    const size_t src = ((size_t(b) * hkv + kvh) * capacity + pos) * row_elems + ch * 8;
    const size_t dst =
        ((size_t(b) * hkv + kvh) * rows + ring_slot(pos, sink, ring_rows)) * row_elems + ch * 8;
    *reinterpret_cast<uint4*>(k_ring + dst) = __ldg(reinterpret_cast<const uint4*>(k_cache + src));
    *reinterpret_cast<uint4*>(v_ring + dst) = __ldg(reinterpret_cast<const uint4*>(v_cache + src));
  }
}

}  // namespace

// Per-sequence rows (16-byte chunks) up to which one CTA per sequence does the append.
constexpr long long kFusedAppendChunks = 4096;

cudaError_t launch_kv_append_ring(const AttnGeom& g, uint16_t* k_ring, uint16_t* v_ring,
                                  int32_t* seq_len, int batch, int ring_rows,
                                  const uint16_t* k_new, const uint16_t* v_new, int n_new,
                                  unsigned* status, cudaStream_t stream) {
  const int chunks = g.head_dim / 8;
  const long long per_seq = (long long)n_new * g.hkv * chunks;
  if (per_seq <= kFusedAppendChunks)
    return launch_pdl(kv_append_ring_fused_kernel, dim3(batch), dim3(256), 0, stream, k_ring,
                      v_ring, seq_len, g.sink, ring_rows, k_new, v_new, n_new, g.hkv, chunks,
                      status);
  long long blocks = (per_seq + 255) / 256;
  const long long cap_blocks = (long long)device_sm_count() * 16 / (batch > 0 ? batch : 1) + 1;
  if (blocks > cap_blocks) blocks = cap_blocks;
  if (blocks < 1) blocks = 1;
  kv_append_ring_kernel<<<dim3(unsigned(blocks), batch), 256, 0, stream>>>(
      k_ring, v_ring, seq_len, g.sink, ring_rows, k_new, v_new, n_new, g.hkv, chunks, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  kv_advance_unbounded_kernel<<<(batch + 127) / 128, 128, 0, stream>>>(seq_len, batch, n_new);
  return cudaGetLastError();
}

cudaError_t launch_kv_compact_ring(const AttnGeom& g, const uint16_t* k_cache,
                                   const uint16_t* v_cache, int capacity, const int32_t* seq_len,
                                   int batch, uint16_t* k_ring, uint16_t* v_ring, int ring_rows,
                                   unsigned* status, cudaStream_t stream) {
  const int chunks = g.head_dim / 8;
  const long long per_seq = (long long)(g.sink + ring_rows) * g.hkv * chunks;
  long long blocks = (per_seq + 255) / 256;
  const long long cap_blocks = (long long)device_sm_count() * 16 / (batch > 0 ? batch : 1) + 1;
  if (blocks > cap_blocks) blocks = cap_blocks;
  if (blocks < 1) blocks = 1;
  kv_compact_ring_kernel<<<dim3(unsigned(blocks), batch), 256, 0, stream>>>(
      k_cache, v_cache, capacity, seq_len, k_ring, v_ring, g.sink, ring_rows, g.hkv, chunks,
      status);
  return cudaGetLastError();
}

cudaError_t launch_kv_append(const AttnGeom& g, uint16_t* k_cache, uint16_t* v_cache,
                             int32_t* seq_len, int batch, int capacity, const uint16_t* k_new,
                             const uint16_t* v_new, int n_new, unsigned* status,
                             cudaStream_t stream) {
  const int chunks = g.head_dim / 8;
  const long long per_seq = (long long)n_new * g.hkv * chunks;
  if (per_seq <= kFusedAppendChunks)
    return launch_pdl(kv_append_fused_kernel, dim3(batch), dim3(256), 0, stream, k_cache,
                      v_cache, seq_len, capacity, k_new, v_new, n_new, g.hkv, chunks, status);
  long long blocks = (per_seq + 255) / 256;
  const long long cap_blocks = (long long)device_sm_count() * 16 / (batch > 0 ? batch : 1) + 1;
  if (blocks > cap_blocks) blocks = cap_blocks;
  if (blocks < 1) blocks = 1;
  // both launches with programmatic dependent launch: each grid is scheduled while the
  // one before it drains and waits (griddepcontrol.wait) for it to complete
  cudaError_t err = launch_pdl(kv_append_copy_kernel, dim3(unsigned(blocks), batch), dim3(256),
                               0, stream, k_cache, v_cache, seq_len, capacity, k_new, v_new,
                               n_new, g.hkv, chunks, status);
  if (err != cudaSuccess) return err;
  return launch_pdl(kv_append_advance_kernel, dim3((batch + 127) / 128), dim3(128), 0, stream,
                    seq_len, batch, capacity, n_new);
}

}  // namespace flux
