// extern "C" entry points of libflux: argument validation, the device status word and
// dispatch to the kernel launchers.  Nothing here allocates device memory.
#include <math.h>
#include <stdio.h>

#include <atomic>
#include <mutex>

#include "../../include/flux.h"
#include "flux_device.cuh"
#include "flux_internal.h"

// Library-wide device status word (one per device context): kernels OR error bits
// into it instead of trapping; flux_get_device_status reads and clears it.
static __device__ unsigned int g_flux_status;

namespace flux {

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
unsigned* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Device address of the status word on the current device, looked up once.
unsigned* status_ptr() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_flux_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_status_ptr[dev];
}

__global__ void sa_block_ranges_kernel(int n_qblocks, int n_sink_blocks, int n_win_blocks,
                                       int32_t* ranges) {
  const int qb = blockIdx.x * blockDim.x + threadIdx.x;
  if (qb >= n_qblocks) return;
  const BlockRanges r = sa_key_blocks(qb, n_sink_blocks, n_win_blocks);
  ranges[3 * qb + 0] = r.sink_end;
  ranges[3 * qb + 1] = r.win_begin;
  ranges[3 * qb + 2] = r.win_end;
}

// One thread waits on an mbarrier that nothing arrives on, through the same bounded
// wait every pipeline wait in the library uses.
__global__ void selftest_wait_kernel(unsigned long long limit_ns, unsigned* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_addr(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  mbar_wait(b, 0, status, limit_ns);
}

// Bounds-guard self-test: a guard refuses index 16 of a 16-entry array.  The checked
// build records FLUX_DEVICE_BOUNDS; the plain build compiles the guard to true, and the
// index check that follows it keeps the access out either way.
__device__ unsigned g_bounds_probe[16];

__global__ void selftest_bounds_kernel(int index, unsigned* status) {
  const bool inside = index >= 0 && index < 16;
  if (FLUX_IN_BOUNDS(inside, status) && inside) g_bounds_probe[index] = 1u;
}

int validate_cfg(const flux_attn_cfg* c) {
  if (!c) return FLUX_ERR_INVALID_ARG;
  if (c->n_layers < 1 || c->n_layers > 1024) return FLUX_ERR_INVALID_ARG;
  if (c->n_q_heads < 1 || c->n_kv_heads < 1) return FLUX_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads != 0) return FLUX_ERR_INVALID_ARG;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FLUX_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return FLUX_ERR_UNSUPPORTED;
  if (c->block != 64 && c->block != 128) return FLUX_ERR_UNSUPPORTED;
  if (c->sink < 0 || c->sink % c->block != 0) return FLUX_ERR_INVALID_ARG;
  if (c->window < c->block || c->window % c->block != 0) return FLUX_ERR_INVALID_ARG;
  return FLUX_OK;
}

AttnGeom geom_of(const flux_attn_cfg* c) {
  AttnGeom g;
  g.n_layers = c->n_layers;
  g.mask_words = (c->n_layers + 31) / 32;
  g.hq = c->n_q_heads;
  g.hkv = c->n_kv_heads;
  g.head_dim = c->head_dim;
  g.block = c->block;
  g.sink = c->sink;
  g.window = c->window;
  return g;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? FLUX_OK : FLUX_ERR_CUDA; }

}  // namespace

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_sm_count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

cudaError_t launch_sa_block_ranges(const AttnGeom& g, int n_qblocks, int32_t* ranges,
                                   cudaStream_t stream) {
  sa_block_ranges_kernel<<<(n_qblocks + 127) / 128, 128, 0, stream>>>(
      n_qblocks, g.sink / g.block, g.window / g.block, ranges);
  return cudaGetLastError();
}

}  // namespace flux

using flux::aligned16;

extern "C" {

int32_t flux_mask_words(int32_t n_layers) { return n_layers <= 0 ? 0 : (n_layers + 31) / 32; }

int32_t flux_version(void) { return 100; }

const char* flux_status_string(int status) {
  switch (status) {
    case FLUX_OK: return "ok";
    case FLUX_ERR_INVALID_ARG: return "invalid argument";
    case FLUX_ERR_UNSUPPORTED: return "unsupported geometry (head_dim, block or group size)";
    case FLUX_ERR_CAPACITY: return "KV cache capacity exceeded";
    case FLUX_ERR_TIMEOUT: return "a device pipeline wait timed out";
    case FLUX_ERR_CUDA: return "CUDA runtime error";
    case FLUX_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int flux_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return FLUX_ERR_INVALID_ARG;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  flux::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)limit_us * 1000ull, status);
  return flux::cuda_status(cudaGetLastError());
}

int flux_selftest_bounds(void* stream) {
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  flux::selftest_bounds_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(16, status);
  return flux::cuda_status(cudaGetLastError());
}

int flux_build_checked(void) {
#ifdef FLUX_CHECKED
  return 1;
#else
  return 0;
#endif
}

int flux_get_device_status(void* stream, uint32_t* bits) {
  if (!bits) return FLUX_ERR_INVALID_ARG;
  unsigned* p = flux::status_ptr();
  if (!p) return FLUX_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, p, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(p, 0, sizeof(unsigned), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return FLUX_ERR_CUDA;
  *bits = host;
  return FLUX_OK;
}

int flux_route(const flux_router_weights* w, const uint16_t* xq, int32_t batch, int32_t seq,
               int32_t pool_len, float tau, uint32_t* fa_mask, double* logits, void* stream) {
  if (!w || !w->w1 || !w->w2 || !xq || !fa_mask) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || seq < 1) return FLUX_ERR_INVALID_ARG;
  if (w->hidden < 8 || w->hidden % 8 != 0 || w->hidden > flux::kRouterMaxHidden)
    return FLUX_ERR_INVALID_ARG;
  if (w->rank < 1 || w->rank > flux::kRouterMaxRank) return FLUX_ERR_INVALID_ARG;
  if (w->n_layers < 1 || w->n_layers > flux::kRouterMaxLayers) return FLUX_ERR_INVALID_ARG;
  if (!isfinite(tau)) return FLUX_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(w->w1)) return FLUX_ERR_INVALID_ARG;
  return flux::cuda_status(flux::launch_route(w->w1, w->b1, w->w2, w->b2, w->hidden, w->rank,
                                              w->n_layers, xq, batch, seq, pool_len, tau,
                                              fa_mask, logits, static_cast<cudaStream_t>(stream)));
}

int flux_kv_append(const flux_attn_cfg* cfg, uint16_t* k_cache, uint16_t* v_cache,
                   int32_t* seq_len, int32_t batch, int32_t capacity, const uint16_t* k_new,
                   const uint16_t* v_new, int32_t n_new, void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!k_cache || !v_cache || !seq_len || !k_new || !v_new) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || capacity < 1 || n_new < 0) return FLUX_ERR_INVALID_ARG;
  if (n_new > capacity) return FLUX_ERR_CAPACITY;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) || !aligned16(v_new))
    return FLUX_ERR_INVALID_ARG;
  if (n_new == 0) return FLUX_OK;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_kv_append(flux::geom_of(cfg), k_cache, v_cache, seq_len,
                                                  batch, capacity, k_new, v_new, n_new, status,
                                                  static_cast<cudaStream_t>(stream)));
}

int flux_prefill(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                 const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                 const int32_t* seq_len, int32_t batch, int32_t capacity, int32_t n_q,
                 uint16_t* o, void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!fa_mask || !q || !k_cache || !v_cache || !seq_len || !o) return FLUX_ERR_INVALID_ARG;
  if (layer < 0 || layer >= cfg->n_layers) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || capacity < 1 || n_q < 0 || n_q > capacity)
    return FLUX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
    return FLUX_ERR_INVALID_ARG;
  if (n_q == 0) return FLUX_OK;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_prefill(flux::geom_of(cfg), layer, fa_mask, q, k_cache,
                                                v_cache, seq_len, batch, capacity, n_q, o, status,
                                                static_cast<cudaStream_t>(stream)));
}

size_t flux_decode_workspace_size(const flux_attn_cfg* cfg, int32_t batch) {
  if (flux::validate_cfg(cfg) != FLUX_OK || batch < 1 || batch > flux::kDecMaxBatch) return 0;
  return flux::decode_workspace_bytes(flux::geom_of(cfg), batch);
}

int flux_decode(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                const int32_t* seq_len, int32_t batch, int32_t capacity, uint16_t* o,
                void* workspace, size_t workspace_bytes, void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!fa_mask || !q || !k_cache || !v_cache || !seq_len || !o) return FLUX_ERR_INVALID_ARG;
  if (layer < 0 || layer >= cfg->n_layers) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > flux::kDecMaxBatch || capacity < 1) return FLUX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return FLUX_ERR_INVALID_ARG;
  const flux::AttnGeom g = flux::geom_of(cfg);
  if (!workspace || workspace_bytes < flux::decode_workspace_bytes(g, batch) ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return FLUX_ERR_WORKSPACE;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_decode(g, layer, fa_mask, q, k_cache, v_cache, nullptr,
                                               nullptr, const_cast<int32_t*>(seq_len), batch,
                                               capacity, 0, o, workspace, status,
                                               static_cast<cudaStream_t>(stream)));
}

int flux_decode_append(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                       const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                       uint16_t* k_cache, uint16_t* v_cache, int32_t* seq_len, int32_t batch,
                       int32_t capacity, uint16_t* o, void* workspace, size_t workspace_bytes,
                       void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!fa_mask || !q || !k_new || !v_new || !k_cache || !v_cache || !seq_len || !o)
    return FLUX_ERR_INVALID_ARG;
  if (layer < 0 || layer >= cfg->n_layers) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > flux::kDecMaxBatch || capacity < 1) return FLUX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_new) ||
      !aligned16(v_new))
    return FLUX_ERR_INVALID_ARG;
  const flux::AttnGeom g = flux::geom_of(cfg);
  if (!workspace || workspace_bytes < flux::decode_workspace_bytes(g, batch) ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return FLUX_ERR_WORKSPACE;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_decode(g, layer, fa_mask, q, k_cache, v_cache, k_new,
                                               v_new, seq_len, batch, capacity, 0, o, workspace,
                                               status, static_cast<cudaStream_t>(stream)));
}

int flux_decode_static(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                       const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                       const int32_t* seq_len, int32_t batch, int32_t capacity, uint16_t* o,
                       void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!fa_mask || !q || !k_cache || !v_cache || !seq_len || !o) return FLUX_ERR_INVALID_ARG;
  if (layer < 0 || layer >= cfg->n_layers) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > flux::kDecMaxBatch || capacity < 1) return FLUX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return FLUX_ERR_INVALID_ARG;
  const flux::AttnGeom g = flux::geom_of(cfg);
  if (flux::decode_workspace_bytes(g, batch) > FLUX_DECODE_STATIC_SCRATCH_BYTES)
    return FLUX_ERR_WORKSPACE;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_decode_static(g, layer, fa_mask, q, k_cache, v_cache,
                                                      seq_len, batch, capacity, o, status,
                                                      static_cast<cudaStream_t>(stream)));
}

int flux_kv_compact_ring(const flux_attn_cfg* cfg, const uint16_t* k_cache,
                         const uint16_t* v_cache, int32_t capacity, const int32_t* seq_len,
                         int32_t batch, uint16_t* k_ring, uint16_t* v_ring, int32_t ring_rows,
                         void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!k_cache || !v_cache || !seq_len || !k_ring || !v_ring) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || capacity < 1) return FLUX_ERR_INVALID_ARG;
  if (ring_rows < cfg->window) return FLUX_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_ring) || !aligned16(v_ring))
    return FLUX_ERR_INVALID_ARG;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_kv_compact_ring(flux::geom_of(cfg), k_cache, v_cache,
                                                        capacity, seq_len, batch, k_ring, v_ring,
                                                        ring_rows, status,
                                                        static_cast<cudaStream_t>(stream)));
}

int flux_kv_append_ring(const flux_attn_cfg* cfg, uint16_t* k_ring, uint16_t* v_ring,
                        int32_t* seq_len, int32_t batch, int32_t ring_rows,
                        const uint16_t* k_new, const uint16_t* v_new, int32_t n_new,
                        void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!k_ring || !v_ring || !seq_len || !k_new || !v_new) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || n_new < 0) return FLUX_ERR_INVALID_ARG;
  if (ring_rows < cfg->window || n_new > ring_rows) return FLUX_ERR_INVALID_ARG;
  if (!aligned16(k_ring) || !aligned16(v_ring) || !aligned16(k_new) || !aligned16(v_new))
    return FLUX_ERR_INVALID_ARG;
  if (n_new == 0) return FLUX_OK;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_kv_append_ring(flux::geom_of(cfg), k_ring, v_ring,
                                                       seq_len, batch, ring_rows, k_new, v_new,
                                                       n_new, status,
                                                       static_cast<cudaStream_t>(stream)));
}

int flux_decode_ring(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                     const uint16_t* q, const uint16_t* k_ring, const uint16_t* v_ring,
                     const int32_t* seq_len, int32_t batch, int32_t ring_rows, uint16_t* o,
                     void* workspace, size_t workspace_bytes, void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!fa_mask || !q || !k_ring || !v_ring || !seq_len || !o) return FLUX_ERR_INVALID_ARG;
  if (layer < 0 || layer >= cfg->n_layers) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > flux::kDecMaxBatch) return FLUX_ERR_INVALID_ARG;
  if (ring_rows < cfg->window) return FLUX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_ring) || !aligned16(v_ring)) return FLUX_ERR_INVALID_ARG;
  const flux::AttnGeom g = flux::geom_of(cfg);
  if (!workspace || workspace_bytes < flux::decode_workspace_bytes(g, batch) ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return FLUX_ERR_WORKSPACE;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_decode(g, layer, fa_mask, q, k_ring, v_ring, nullptr,
                                               nullptr, const_cast<int32_t*>(seq_len), batch, 0,
                                               ring_rows, o, workspace, status,
                                               static_cast<cudaStream_t>(stream)));
}

int flux_decode_append_ring(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                            const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                            uint16_t* k_ring, uint16_t* v_ring, int32_t* seq_len, int32_t batch,
                            int32_t ring_rows, uint16_t* o, void* workspace,
                            size_t workspace_bytes, void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!fa_mask || !q || !k_new || !v_new || !k_ring || !v_ring || !seq_len || !o)
    return FLUX_ERR_INVALID_ARG;
  if (layer < 0 || layer >= cfg->n_layers) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > flux::kDecMaxBatch) return FLUX_ERR_INVALID_ARG;
  if (ring_rows < cfg->window) return FLUX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_ring) || !aligned16(v_ring) || !aligned16(k_new) ||
      !aligned16(v_new))
    return FLUX_ERR_INVALID_ARG;
  const flux::AttnGeom g = flux::geom_of(cfg);
  if (!workspace || workspace_bytes < flux::decode_workspace_bytes(g, batch) ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return FLUX_ERR_WORKSPACE;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_decode(g, layer, fa_mask, q, k_ring, v_ring, k_new,
                                               v_new, seq_len, batch, 0, ring_rows, o, workspace,
                                               status, static_cast<cudaStream_t>(stream)));
}

int flux_prefill_tile_plan(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                           const int32_t* seq_len, int32_t batch, int32_t capacity, int32_t n_q,
                           int32_t* tiles, int32_t max_tiles, void* stream) {
  static_assert(FLUX_TILE_MASKED == flux::kTilePlanMasked, "tile-plan flag");
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!fa_mask || !seq_len || !tiles) return FLUX_ERR_INVALID_ARG;
  if (layer < 0 || layer >= cfg->n_layers) return FLUX_ERR_INVALID_ARG;
  if (batch < 1 || batch > 65535 || capacity < 1 || n_q < 0 || n_q > capacity)
    return FLUX_ERR_INVALID_ARG;
  if (max_tiles < (capacity + 127) / 128) return FLUX_ERR_INVALID_ARG;
  if (n_q == 0) return FLUX_OK;
  unsigned* status = flux::status_ptr();
  if (!status) return FLUX_ERR_CUDA;
  return flux::cuda_status(flux::launch_prefill_tile_plan(
      flux::geom_of(cfg), layer, fa_mask, seq_len, batch, capacity, n_q, tiles, max_tiles, status,
      static_cast<cudaStream_t>(stream)));
}

int flux_sa_block_ranges(const flux_attn_cfg* cfg, int32_t n_qblocks, int32_t* ranges,
                         void* stream) {
  const int st = flux::validate_cfg(cfg);
  if (st != FLUX_OK) return st;
  if (!ranges || n_qblocks < 0) return FLUX_ERR_INVALID_ARG;
  if (n_qblocks == 0) return FLUX_OK;
  return flux::cuda_status(flux::launch_sa_block_ranges(flux::geom_of(cfg), n_qblocks, ranges,
                                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
