/*
 * flux.h -- C ABI of the B200 (sm_100a) hybrid-attention library "libflux".
 *
 * The library runs the hot path of Flux Attention ("Flux Attention: Context-Aware
 * Hybrid Attention for Efficient LLMs Inference", arXiv 2604.07394):
 *
 *   flux_route      Layer Router (Figure 2): pool the query hidden states x_Q over
 *                   the sequence boundaries (Figure 8), run a two-layer MLP and take
 *                   a hard FA/SA decision per layer (Table 19 caption), written as a
 *                   device-side bitmask.  The routing is decided once at prefill and
 *                   reused by every decode step (Table 3, Flux Attention row).
 *   flux_kv_append  write new K/V rows into a layer's contiguous KV cache.
 *   flux_prefill    causal grouped-query attention of a prompt, Full Attention (FA)
 *                   or streaming Sparse Attention (SA = attention-sink blocks plus a
 *                   local window of KV blocks; Table 6, Figure 1 caption), chosen on
 *                   the device from the layer's bit in the routing mask.
 *   flux_decode     one autoregressive step of the same attention over the cache
 *                   (split-KV partial softmax, merged by the last CTA of each split);
 *                   flux_decode_append also appends the step's new K/V row.
 *
 * Conventions shared by every call
 *   - Every pointer argument that names tensor data is a DEVICE pointer owned by the
 *     caller.  The library allocates and frees nothing; scratch space (the decode
 *     workspace, zero-filled once by the caller) is passed in by the caller.
 *   - bf16 tensors are passed as uint16_t (raw bf16 bit patterns), row-major, densely
 *     packed, with the layouts stated per call.  Base pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Every compute call is asynchronous on that stream and returns a flux_status.
 *     Host-detected errors (bad arguments, unsupported shapes) return before any
 *     launch.  Errors the device detects while running (a KV append past capacity, a
 *     pipeline wait that ran out of time) never trap: the kernel skips the faulty
 *     work, sets a bit in the library's device status word and returns; read and
 *     clear that word with flux_get_device_status().
 *   - Geometry: head_dim d in {64, 128}; SA block size in {64, 128}; sink and window
 *     are multiples of the block size, window >= block.  Query head h reads KV head
 *     h / (n_q_heads / n_kv_heads).  Softmax scale is 1/sqrt(d).
 *   - SA visibility (block-granular reading of the streaming pattern): from query
 *     position t (query block qb = t / block) key j is visible iff j <= t and its
 *     block jb = j / block satisfies jb < sink/block or jb >= qb - window/block + 1.
 *     FA visibility is j <= t.
 */
#ifndef FLUX_H
#define FLUX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes of every call. */
typedef enum flux_status {
  FLUX_OK = 0,
  FLUX_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent shapes */
  FLUX_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim, block or group size */
  FLUX_ERR_CAPACITY = 3,     /* host-visible capacity violation (n_new > capacity) */
  FLUX_ERR_TIMEOUT = 4,      /* reported through the device status word only */
  FLUX_ERR_CUDA = 5,         /* a CUDA runtime call or a kernel launch failed */
  FLUX_ERR_WORKSPACE = 6     /* workspace missing or smaller than required */
} flux_status;

/* Bits of the device status word (flux_get_device_status). */
#define FLUX_DEVICE_CAPACITY 0x1u /* a kv_append would pass the capacity; skipped */
#define FLUX_DEVICE_TIMEOUT 0x2u  /* a pipeline wait ran out of time; output invalid */
#define FLUX_DEVICE_BAD_LENGTH 0x4u /* seq_len < n_q in prefill, or seq_len > capacity */
#define FLUX_DEVICE_RING_ROUTE 0x8u /* flux_decode_ring saw a sequence routed to FA */
#define FLUX_DEVICE_LAYOUT 0x10u    /* prefill: dynamic shared memory not 1024-byte aligned;
                                       nothing computed (never seen on B200) */
#define FLUX_DEVICE_BOUNDS 0x20u    /* checked build only: a guarded global access (decode
                                       copies, cache and workspace writes, KV appends)
                                       would have left its buffer; it was skipped */

/* Attention geometry of one model; the same struct serves every layer. */
typedef struct flux_attn_cfg {
  int32_t n_layers;   /* layers covered by the routing mask (1..1024)             */
  int32_t n_q_heads;  /* Hq                                                        */
  int32_t n_kv_heads; /* Hkv; Hq % Hkv == 0; group Hq/Hkv in {1, 2, 4, 8}          */
  int32_t head_dim;   /* d in {64, 128}                                            */
  int32_t block;      /* SA block size in keys, 64 or 128                          */
  int32_t sink;       /* SA attention-sink tokens, multiple of block, >= 0         */
  int32_t window;     /* SA local window tokens, multiple of block, >= block       */
} flux_attn_cfg;

/* Layer Router parameters (Figure 2), bf16, (out, in) layout of a linear layer. */
typedef struct flux_router_weights {
  const uint16_t* w1; /* [rank][hidden]                                  */
  const uint16_t* b1; /* [rank], or NULL for a zero bias                 */
  const uint16_t* w2; /* [n_layers][rank]                                */
  const uint16_t* b2; /* [n_layers], or NULL for a zero bias             */
  int32_t hidden;     /* h, a multiple of 8, <= 16384                    */
  int32_t rank;       /* r, 1..1024                                      */
  int32_t n_layers;   /* 1..1024                                         */
} flux_router_weights;

/* Number of uint32 words per sequence in a routing mask: ceil(n_layers / 32). */
int32_t flux_mask_words(int32_t n_layers);

/*
 * flux_route -- Layer Router (Figure 2; pooling window of Figure 8; hard decision of
 * the per-layer soft FA probability, Table 19 caption).
 *   xq       [batch][seq][hidden] bf16 query hidden states x_Q.
 *   pool_len L: mean over the first ceil(L/2) and the last floor(L/2) tokens; L <= 0
 *            or seq <= L pools every token.
 *   z        = W2 relu(W1 mean(x_Q) + b1) + b2, accumulated in fp64 on the device.
 *   fa_mask  [batch][flux_mask_words(n_layers)] uint32, written: bit (l % 32) of word
 *            l / 32 is 1 iff z_l > tau (layer l runs FA), 0 for SA; unused bits 0.
 *   logits   optional [batch][n_layers] double, the z values (NULL to skip).
 * One kernel launch (a cluster of CTAs per sequence); reads only the pooled rows.
 */
int flux_route(const flux_router_weights* w, const uint16_t* xq, int32_t batch,
               int32_t seq, int32_t pool_len, float tau, uint32_t* fa_mask,
               double* logits, void* stream);

/*
 * flux_kv_append -- append n_new rows per sequence to one layer's KV cache: the
 * persistent decode-time KV cache whose per-layer size Tables 15/16 report (the keys
 * and values every later FA or SA query of that layer reads).
 *   k_cache, v_cache  [batch][n_kv_heads][capacity][head_dim] bf16 (read/write).
 *   seq_len           [batch] int32 (read/write): rows are written at positions
 *                     [seq_len[b], seq_len[b] + n_new) and seq_len[b] += n_new.
 *   k_new, v_new      [batch][n_new][n_kv_heads][head_dim] bf16.
 * A sequence with seq_len[b] + n_new > capacity is left untouched (rows and
 * length) and FLUX_DEVICE_CAPACITY is set.  Up to 4096 16-byte chunks of new rows per
 * sequence (decode-sized appends): one launch, a CTA per sequence that copies its rows
 * and then advances its length (programmatic dependent launch, so it may start while
 * the previous kernel on the stream drains); larger appends: a copy launch, then a
 * length-update launch.
 */
int flux_kv_append(const flux_attn_cfg* cfg, uint16_t* k_cache, uint16_t* v_cache,
                   int32_t* seq_len, int32_t batch, int32_t capacity,
                   const uint16_t* k_new, const uint16_t* v_new, int32_t n_new,
                   void* stream);

/*
 * flux_prefill -- attention of n_q prompt queries per sequence for layer `layer`
 * (Figure 2 routing; FA = causal dense path, SA = streaming sink + window path of
 * Table 6), after their K/V rows have been appended.
 *   fa_mask  [batch][flux_mask_words(n_layers)] from flux_route (or the caller).
 *   q        [batch][n_q][n_q_heads][head_dim] bf16; query i of sequence b sits at
 *            position t = seq_len[b] - n_q + i.
 *   k_cache, v_cache, seq_len  as written by flux_kv_append (seq_len read only).
 *   o        [batch][n_q][n_q_heads][head_dim] bf16, written.
 * tcgen05 / TMEM tensor-core kernel fed by TMA (two softmax warpgroups, P staged in
 * shared memory; 226 KB of shared memory per CTA at head_dim 128); SA visits only the
 * sink and window KV tiles.  seq_len[b] < n_q or > capacity sets
 * FLUX_DEVICE_BAD_LENGTH and leaves that sequence's output unwritten.
 */
int flux_prefill(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                 const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                 const int32_t* seq_len, int32_t batch, int32_t capacity, int32_t n_q,
                 uint16_t* o, void* stream);

/* Bytes of device workspace flux_decode needs for this geometry and batch: arrival
 * counters at fixed offsets (4352 bytes), then split partial results. */
size_t flux_decode_workspace_size(const flux_attn_cfg* cfg, int32_t batch);

/*
 * flux_decode -- one decode step for layer `layer` (Table 3: the prefill route is
 * reused), after the new token's K/V row has been appended.
 *   q   [batch][n_q_heads][head_dim] bf16, the query at position seq_len[b] - 1.
 *   o   [batch][n_q_heads][head_dim] bf16, written.
 *   workspace  caller-owned device buffer of >= flux_decode_workspace_size() bytes,
 *              ZERO-FILLED ONCE before its first use (cudaMemset): its arrival
 *              counters must start at zero, and every call leaves them at zero, so one
 *              workspace serves any later call of any geometry that fits it.  Calls
 *              that share a workspace must not overlap on the GPU.  After a call that
 *              reported FLUX_DEVICE_TIMEOUT, zero it again.
 * One kernel launch (programmatic dependent launch, so it may start while the
 * previous kernel on the stream drains): a persistent split-KV kernel (bulk-copy
 * pipeline, 128-bit shared loads, warp-shuffle reductions); the CTA that finishes a
 * split pair merges its partial results.  SA reads only the sink and window rows.
 * seq_len[b] == 0 writes zeros; seq_len[b] > capacity sets FLUX_DEVICE_BAD_LENGTH.
 */
int flux_decode(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                const int32_t* seq_len, int32_t batch, int32_t capacity, uint16_t* o,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * flux_decode_append -- flux_kv_append of one new row per sequence followed by
 * flux_decode, in one kernel launch (the decode step of one layer: Table 3's decode
 * reusing the prefill route, over the persistent KV cache of Tables 15/16).
 *   k_new, v_new  [batch][1][n_kv_heads][head_dim] bf16, the step's new key and value.
 *   k_cache, v_cache, seq_len  read and written: for every sequence with room
 *                  (seq_len[b] < capacity) the new row is written at position
 *                  seq_len[b] and seq_len[b] is advanced by one, exactly as
 *                  flux_kv_append would; the query q[b] sits at the new row's position.
 *   o, workspace   as for flux_decode.
 * Results equal flux_kv_append + flux_decode bit for bit (same keys, same split plan,
 * same arithmetic: the new key is streamed from k_new instead of the cache).  A
 * sequence without room writes zeros, keeps its rows and length and sets
 * FLUX_DEVICE_CAPACITY.
 */
int flux_decode_append(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                       const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                       uint16_t* k_cache, uint16_t* v_cache, int32_t* seq_len, int32_t batch,
                       int32_t capacity, uint16_t* o, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Size of the scratch array flux_decode_static keeps inside the library (32 MiB). */
#define FLUX_DECODE_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * flux_decode_static -- flux_decode without a caller workspace.  The paper has no
 * counterpart: this is a deployment convenience of this library.
 *   Meant for callers that cannot allocate device memory or hand the library a
 *   buffer: plugin hosts that give an op no scratch argument, real-time serving loops
 *   that forbid allocation once they are running, and code that runs while some other
 *   component owns the device allocator.
 *   Same arguments and results as flux_decode, minus the workspace.  The split
 *   partials go to a fixed FLUX_DECODE_STATIC_SCRATCH_BYTES array inside the library,
 *   which every GPU that loads the library holds until the process exits; this call
 *   allocates and frees nothing.
 *   Limit: a call whose flux_decode_workspace_size(cfg, batch) exceeds
 *   FLUX_DECODE_STATIC_SCRATCH_BYTES returns FLUX_ERR_WORKSPACE without launching
 *   (the Llama-3.1-8B decode geometry fits up to batch 31).
 *   The first call on a device looks up the array's device address (with that
 *   device current) and caches it.  Under CUDA's lazy module loading (the default)
 *   that first use is also when the device loads the library's decode module and so
 *   reserves the array: make a first (warm-up) call at initialisation, while
 *   allocation is still allowed, and before any stream capture.
 *   All calls share the one array, so calls that can overlap on the GPU (different
 *   streams, or devices sharing a context) race and corrupt each other's results;
 *   serialise them.  The array keeps the last call's contents.  Only its arrival
 *   counters must start at zero: the array is zeroed when the module loads, every call
 *   leaves them at zero, and the partial records are written before they are read.
 */
int flux_decode_static(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                       const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                       const int32_t* seq_len, int32_t batch, int32_t capacity, uint16_t* o,
                       void* stream);

/*
 * SA-layer KV eviction (the persistent decode-time KV saving of layers routed to SA,
 * Tables 15/16).  An SA decode query only reads the sink rows and at most `window`
 * recent rows, so after prefill an SA layer's cache can shrink to a ring cache of
 * sink + ring_rows rows per (sequence, KV head), ring_rows >= window: position p < sink
 * stays in row p, position p >= sink lives in row sink + (p - sink) % ring_rows.
 * seq_len keeps counting logical positions.  Layout [batch][n_kv_heads][sink +
 * ring_rows][head_dim] bf16.
 *
 * flux_kv_compact_ring -- copy the retained rows (positions [0, min(sink, seq_len))
 *   and [max(sink, seq_len - ring_rows), seq_len)) of a full cache
 *   [batch][n_kv_heads][capacity][head_dim] to their ring rows.  Other ring rows are
 *   left as they were.  seq_len[b] > capacity sets FLUX_DEVICE_BAD_LENGTH.
 */
int flux_kv_compact_ring(const flux_attn_cfg* cfg, const uint16_t* k_cache,
                         const uint16_t* v_cache, int32_t capacity, const int32_t* seq_len,
                         int32_t batch, uint16_t* k_ring, uint16_t* v_ring, int32_t ring_rows,
                         void* stream);

/* flux_kv_append_ring -- flux_kv_append into a ring cache: rows for positions
 * [seq_len[b], seq_len[b] + n_new) go to their ring rows (n_new <= ring_rows) and
 * seq_len[b] += n_new; a ring never runs out of room. */
int flux_kv_append_ring(const flux_attn_cfg* cfg, uint16_t* k_ring, uint16_t* v_ring,
                        int32_t* seq_len, int32_t batch, int32_t ring_rows,
                        const uint16_t* k_new, const uint16_t* v_new, int32_t n_new,
                        void* stream);

/* flux_decode_ring -- flux_decode of an SA layer over ring caches: same visible keys,
 * same split plan and arithmetic as flux_decode over the full cache, so the results
 * are identical.  A sequence routed to FA writes zeros and sets
 * FLUX_DEVICE_RING_ROUTE (a ring holds only what SA reads). */
int flux_decode_ring(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                     const uint16_t* q, const uint16_t* k_ring, const uint16_t* v_ring,
                     const int32_t* seq_len, int32_t batch, int32_t ring_rows, uint16_t* o,
                     void* workspace, size_t workspace_bytes, void* stream);

/* flux_decode_append_ring -- flux_kv_append_ring of one new row per sequence followed
 * by flux_decode_ring, in one kernel launch; results equal the two calls bit for bit.
 * A sequence routed to FA writes zeros, is not appended and sets
 * FLUX_DEVICE_RING_ROUTE. */
int flux_decode_append_ring(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                            const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                            uint16_t* k_ring, uint16_t* v_ring, int32_t* seq_len, int32_t batch,
                            int32_t ring_rows, uint16_t* o, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * flux_sa_block_ranges -- the SA key-block set of each query block, as the kernels
 * compute it (streaming pattern of Table 6).  For query block qb (queries
 * qb*block .. qb*block+block-1) the visible key blocks are [0, r[0]) united with
 * [r[1], r[2]), where r = ranges + 3*qb.  ranges: [n_qblocks][3] int32 device memory.
 */
int flux_sa_block_ranges(const flux_attn_cfg* cfg, int32_t n_qblocks, int32_t* ranges,
                         void* stream);

/*
 * flux_prefill_tile_plan -- the KV tiles flux_prefill visits, for checking the SA
 * block indices of the prefill kernel exactly (streaming pattern of Table 6: sink
 * blocks plus a local window of blocks, Figure 1 caption).  Same arguments as
 * flux_prefill minus q, the caches and o; computed on the device by the tile schedule
 * the prefill kernel itself runs.
 *   tiles      [batch][ceil(n_q / 128)][max_tiles] int32 device memory, written: entry
 *              i of query tile m (queries m*128 .. m*128 + 127 of the prompt) is the
 *              index kt of the i-th 128-key tile (keys kt*128 .. kt*128 + 127) the
 *              kernel visits for it, OR FLUX_TILE_MASKED when the kernel applies the
 *              per-key mask in that tile (some query of the tile does not see some key
 *              of it); -1 after the last visited tile.
 *   max_tiles  >= ceil(capacity / 128), else FLUX_ERR_INVALID_ARG.
 * A sequence with seq_len[b] < n_q or > capacity gets only -1 entries and sets
 * FLUX_DEVICE_BAD_LENGTH, as flux_prefill would.
 */
#define FLUX_TILE_MASKED 0x40000000
int flux_prefill_tile_plan(const flux_attn_cfg* cfg, int32_t layer, const uint32_t* fa_mask,
                           const int32_t* seq_len, int32_t batch, int32_t capacity, int32_t n_q,
                           int32_t* tiles, int32_t max_tiles, void* stream);

/* flux_selftest_wait_timeout -- failure-detection self-test (the paper has no
 * counterpart): one thread waits on an mbarrier that nothing releases, through the
 * bounded wait every pipeline wait of the library uses, with a limit of limit_us
 * microseconds (1..1000000).  The wait gives up, FLUX_DEVICE_TIMEOUT is set in the
 * device status word and the kernel returns; the context stays usable. */
int flux_selftest_wait_timeout(uint32_t limit_us, void* stream);

/* Checked build (libflux_checked.so: every kernel compiled with FLUX_CHECKED): global
 * accesses whose indices come from run-time data -- the decode kernel's K/V/q copies,
 * its cache-row and split-partial writes and arrival counters, every KV append and
 * ring compaction -- are guarded; a failing guard sets FLUX_DEVICE_BOUNDS and skips the
 * access, nothing traps.  (Prefill reads K/V only through TMA boxes, which the hardware
 * bounds, and writes rows < n_q by construction.)  The plain libflux.so compiles the
 * guards away.  Same exported symbols, same results.
 *
 * flux_build_checked -- 1 in the checked build, 0 in the plain one (host only).
 * flux_selftest_bounds -- a guard refuses index 16 of a 16-entry device array: the
 *   checked build sets FLUX_DEVICE_BOUNDS, the plain build leaves the status word as it
 *   was; neither touches memory outside the array. */
int flux_build_checked(void);
int flux_selftest_bounds(void* stream);

/* Copy the device status word of the current device to *bits and clear it.
 * Synchronises `stream` first. */
int flux_get_device_status(void* stream, uint32_t* bits);

/* Static English text for a flux_status value. */
const char* flux_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t flux_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLUX_H */
