// Layer Router of Flux Attention (Figure 2): x_Q -> boundary mean-pool (Figure 8) ->
// Linear(h->r) -> ReLU -> Linear(r->n_layers) -> hard FA/SA decision per layer (the
// soft FA probability of the Table 19 caption, thresholded) -> device bitmask.
//
// One kernel launch, one 8-CTA thread-block cluster per sequence; intermediate
// vectors live in shared memory and move between the CTAs of a cluster through
// distributed shared memory, so the router needs no workspace:
//   1. each CTA sums a contiguous share of the pooled tokens (16-byte loads);
//   2. each CTA reduces one slice of the columns over the 8 partial sums (DSMEM) and
//      divides by the token count; then every CTA gathers the full pooled vector;
//   3. each CTA evaluates its share of the hidden units (a warp per row of W1);
//   4. CTA 0 gathers the hidden vector, evaluates the per-layer logits, compares them
//      with tau and writes the packed mask (and optionally the logits).
// Accumulation is fp64 (inputs are exact in fp64), so the hard decisions carry no
// fp32 rounding and match an fp64 evaluation up to ~1e-13 relative.
#include <cooperative_groups.h>

#include "flux_device.cuh"
#include "flux_internal.h"

namespace cg = cooperative_groups;

namespace flux {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 256;
constexpr int kMaxChunksPerThread = kRouterMaxHidden / 8 / kThreads;  // 8

struct RouterArgs {
  const uint16_t* w1;
  const uint16_t* b1;
  const uint16_t* w2;
  const uint16_t* b2;
  int hidden, rank, n_layers;
  const uint16_t* xq;
  int seq, pool_len;
  float tau;
  uint32_t* fa_mask;
  int mask_words;
  double* logits;
};

__device__ __forceinline__ double bf16_to_double(uint16_t x) {
  return double(__uint_as_float(uint32_t(x) << 16));
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads)
    router_kernel(const RouterArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank_in_cluster = int(cluster.block_rank());
  const int b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(16) uint8_t smem[];
  double* part = reinterpret_cast<double*>(smem);            // [hidden]: partial, then full p
  const int slice = (a.hidden + kCluster - 1) / kCluster;
  double* pslice = part + a.hidden;                           // [slice]
  const int rows_per = (a.rank + kCluster - 1) / kCluster;
  double* uslice = pslice + slice;                            // [rows_per]
  double* ufull = uslice + rows_per;                          // [rank] (CTA 0)
  uint32_t* words = reinterpret_cast<uint32_t*>(ufull + a.rank);  // [mask_words]

  // ---- 1. partial sums over this CTA's share of the pooled tokens
  int n_tok, n_prefix, suffix_start;
  if (a.pool_len <= 0 || a.seq <= a.pool_len) {
    n_tok = a.seq;
    n_prefix = a.seq;
    suffix_start = a.seq;
  } else {
    n_tok = a.pool_len;
    n_prefix = (a.pool_len + 1) / 2;
    suffix_start = a.seq - a.pool_len / 2;
  }
  const int per_cta = (n_tok + kCluster - 1) / kCluster;
  const int j0 = rank_in_cluster * per_cta;
  const int j1 = min(n_tok, j0 + per_cta);
  const int n_chunks = a.hidden / 8;
  double acc[kMaxChunksPerThread][8];
#pragma unroll
  for (int i = 0; i < kMaxChunksPerThread; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[i][e] = 0.0;
  const uint16_t* xb = a.xq + size_t(b) * a.seq * a.hidden;
  for (int j = j0; j < j1; ++j) {
    const int t = (j < n_prefix) ? j : suffix_start + (j - n_prefix);
    const uint4* row = reinterpret_cast<const uint4*>(xb + size_t(t) * a.hidden);
#pragma unroll
    for (int i = 0; i < kMaxChunksPerThread; ++i) {
      const int cc = tid + i * kThreads;
      if (cc < n_chunks) {
        const uint4 raw = __ldg(row + cc);
        float f[8];
        bf16x8_to_float(raw, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] += double(f[e]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxChunksPerThread; ++i) {
    const int cc = tid + i * kThreads;
    if (cc < n_chunks)
#pragma unroll
      for (int e = 0; e < 8; ++e) part[cc * 8 + e] = acc[i][e];
  }
  cluster.sync();

  // ---- 2. reduce my column slice over the 8 partials, divide, then gather
  const int c0 = rank_in_cluster * slice;
  const int c1 = min(a.hidden, c0 + slice);
  for (int col = c0 + tid; col < c1; col += kThreads) {
    double s = 0.0;
    for (int r = 0; r < kCluster; ++r) s += cluster.map_shared_rank(part, r)[col];
    pslice[col - c0] = s / double(n_tok);
  }
  cluster.sync();
  for (int col = tid; col < a.hidden; col += kThreads) {
    const int owner = col / slice;
    part[col] = cluster.map_shared_rank(pslice, owner)[col - owner * slice];
  }
  __syncthreads();

  // ---- 3. hidden units of my row slice: u_k = relu(W1[k] . p + b1[k])
  const int k0 = rank_in_cluster * rows_per;
  const int k1 = min(a.rank, k0 + rows_per);
  for (int k = k0 + warp; k < k1; k += kThreads / 32) {
    const uint4* wrow = reinterpret_cast<const uint4*>(a.w1 + size_t(k) * a.hidden);
    double s = 0.0;
    for (int cc = lane; cc < n_chunks; cc += 32) {
      const uint4 raw = __ldg(wrow + cc);
      float f[8];
      bf16x8_to_float(raw, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fma(double(f[e]), part[cc * 8 + e], s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) {
      const double bias = a.b1 ? bf16_to_double(a.b1[k]) : 0.0;
      const double pre = s + bias;
      uslice[k - k0] = pre > 0.0 ? pre : 0.0;
    }
  }
  cluster.sync();

  // ---- 4. CTA 0: logits, hard decisions, packed mask
  if (rank_in_cluster == 0) {
    for (int k = tid; k < a.rank; k += kThreads) {
      const int owner = k / rows_per;
      ufull[k] = cluster.map_shared_rank(uslice, owner)[k - owner * rows_per];
    }
    for (int w = tid; w < a.mask_words; w += kThreads) words[w] = 0u;
    __syncthreads();
    for (int l = warp; l < a.n_layers; l += kThreads / 32) {
      const uint16_t* wrow = a.w2 + size_t(l) * a.rank;
      double s = 0.0;
      for (int k = lane; k < a.rank; k += 32) s = fma(bf16_to_double(wrow[k]), ufull[k], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (lane == 0) {
        const double z = s + (a.b2 ? bf16_to_double(a.b2[l]) : 0.0);
        if (a.logits) a.logits[size_t(b) * a.n_layers + l] = z;
        if (z > double(a.tau)) atomicOr(words + (l >> 5), 1u << (l & 31));
      }
    }
    __syncthreads();
    for (int w = tid; w < a.mask_words; w += kThreads)
      a.fa_mask[size_t(b) * a.mask_words + w] = words[w];
  }
  cluster.sync();  // keep every CTA's shared memory alive until CTA 0 has read it
}

}  // namespace

cudaError_t launch_route(const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                         const uint16_t* b2, int hidden, int rank, int n_layers,
                         const uint16_t* xq, int batch, int seq, int pool_len, float tau,
                         uint32_t* fa_mask, double* logits, cudaStream_t stream) {
  RouterArgs a;
  a.w1 = w1;
  a.b1 = b1;
  a.w2 = w2;
  a.b2 = b2;
  a.hidden = hidden;
  a.rank = rank;
  a.n_layers = n_layers;
  a.xq = xq;
  a.seq = seq;
  a.pool_len = pool_len;
  a.tau = tau;
  a.fa_mask = fa_mask;
  a.mask_words = (n_layers + 31) / 32;
  a.logits = logits;
  const int slice = (hidden + kCluster - 1) / kCluster;
  const int rows_per = (rank + kCluster - 1) / kCluster;
  const size_t smem = size_t(hidden + slice + rows_per + rank) * 8 + size_t(a.mask_words) * 4;
  cudaError_t err = cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem));
  if (err != cudaSuccess) return err;
  router_kernel<<<dim3(kCluster, batch), kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace flux
