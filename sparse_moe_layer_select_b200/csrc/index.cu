// index.cu -- expert order of the (token, slot) pairs and the tile list of
// the grouped expert GEMMs.
//
// The grouped GEMM takes tokens laid out expert by expert (Laguna M.1/XS.2
// Technical Report summary, Key claims, report §3.1.2, Fig. 2: tokens are
// copied "in expert order").  Here that order is an index, not a copy:
//
//   counts[e]  rows of expert e;  offsets = exclusive prefix sum (E + 1)
//   perm[r]    = t * k + j for the r-th row in expert order, rows of one
//                expert in ascending (t, j) -- a stable counting sort.
//   tiles      (expert, first row, rows) blocks of at most 128 rows, in
//              expert order, followed by the shared expert's token blocks.
//
// Three launches, all deterministic:
//   index_hist_kernel     per-chunk expert histogram (chunk = 1024 entries)
//   index_scan_kernel     one CTA: per-expert running sums over chunks, an
//                         exclusive scan over experts, tile list
//   index_scatter_kernel  one warp per chunk: entries in index order, ranks
//                         among equal experts from __match_any_sync
#include "kernels.h"
#include "status.cuh"

namespace moe {

namespace {

constexpr int kMaxE = 512;

__global__ void __launch_bounds__(256)
    index_hist_kernel(const int32_t *__restrict__ topk_idx, int n, int E,
                      int *__restrict__ chunk_hist, int *status) {
  __shared__ int h[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kIndexChunk;
  const int end = min(n, base + kIndexChunk);
  for (int i = base + threadIdx.x; i < end; i += blockDim.x) {
    const int e = topk_idx[i];
    if (e < 0 || e >= E) {
      record_status(status, MOE_ERR_DEVICE_BOUNDS, SITE_PERMUTE_EXPERT_ID);
      continue;
    }
    atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_hist[static_cast<size_t>(blockIdx.x) * E + e] = h[e];
}

// Block-wide exclusive scan of one value per thread (blockDim.x == 512).
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_sums, int *total) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += y;
    }
    if (lane < nw) warp_sums[lane] = s;  // inclusive warp totals
    if (lane == nw - 1) *total = s;
  }
  __syncthreads();
  const int prev = warp > 0 ? warp_sums[warp - 1] : 0;
  const int r = prev + x - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(512)
    index_scan_kernel(int *__restrict__ chunk_hist, int nchunks, int E, int T, int with_shared,
                      int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                      Tile *__restrict__ tiles, int *__restrict__ header) {
  __shared__ int warp_sums[32];
  __shared__ int total_rows, total_tiles;
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      int *p = chunk_hist + static_cast<size_t>(c) * E + e;
      const int v = *p;
      *p = cnt;  // chunk base relative to the expert's first row
      cnt += v;
    }
  }
  const int off = block_exclusive_scan(e < E ? cnt : 0, warp_sums, &total_rows);
  const int ntile = e < E ? (cnt + kBlockM - 1) / kBlockM : 0;
  const int toff = block_exclusive_scan(ntile, warp_sums, &total_tiles);
  if (e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    for (int c = 0; c < nchunks; ++c) chunk_hist[static_cast<size_t>(c) * E + e] += off;
    for (int i = 0; i < ntile; ++i) {
      Tile t;
      t.group = e;
      t.row0 = off + i * kBlockM;
      t.nrows = min(kBlockM, cnt - i * kBlockM);
      t.pad = 0;
      tiles[toff + i] = t;
    }
  }
  if (e == 0) offsets[E] = total_rows;
  const int nshared = with_shared ? (T + kBlockM - 1) / kBlockM : 0;
  for (int i = threadIdx.x; i < nshared; i += blockDim.x) {
    Tile t;
    t.group = E;
    t.row0 = i * kBlockM;
    t.nrows = min(kBlockM, T - i * kBlockM);
    t.pad = 0;
    tiles[total_tiles + i] = t;
  }
  if (threadIdx.x == 0) reinterpret_cast<WsHeader *>(header)->n_tiles = total_tiles + nshared;
}

__global__ void __launch_bounds__(32)
    index_scatter_kernel(const int32_t *__restrict__ topk_idx, int n, int E,
                         const int *__restrict__ chunk_base, int32_t *__restrict__ perm) {
  __shared__ int fill[kMaxE];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) fill[e] = chunk_base[static_cast<size_t>(blockIdx.x) * E + e];
  __syncwarp();
  const int base = blockIdx.x * kIndexChunk;
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r < kIndexChunk; r += 32) {
    const int i = base + r + lane;
    int e = -1;
    if (i < n) {
      e = topk_idx[i];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned m = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(m & lt);
    if (e >= 0) perm[fill[e] + rank] = i;
    __syncwarp();
    if (e >= 0 && rank == 0) fill[e] += __popc(m);
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_index(const int32_t *topk_idx, int T, int k, int E, int with_shared,
                         int *chunk_hist, Tile *tiles, int *status, int32_t *counts,
                         int32_t *offsets, int32_t *perm, cudaStream_t s, int *launches) {
  const int n = T * k;
  const int nchunks = (n + kIndexChunk - 1) / kIndexChunk;
  index_hist_kernel<<<nchunks, 256, 0, s>>>(topk_idx, n, E, chunk_hist, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  index_scan_kernel<<<1, 512, 0, s>>>(chunk_hist, nchunks, E, T, with_shared, counts, offsets,
                                      tiles, status);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  index_scatter_kernel<<<nchunks, 32, 0, s>>>(topk_idx, n, E, chunk_hist, perm);
  *launches += 3;
  return cudaGetLastError();
}

}  // namespace moe
