// index.cu -- expert order of the (token, slot) pairs and the tile list of
// the grouped expert GEMMs.
//
// The grouped GEMM takes tokens laid out expert by expert (Laguna M.1/XS.2
// Technical Report summary, Key claims, report §3.1.2, Fig. 2: tokens are
// copied "in expert order").  Here that order is an index, not a copy:
//
//   counts[e]  rows of expert e;  offsets = exclusive prefix sum (E + 1)
//   perm[r]    = t * k + j for the r-th row in expert order, rows of one
//                expert in ascending (t, j) -- a stable counting sort.  Pairs
//                with expert id kNotRouted (-1: padding tokens) are left out:
//                offsets[E] counts the routed pairs only.
//   tiles      (expert, first row, rows) blocks of at most tile_rows rows
//              (128 for single-CTA GEMMs, 256 for CTA-pair GEMMs), in expert
//              order, followed by the shared expert's token blocks.
//
// The (t, j) entries are cut into chunks of index_chunk_entries(n) (1024 to
// 4096, kernels.h), one CTA of 8 warps per chunk, each warp owning an eighth
// of the chunk's consecutive entries:
//   index_hist_scan_kernel  per-chunk expert histogram; the CTA that
//                         finishes last then sums per expert over chunks,
//                         scans over experts, writes the chunk bases and the
//                         tile lists
//   index_scatter_kernel  per chunk: per-warp histograms and their scan give
//                         each warp its first row per expert; each warp then
//                         places its entries in order, ranks among equal
//                         experts from __match_any_sync (stable, deterministic)
// With a single chunk (decode-sized batches) one CTA does all three steps in
// one launch (index_single_kernel), or, inside a layer forward with E <= 256,
// the last CTA of the router's selection kernel does (router_cc.cu).  The
// device steps themselves are in index_common.cuh.
#include "index_common.cuh"
#include "kernels.h"
#include "status.cuh"

namespace moe {

namespace {

using namespace idx;

// Per-chunk histograms; the CTA that finishes last (a ticket counter in the
// workspace header, zeroed by every call) then runs the scan and writes the
// tile lists.  Nothing waits: the other CTAs simply exit.
__global__ void __launch_bounds__(512)
    index_hist_scan_kernel(const int32_t *__restrict__ topk_idx, int n, int E, int nchunks, int T,
                           int with_shared, int *__restrict__ chunk_hist,
                           int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                           Tile *__restrict__ tiles, Tile *__restrict__ tiles_pair,
                           int *__restrict__ header, int sub) {
  __shared__ int h[kIdxWarps * kMaxE];
  __shared__ int warp_sums[32];
  __shared__ int totals[3];
  __shared__ int ticket;
  chunk_warp_hist(topk_idx, n, E, blockIdx.x, h, header, sub);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) s += h[w * E + e];
    chunk_hist[static_cast<size_t>(blockIdx.x) * E + e] = s;
  }
  __threadfence();  // this chunk's totals are visible before the ticket is taken
  __syncthreads();
  if (threadIdx.x == 0)
    ticket = atomicAdd(&reinterpret_cast<WsHeader *>(header)->index_done, 1);
  __syncthreads();
  if (ticket != nchunks - 1) return;
  __threadfence();
  scan_and_tiles(chunk_hist, nchunks, E, T, with_shared, counts, offsets, tiles, tiles_pair,
                 header, warp_sums, totals);
}

__global__ void __launch_bounds__(kIdxWarps * 32)
    index_scatter_kernel(const int32_t *__restrict__ topk_idx, int n, int E,
                         const int *__restrict__ chunk_base, int32_t *__restrict__ perm,
                         int32_t *__restrict__ inv, int sub) {
  __shared__ int h[kIdxWarps * kMaxE];
  chunk_warp_hist(topk_idx, n, E, blockIdx.x, h, nullptr, sub);
  warp_bases(E, chunk_base + static_cast<size_t>(blockIdx.x) * E, h);
  chunk_warp_scatter(topk_idx, n, E, blockIdx.x, h, perm, inv, sub);
}

// All of the above for a single chunk (n <= kIndexChunk), in one CTA of 512
// threads.
__global__ void __launch_bounds__(512)
    index_single_kernel(const int32_t *__restrict__ topk_idx, int n, int E, int T,
                        int with_shared, int *__restrict__ chunk_hist,
                        int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                        int32_t *__restrict__ perm, int32_t *__restrict__ inv,
                        Tile *__restrict__ tiles, Tile *__restrict__ tiles_pair, int *header) {
  __shared__ int h[kIdxWarps * kMaxE];
  __shared__ int warp_sums[32];
  __shared__ int totals[3];
  index_single_cta(topk_idx, n, E, T, with_shared, chunk_hist, counts, offsets, perm, inv, tiles,
                   tiles_pair, header, h, warp_sums, totals);
}

}  // namespace

cudaError_t launch_index(const int32_t *topk_idx, int T, int k, int E, int with_shared,
                         int *chunk_hist, Tile *tiles, int *status, int32_t *counts,
                         int32_t *offsets, int32_t *perm, cudaStream_t s, int *launches,
                         Tile *tiles_pair, int32_t *inv) {
  const int n = T * k;
  const int chunk = index_chunk_entries(n);
  const int nchunks = (n + chunk - 1) / chunk;
  if (nchunks == 1) {
    index_single_kernel<<<1, 512, 0, s>>>(topk_idx, n, E, T, with_shared, chunk_hist, counts,
                                          offsets, perm, inv, tiles, tiles_pair, status);
    *launches += 1;
    return cudaGetLastError();
  }
  index_hist_scan_kernel<<<nchunks, 512, 0, s>>>(topk_idx, n, E, nchunks, T, with_shared,
                                                  chunk_hist, counts, offsets, tiles, tiles_pair,
                                                  status, chunk / kIdxWarps);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  index_scatter_kernel<<<nchunks, kIdxWarps * 32, 0, s>>>(topk_idx, n, E, chunk_hist, perm, inv,
                                                          chunk / kIdxWarps);
  *launches += 2;
  return cudaGetLastError();
}

}  // namespace moe
