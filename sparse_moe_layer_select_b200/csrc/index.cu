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
// The (t, j) entries are cut into chunks of kIndexChunk = 4096, one CTA of 8
// warps per chunk, each warp owning 512 consecutive entries:
//   index_hist_scan_kernel  per-chunk expert histogram; the CTA that
//                         finishes last then sums per expert over chunks,
//                         scans over experts, writes the chunk bases and the
//                         tile lists
//   index_scatter_kernel  per chunk: per-warp histograms and their scan give
//                         each warp its first row per expert; each warp then
//                         places its entries in order, ranks among equal
//                         experts from __match_any_sync (stable, deterministic)
// With a single chunk (decode-sized batches) one CTA does all three steps in
// one launch (index_single_kernel).
#include "kernels.h"
#include "status.cuh"

namespace moe {

namespace {

constexpr int kMaxE = 512;
constexpr int kIdxWarps = 8;
constexpr int kSub = kIndexChunk / kIdxWarps;  // 512 entries per warp
static_assert(kIndexChunk % (kIdxWarps * 32) == 0, "chunk layout");

// Block-wide exclusive scan of one value per thread (blockDim.x a multiple of
// 32, at most 1024).
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

// Per-warp expert histograms of one chunk into h[kIdxWarps][E] (shared).
__device__ __forceinline__ void chunk_warp_hist(const int32_t *__restrict__ topk_idx, int n,
                                                int E, int chunk, int *h, int *status) {
  for (int i = threadIdx.x; i < kIdxWarps * E; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int base = chunk * kIndexChunk + warp * kSub;
  if (warp < kIdxWarps) {  // (a larger CTA's other warps only clear and wait)
    int *hw = h + warp * E;
    int ids[kSub / 32];  // all loads first: one memory round trip per warp
#pragma unroll
    for (int q = 0; q < kSub / 32; ++q) {
      const int i = base + q * 32 + lane;
      ids[q] = i < n ? topk_idx[i] : kNotRouted;
    }
#pragma unroll
    for (int q = 0; q < kSub / 32; ++q) {
      const int e = ids[q];
      if (e == kNotRouted) continue;
      if (e < 0 || e >= E) {
        if (status) record_status(status, MOE_ERR_DEVICE_BOUNDS, SITE_PERMUTE_EXPERT_ID);
        continue;
      }
      atomicAdd(&hw[e], 1);
    }
  }
  __syncthreads();
}

// Each warp places its 512 entries: fill[warp][e] holds its next row of e.
__device__ __forceinline__ void chunk_warp_scatter(const int32_t *__restrict__ topk_idx, int n,
                                                   int E, int chunk, int *fill,
                                                   int32_t *__restrict__ perm,
                                                   int32_t *__restrict__ inv) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int *fw = fill + warp * E;
  const int base = chunk * kIndexChunk + warp * kSub;
  int ids[kSub / 32];  // all loads first: one memory round trip per warp
#pragma unroll
  for (int q = 0; q < kSub / 32; ++q) {
    const int i = base + q * 32 + lane;
    ids[q] = i < n ? topk_idx[i] : -1;
  }
#pragma unroll
  for (int q = 0; q < kSub / 32; ++q) {
    const int r = q * 32;
    const int i = base + r + lane;
    if (base + r >= n) break;  // warp-uniform
    int e = ids[q];
    if (e < 0 || e >= E) e = -1;
    const unsigned m = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(m & lt);
    if (e >= 0) {
      const int pos = fw[e] + rank;
      perm[pos] = i;
      if (inv) inv[i] = pos;  // expert-order row of entry i = t * k + j
    } else if (inv && i < n) {
      inv[i] = -1;  // not routed
    }
    __syncwarp();
    if (e >= 0 && rank == 0) fw[e] += __popc(m);
    __syncwarp();
  }
}

// Turn the chunk's per-warp histograms h[w][e] into per-warp first rows,
// starting from the chunk's base row of each expert.
__device__ __forceinline__ void warp_bases(int E, const int *chunk_base_e, int *h) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = chunk_base_e[e];
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) {
      const int c = h[w * E + e];
      h[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
}

// One tile list: blocks of at most tile_rows rows of each expert in expert
// order, then the shared-expert blocks (token rows); returns the count.
__device__ __forceinline__ int write_tiles(int e, int cnt, int off, int E, int T, int with_shared,
                                           int tile_rows, Tile *__restrict__ tiles,
                                           int *warp_sums, int *total) {
  const int ntile = e < E ? (cnt + tile_rows - 1) / tile_rows : 0;
  const int toff = block_exclusive_scan(ntile, warp_sums, total);
  for (int i = 0; i < ntile; ++i) {
    Tile t;
    t.group = e;
    t.row0 = off + i * tile_rows;
    t.nrows = min(tile_rows, cnt - i * tile_rows);
    t.pad = 0;
    tiles[toff + i] = t;
  }
  const int nshared = with_shared ? (T + tile_rows - 1) / tile_rows : 0;
  for (int i = threadIdx.x; i < nshared; i += blockDim.x) {
    Tile t;
    t.group = E;
    t.row0 = i * tile_rows;
    t.nrows = min(tile_rows, T - i * tile_rows);
    t.pad = 0;
    tiles[*total + i] = t;
  }
  return *total + nshared;
}

// Expert sums over chunks, exclusive scan over experts, chunk bases and the
// tile lists (128-row tiles; 256-row tiles too when tiles_pair is given).
// One CTA of 512 threads (one thread per expert).
__device__ __forceinline__ void scan_and_tiles(int *__restrict__ chunk_hist, int nchunks, int E,
                                               int T, int with_shared,
                                               int32_t *__restrict__ counts,
                                               int32_t *__restrict__ offsets,
                                               Tile *__restrict__ tiles,
                                               Tile *__restrict__ tiles_pair,
                                               int *__restrict__ header, int *warp_sums,
                                               int *totals) {
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E) {
    int c = 0;
    for (; c + 8 <= nchunks; c += 8) {  // eight independent loads in flight
      int v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = __ldcg(&chunk_hist[static_cast<size_t>(c + q) * E + e]);
#pragma unroll
      for (int q = 0; q < 8; ++q) cnt += v[q];
    }
    for (; c < nchunks; ++c) cnt += __ldcg(&chunk_hist[static_cast<size_t>(c) * E + e]);
  }
  const int off = block_exclusive_scan(e < E ? cnt : 0, warp_sums, &totals[0]);
  if (e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    int run = off;
    int c = 0;
    for (; c + 8 <= nchunks; c += 8) {
      int v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = __ldcg(&chunk_hist[static_cast<size_t>(c + q) * E + e]);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        chunk_hist[static_cast<size_t>(c + q) * E + e] = run;  // chunk base row of expert e
        run += v[q];
      }
    }
    for (; c < nchunks; ++c) {
      const int v = __ldcg(&chunk_hist[static_cast<size_t>(c) * E + e]);
      chunk_hist[static_cast<size_t>(c) * E + e] = run;
      run += v;
    }
  }
  if (e == 0) offsets[E] = totals[0];
  const int n1 = write_tiles(e, cnt, off, E, T, with_shared, kBlockM, tiles, warp_sums, &totals[1]);
  int n2 = 0;
  if (tiles_pair != nullptr)
    n2 = write_tiles(e, cnt, off, E, T, with_shared, 2 * kBlockM, tiles_pair, warp_sums,
                     &totals[2]);
  if (threadIdx.x == 0 && header) {
    reinterpret_cast<WsHeader *>(header)->n_tiles = n1;
    reinterpret_cast<WsHeader *>(header)->n_tiles_pair = n2;
  }
}

// Per-chunk histograms; the CTA that finishes last (a ticket counter in the
// workspace header, zeroed by every call) then runs the scan and writes the
// tile lists.  Nothing waits: the other CTAs simply exit.
__global__ void __launch_bounds__(512)
    index_hist_scan_kernel(const int32_t *__restrict__ topk_idx, int n, int E, int nchunks, int T,
                           int with_shared, int *__restrict__ chunk_hist,
                           int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                           Tile *__restrict__ tiles, Tile *__restrict__ tiles_pair,
                           int *__restrict__ header) {
  __shared__ int h[kIdxWarps * kMaxE];
  __shared__ int warp_sums[32];
  __shared__ int totals[3];
  __shared__ int ticket;
  chunk_warp_hist(topk_idx, n, E, blockIdx.x, h, header);
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
                         int32_t *__restrict__ inv) {
  __shared__ int h[kIdxWarps * kMaxE];
  chunk_warp_hist(topk_idx, n, E, blockIdx.x, h, nullptr);
  warp_bases(E, chunk_base + static_cast<size_t>(blockIdx.x) * E, h);
  chunk_warp_scatter(topk_idx, n, E, blockIdx.x, h, perm, inv);
}

// All of the above for a single chunk (n <= kIndexChunk), in one CTA of 512
// threads: warps 0..7 do the histogram and scatter, all 16 the scan.
__global__ void __launch_bounds__(512)
    index_single_kernel(const int32_t *__restrict__ topk_idx, int n, int E, int T,
                        int with_shared, int *__restrict__ chunk_hist,
                        int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                        int32_t *__restrict__ perm, int32_t *__restrict__ inv,
                        Tile *__restrict__ tiles, Tile *__restrict__ tiles_pair, int *header) {
  __shared__ int h[kIdxWarps * kMaxE];
  __shared__ int warp_sums[32];
  __shared__ int totals[3];
  const int warp = threadIdx.x >> 5;
  chunk_warp_hist(topk_idx, n, E, 0, h, header);  // warps 0..7
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) s += h[w * E + e];
    chunk_hist[e] = s;
  }
  __syncthreads();
  scan_and_tiles(chunk_hist, 1, E, T, with_shared, counts, offsets, tiles, tiles_pair, header,
                 warp_sums, totals);
  __syncthreads();
  warp_bases(E, chunk_hist, h);
  if (warp < kIdxWarps) chunk_warp_scatter(topk_idx, n, E, 0, h, perm, inv);
}

}  // namespace

cudaError_t launch_index(const int32_t *topk_idx, int T, int k, int E, int with_shared,
                         int *chunk_hist, Tile *tiles, int *status, int32_t *counts,
                         int32_t *offsets, int32_t *perm, cudaStream_t s, int *launches,
                         Tile *tiles_pair, int32_t *inv) {
  const int n = T * k;
  const int nchunks = (n + kIndexChunk - 1) / kIndexChunk;
  if (nchunks == 1) {
    index_single_kernel<<<1, 512, 0, s>>>(topk_idx, n, E, T, with_shared, chunk_hist, counts,
                                          offsets, perm, inv, tiles, tiles_pair, status);
    *launches += 1;
    return cudaGetLastError();
  }
  index_hist_scan_kernel<<<nchunks, 512, 0, s>>>(topk_idx, n, E, nchunks, T, with_shared,
                                                  chunk_hist, counts, offsets, tiles, tiles_pair,
                                                  status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  index_scatter_kernel<<<nchunks, kIdxWarps * 32, 0, s>>>(topk_idx, n, E, chunk_hist, perm, inv);
  *launches += 2;
  return cudaGetLastError();
}

}  // namespace moe
