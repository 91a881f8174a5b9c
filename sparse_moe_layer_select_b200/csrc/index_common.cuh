// index_common.cuh -- device steps of the index builder (expert order of the
// (token, slot) pairs and the GEMM tile lists), shared by the index kernels
// (index.cu) and by the router's select kernel, whose last CTA builds the
// index of a single-chunk batch in the same launch (router_cc.cu).  The
// layout of the outputs is described at the top of index.cu.
#pragma once
#include "kernels.h"
#include "status.cuh"

namespace moe {
namespace idx {

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
                                                int E, int chunk, int *h, int *status,
                                                int sub = kSub) {
  for (int i = threadIdx.x; i < kIdxWarps * E; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int base = (chunk * kIdxWarps + warp) * sub;  // chunks of kIdxWarps * sub entries
  if (warp < kIdxWarps) {  // (a larger CTA's other warps only clear and wait)
    int *hw = h + warp * E;
    int ids[kSub / 32];  // all loads first: one memory round trip per warp
#pragma unroll
    for (int q = 0; q < kSub / 32; ++q) {
      const int i = base + q * 32 + lane;
      ids[q] = (q * 32 < sub && i < n) ? __ldcg(&topk_idx[i]) : kNotRouted;
    }
#pragma unroll
    for (int q = 0; q < kSub / 32; ++q) {
      if (q * 32 >= sub) break;
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

// The lanes of the warp whose id equals this lane's (ids in [-1, 1023)): an
// AND over ten bit-plane ballots, the same mask __match_any_sync returns at a
// fraction of its cost (one ballot per bit of the id).
__device__ __forceinline__ unsigned lanes_with_same_id(int e) {
  const unsigned v = static_cast<unsigned>(e) & 0x3ffu;  // -1 -> 1023, above every expert id
  unsigned m = 0xffffffffu;
#pragma unroll
  for (int b = 0; b < 10; ++b) {
    const unsigned bit = (v >> b) & 1u;
    const unsigned votes = __ballot_sync(0xffffffffu, bit);
    m &= bit ? votes : ~votes;
  }
  return m;
}

// Each warp places its `sub` consecutive entries (512 in a multi-chunk
// batch; fewer, spread over all eight warps, in a single small chunk):
// fill[warp][e] holds its next row of e.
__device__ __forceinline__ void chunk_warp_scatter(const int32_t *__restrict__ topk_idx, int n,
                                                   int E, int chunk, int *fill,
                                                   int32_t *__restrict__ perm,
                                                   int32_t *__restrict__ inv, int sub = kSub) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int *fw = fill + warp * E;
  const int base = (chunk * kIdxWarps + warp) * sub;  // chunks of kIdxWarps * sub entries
  int ids[kSub / 32];  // all loads first: one memory round trip per warp
#pragma unroll
  for (int q = 0; q < kSub / 32; ++q) {
    const int i = base + q * 32 + lane;
    ids[q] = (q * 32 < sub && i < n) ? __ldcg(&topk_idx[i]) : -1;
  }
#pragma unroll
  for (int q = 0; q < kSub / 32; ++q) {
    const int r = q * 32;
    const int i = base + r + lane;
    if (r >= sub || base + r >= n) break;  // warp-uniform
    int e = ids[q];
    if (e < 0 || e >= E) e = -1;
    const unsigned m = lanes_with_same_id(e);
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

// The same tile list as write_tiles, with the routed tiles written by every
// thread of the CTA -- tile ti's expert found by a binary search over the
// experts' first tiles -- so that a skewed expert's many tiles are not one
// thread's serial stores.  s_first, s_row0, s_cnt: shared arrays of E ints.
__device__ __forceinline__ int write_tiles_spread(int e, int cnt, int off, int E, int T,
                                                  int with_shared, int tile_rows,
                                                  Tile *__restrict__ tiles, int *warp_sums,
                                                  int *total, int *s_first, int *s_row0,
                                                  int *s_cnt) {
  const int ntile = e < E ? (cnt + tile_rows - 1) / tile_rows : 0;
  const int toff = block_exclusive_scan(ntile, warp_sums, total);
  if (e < E) {
    s_first[e] = toff;
    s_row0[e] = off;
    s_cnt[e] = cnt;
  }
  __syncthreads();
  const int nrouted = *total;
  for (int ti = threadIdx.x; ti < nrouted; ti += blockDim.x) {
    int lo = 0, hi = E - 1;  // the last expert whose first tile is <= ti
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_first[mid] <= ti) lo = mid;
      else hi = mid - 1;
    }
    const int i = ti - s_first[lo];
    Tile t;
    t.group = lo;
    t.row0 = s_row0[lo] + i * tile_rows;
    t.nrows = min(tile_rows, s_cnt[lo] - i * tile_rows);
    t.pad = 0;
    tiles[ti] = t;
  }
  const int nshared = with_shared ? (T + tile_rows - 1) / tile_rows : 0;
  for (int i = threadIdx.x; i < nshared; i += blockDim.x) {
    Tile t;
    t.group = E;
    t.row0 = i * tile_rows;
    t.nrows = min(tile_rows, T - i * tile_rows);
    t.pad = 0;
    tiles[nrouted + i] = t;
  }
  return nrouted + nshared;
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

// The whole index of a single chunk (n <= kIndexChunk entries) in one CTA of
// at least max(E, 256) threads: warps 0..7 do the histogram and the scatter,
// all warps the scan; the counts and bases never leave shared memory.  h:
// kIdxWarps * kMaxE ints of shared memory.
__device__ __forceinline__ void index_single_cta(const int32_t *__restrict__ topk_idx, int n,
                                                 int E, int T, int with_shared,
                                                 int *__restrict__ chunk_hist,
                                                 int32_t *__restrict__ counts,
                                                 int32_t *__restrict__ offsets,
                                                 int32_t *__restrict__ perm,
                                                 int32_t *__restrict__ inv,
                                                 Tile *__restrict__ tiles,
                                                 Tile *__restrict__ tiles_pair, int *header, int *h,
                                                 int *warp_sums, int *totals) {
  (void)chunk_hist;  // one chunk: its totals and bases stay in shared memory
  const int warp = threadIdx.x >> 5;
  // entries per warp: the chunk spread over all eight warps, in whole warps of entries
  const int sub = max(32, (n + kIdxWarps * 32 - 1) / (kIdxWarps * 32) * 32);
  chunk_warp_hist(topk_idx, n, E, 0, h, header, sub);  // warps 0..7
  // one thread per expert: its count, the exclusive scan over experts, and each
  // warp's first row of the expert (in place of the per-warp counts in h)
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E) {
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) cnt += h[w * E + e];
  }
  const int off = block_exclusive_scan(e < E ? cnt : 0, warp_sums, &totals[0]);
  if (e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    int run = off;
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) {
      const int c = h[w * E + e];
      h[w * E + e] = run;
      run += c;
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
  __syncthreads();  // the bases in h are complete
  if (warp < kIdxWarps) chunk_warp_scatter(topk_idx, n, E, 0, h, perm, inv, sub);
}

}  // namespace idx
}  // namespace moe
