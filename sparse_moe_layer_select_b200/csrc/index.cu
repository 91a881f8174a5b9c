// index.cu -- expert order of the (token, slot) pairs and the tile list of
// the grouped expert GEMMs.
//
// The grouped GEMM takes tokens laid out expert by expert (Laguna M.1/XS.2
// Technical Report summary, Key claims, report §3.1.2, Fig. 2: the tokens are
// copied so that each expert's rows are contiguous).  Here that order is an
// index, not a copy:
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
//                         experts from bit-plane ballots (stable, deterministic)
// With a single chunk (decode-sized batches) one CTA does all three steps in
// one launch (index_single_kernel), or, inside a layer forward with E <= 256,
// the last CTA of the router's selection kernel does (router_cc.cu).  With up
// to as many chunks as can be resident at once, one cooperative launch does
// them (index_coop_kernel, a grid barrier between the histograms and the
// scatter); beyond that the two kernels above run.  The device steps
// themselves are in index_common.cuh.
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

// All of the above in one cooperative launch (every chunk's CTA resident at
// once): each CTA keeps its per-warp histograms in shared memory, publishes its
// chunk totals and waits at a grid barrier (an arrival counter in the workspace
// header, a bounded spin); then every CTA derives its own chunk's base row of
// each expert from the totals (the sum over the chunks before it plus the
// expert's offset, an exclusive scan over experts that each CTA repeats), CTA
// 0 writes counts, offsets and the tile lists, and every CTA scatters its
// entries.  One launch and no second pass over the routing instead of two.
__global__ void __launch_bounds__(512)
    index_coop_kernel(const int32_t *__restrict__ topk_idx, int n, int E, int T, int with_shared,
                      int *__restrict__ chunk_hist, int32_t *__restrict__ counts,
                      int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                      int32_t *__restrict__ inv, Tile *__restrict__ tiles,
                      Tile *__restrict__ tiles_pair, int *__restrict__ header, int sub) {
  __shared__ int h[kIdxWarps * kMaxE];
  __shared__ int warp_sums[32];
  __shared__ int totals[3];
  __shared__ int go;
  __shared__ int s_first[kMaxE], s_row0[kMaxE], s_cnt[kMaxE];
  const int nchunks = gridDim.x;
  chunk_warp_hist(topk_idx, n, E, blockIdx.x, h, header, sub);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) s += h[w * E + e];
    chunk_hist[static_cast<size_t>(blockIdx.x) * E + e] = s;
  }
  __threadfence();  // this chunk's totals are visible before its arrival
  __syncthreads();
  if (threadIdx.x == 0) {
    int *arrived = &reinterpret_cast<WsHeader *>(header)->index_arrived;
    atomicAdd(arrived, 1);
    const long long t0 = clock64();
    int ok = 1;
    while (*reinterpret_cast<volatile int *>(arrived) < nchunks) {
      if (clock64() - t0 > kWaitLimitCycles) {
        record_status(header, MOE_ERR_DEVICE_TIMEOUT, SITE_INDEX_GRID_BARRIER);
        ok = 0;
        break;
      }
    }
    __threadfence();
    go = ok;
  }
  __syncthreads();
  if (!go) return;
  // this chunk's base row of each expert: offset of the expert + rows in earlier chunks
  const int e = threadIdx.x;
  int total = 0, before = 0;
  if (e < E) {
    int c = 0;
    for (; c + 32 <= nchunks; c += 32) {  // 32 independent loads in flight
      int v[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = __ldcg(&chunk_hist[static_cast<size_t>(c + q) * E + e]);
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        total += v[q];
        before += (c + q) < static_cast<int>(blockIdx.x) ? v[q] : 0;
      }
    }
    for (; c < nchunks; ++c) {
      const int v = __ldcg(&chunk_hist[static_cast<size_t>(c) * E + e]);
      total += v;
      before += c < static_cast<int>(blockIdx.x) ? v : 0;
    }
  }
  const int off = block_exclusive_scan(e < E ? total : 0, warp_sums, &totals[0]);
  // CTA 0 writes counts, offsets and the 128-row tile list, CTA 1 (CTA 0 with
  // a single chunk) the 256-row list, each spread over the CTA's threads.
  const int pair_writer = nchunks > 1 ? 1 : 0;
  if (blockIdx.x == 0) {
    if (e < E) {
      counts[e] = total;
      offsets[e] = off;
    }
    if (e == 0) offsets[E] = totals[0];
    const int n1 = write_tiles_spread(e, total, off, E, T, with_shared, kBlockM, tiles, warp_sums,
                                      &totals[1], s_first, s_row0, s_cnt);
    if (threadIdx.x == 0) {
      reinterpret_cast<WsHeader *>(header)->n_tiles = n1;
      if (tiles_pair == nullptr) reinterpret_cast<WsHeader *>(header)->n_tiles_pair = 0;
    }
  }
  if (tiles_pair != nullptr && static_cast<int>(blockIdx.x) == pair_writer) {
    const int n2 = write_tiles_spread(e, total, off, E, T, with_shared, 2 * kBlockM, tiles_pair,
                                      warp_sums, &totals[2], s_first, s_row0, s_cnt);
    if (threadIdx.x == 0) reinterpret_cast<WsHeader *>(header)->n_tiles_pair = n2;
  }
  // per-warp first rows of this chunk (the shared-memory histograms of phase 1)
  if (e < E) {
    int run = off + before;
#pragma unroll
    for (int w = 0; w < kIdxWarps; ++w) {
      const int c = h[w * E + e];
      h[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  // the chunk's entries belong to its first kIdxWarps warps (sub entries each); the
  // CTA's other warps only took part in the scans
  if ((threadIdx.x >> 5) < kIdxWarps) chunk_warp_scatter(topk_idx, n, E, blockIdx.x, h, perm, inv, sub);
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

// How many index_coop_kernel CTAs can be resident at once on the current
// device (0 if the query fails): the one-launch builder is used only for up to
// that many chunks.
int coop_index_max_ctas() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, index_coop_kernel, 512, 0) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 0;
    cached[dev] = per_sm * sms > 0 ? per_sm * sms : -1;
  }
  return cached[dev] > 0 ? cached[dev] : 0;
}

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
  if (E <= 512 && nchunks <= coop_index_max_ctas()) {
    // one cooperative launch: all chunk CTAs are resident together
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nchunks);
    cfg.blockDim = dim3(512);
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeCooperative;
    attr.val.cooperative = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const int sub = chunk / kIdxWarps;
    *launches += 1;
    return cudaLaunchKernelEx(&cfg, index_coop_kernel, topk_idx, n, E, T, with_shared, chunk_hist,
                              counts, offsets, perm, inv, tiles, tiles_pair, status, sub);
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
