// permute_static.cu -- moe_permute_static: the expert-order permutation for
// callers that cannot allocate device memory.
//
// Some callers can't call cudaMalloc: code running inside another runtime's
// memory pool or arena that forbids outside allocations, or plugins loaded
// into a host process that owns all device memory.  For them the
// index builder's scratch (status word, per-chunk expert histograms, tile
// list) lives in a file-scope device array of fixed size instead of a
// caller-provided workspace.  Every GPU that loads this library keeps the
// array until the process exits.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "../../include/moe.h"
#include "kernels.h"
#include "status.cuh"

namespace {

using namespace moe;

// MOE_STATIC_SCRATCH_BYTES (512 KiB): status word, per-chunk expert histograms
// and the 128-row tile list, each section rounded up to 256 bytes (the size
// test in moe_permute_static; T * k up to 1,384,448 pairs at E = 256 and
// 823,296 at E = 512).
static __device__ __align__(256) unsigned char g_permute_scratch[MOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void *g_static_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address must come
// from cudaGetSymbolAddress, once per device, with that device current.
cudaError_t static_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return cudaSuccess;
}

inline size_t a256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

extern "C" moe_status moe_permute_static(const moe_dims_t *dims, const int32_t *topk_idx,
                                         int32_t *counts, int32_t *offsets, int32_t *perm,
                                         void *stream) {
  if (dims == nullptr || dims->struct_size != sizeof(moe_dims_t)) return MOE_ERR_INVALID_ARG;
  const int T = dims->T, E = dims->num_experts, k = dims->num_experts_per_tok;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > 512 || k < 1 || k > 16 || k > E) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!topk_idx || !counts || !offsets || !perm) return MOE_ERR_INVALID_ARG;
  const void *ptrs[] = {topk_idx, counts, offsets, perm};
  for (const void *p : ptrs)
    if (reinterpret_cast<uintptr_t>(p) & 15) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
  const size_t n = static_cast<size_t>(T) * k;
  const size_t nchunks = std::max<size_t>((n + index_chunk_entries(n) - 1) / index_chunk_entries(n), 1);
  const size_t max_tiles = (n + kBlockM - 1) / kBlockM + E;
  const size_t off_hist = a256(sizeof(WsHeader));
  const size_t off_tiles = off_hist + a256(nchunks * E * sizeof(int));
  const size_t need = off_tiles + a256(max_tiles * sizeof(Tile));
  set_last_launch_count(0);
  if (need > MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  void *base = nullptr;
  if (static_scratch(&base) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char *b = static_cast<char *>(base);
  if (cudaMemsetAsync(b, 0, sizeof(WsHeader), s) != cudaSuccess) return MOE_ERR_CUDA;
  int launches = 0;
  if (launch_index(topk_idx, T, k, E, 0, reinterpret_cast<int *>(b + off_hist),
                   reinterpret_cast<Tile *>(b + off_tiles), reinterpret_cast<int *>(b), counts,
                   offsets, perm, s, &launches) != cudaSuccess)
    return MOE_ERR_CUDA;
  set_last_launch_count(launches);
  return MOE_OK;
}
