// gemm_common.cuh -- per-item decoding and epilogues shared by the
// single-CTA and the CTA-pair tcgen05 GEMM kernels of the MoE layer.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "ptx.cuh"
#include "status.cuh"

namespace moe {
namespace gemm {

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

constexpr float kF16Max = 65504.f;

// Per-item description shared by all roles.
struct Item {
  int group;   // expert id, E = shared expert, -1 = router tile
  int row0;    // first row (expert-order row, token for shared/router)
  int nrows;   // valid rows (<= 128)
  int j;       // N tile index
  int nk;      // K blocks
  bool skip;   // no work (N tile beyond this group's width)
};

template <int MODE>
__device__ __forceinline__ Item decode_item(const GemmParams &p, int item) {
  Item it;
  if (MODE == MODE_ROUTER) {
    it.group = -1;
    it.row0 = item * kBlockM;
    it.nrows = min(kBlockM, p.T - it.row0);
    it.j = 0;
    it.nk = p.d / kBlockK;
    it.skip = false;
    return it;
  }
  const int ti = item / p.n_ntiles;
  it.j = item - ti * p.n_ntiles;
  const int4 t = *reinterpret_cast<const int4 *>(&p.tiles[ti]);
  it.group = t.x;
  it.row0 = t.y;
  it.nrows = t.z;
  const bool shared = it.group == p.E;
  if (MODE == MODE_GEMM1) {
    const int width = shared ? p.Fs : p.F;
    it.skip = it.j * p.n_half >= width;
    it.nk = p.d / kBlockK;
  } else {
    it.skip = false;
    it.nk = (shared ? p.Fs : p.F) / kBlockK;
  }
  return it;
}

// Width, in logit units, of the ambiguous band at the k-th/(k+1)-th boundary
// whose experts the select kernel re-decides on float64 logits (see
// router_cc.cu); far above twice the fp32 logit error of either logit path.
constexpr float kRefineBand = 2e-4f;

// Router epilogue: each thread owns one token row and writes its E fp32
// logits (bias added) as 16-byte vectors; selection happens in the
// warp-per-token select kernel that follows.
__device__ __forceinline__ void router_epilogue(const GemmParams &p, const Item &it,
                                                       uint32_t taddr, int row_local,
                                                       const float *bias_s) {
  const bool valid = row_local < it.nrows;
  float *dst = p.logits_out + static_cast<size_t>(it.row0 + row_local) * p.E;
  for (int c = 0; c < p.E; c += 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr + c, r);
    tmem_ld_wait();
    if (valid) {
      if (c + 32 <= p.E) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4 *>(dst + c + i) =
              make_float4(__uint_as_float(r[i]) + bias_s[c + i],
                          __uint_as_float(r[i + 1]) + bias_s[c + i + 1],
                          __uint_as_float(r[i + 2]) + bias_s[c + i + 2],
                          __uint_as_float(r[i + 3]) + bias_s[c + i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c + i < p.E) dst[c + i] = __uint_as_float(r[i]) + bias_s[c + i];
      }
    }
  }
}

// Output staging of one epilogue warp: two 4 KB buffers, each one box of 32
// rows x 64 fp16 columns in the 128-byte-swizzled layout the store tensor
// maps use.  A box whose 32 rows are all valid is written by one TMA store;
// a partially valid box (the last rows of a tile) is written row by row, so
// no store ever reaches rows past the tile.
struct EpiStage {
  uint8_t *buf;  // this warp's 8 KB, 1024-byte aligned
  int cur;
};

constexpr int kEpiBytesPerWarp = 2 * 32 * 128;

__device__ __forceinline__ void store_box(EpiStage &st, const uint32_t (&packed)[32], int lane,
                                          bool full_box, bool row_valid, const CUtensorMap *tm,
                                          int col, int box_row, uint16_t *row_dst) {
  if (full_box) {
    uint8_t *b = st.buf + st.cur * (32 * 128);
    if (lane == 0) bulk_wait_read_le1();  // the store that last used this buffer has read it
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4 *>(b + lane * 128 + ((c ^ (lane & 7)) << 4)) =
          make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tm, b, col, box_row);
      bulk_commit_group();
    }
    st.cur ^= 1;
  } else if (row_valid) {
    uint4 *d4 = reinterpret_cast<uint4 *>(row_dst);
#pragma unroll
    for (int v = 0; v < 8; ++v)
      d4[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
  }
}

// silu(g) * u with a fast reciprocal (the result is rounded to fp16).
__device__ __forceinline__ float swiglu(float g, float u) {
  return __fdividef(g, 1.f + __expf(-g)) * u;
}

// GEMM1 epilogue: h = silu(gate) * up for this thread's row, fp16, 64
// columns per store box.
__device__ __forceinline__ void swiglu_epilogue(const GemmParams &p, const Item &it,
                                                uint32_t taddr, int row_local, EpiStage &st,
                                                const CUtensorMap *tm_h, const CUtensorMap *tm_hsh) {
  const bool shared = it.group == p.E;
  const int q = row_local >> 5;
  const int lane = row_local & 31;
  const bool valid = row_local < it.nrows;
  const bool full_box = (q + 1) * 32 <= it.nrows;
  uint16_t *row_dst = shared ? p.h_shared + static_cast<size_t>(it.row0 + row_local) * p.Fs
                             : p.h + static_cast<size_t>(it.row0 + row_local) * p.F;
  const int col0 = it.j * p.n_half;
  float amax = 0.f;
  for (int cb = 0; cb < p.n_half; cb += 64) {
    uint32_t packed[32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t g[32], u[32];
      tmem_ld_32x32b_x32(taddr + cb + 32 * half, g);
      tmem_ld_32x32b_x32(taddr + p.n_half + cb + 32 * half, u);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float h0 = swiglu(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i]));
        const float h1 = swiglu(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1]));
        amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
        packed[16 * half + i] = pack_f16x2(h0, h1);
      }
    }
    store_box(st, packed, lane, full_box, valid, shared ? tm_hsh : tm_h, col0 + cb,
              it.row0 + q * 32, row_dst + col0 + cb);
  }
  if (valid && amax > kF16Max) record_status(p.status, MOE_ERR_DEVICE_BOUNDS, SITE_H_FP16_RANGE);
}

// GEMM2 epilogue: routed rows -> routed_scale * w * o into o_out (expert-order
// rows); shared-expert rows -> o into s_out (token rows).  fp16, 64 columns
// per store box.
__device__ __forceinline__ void down_epilogue(const GemmParams &p, const Item &it, uint32_t taddr,
                                              int row_local, EpiStage &st,
                                              const CUtensorMap *tm_o, const CUtensorMap *tm_s) {
  const bool shared = it.group == p.E;
  const int q = row_local >> 5;
  const int lane = row_local & 31;
  const bool valid = row_local < it.nrows;
  const bool full_box = (q + 1) * 32 <= it.nrows;
  float scale = 1.f;
  if (valid && !shared) scale = p.routed_scale * p.topk_w[p.perm[it.row0 + row_local]];
  uint16_t *row_dst = (shared ? p.s_out : p.o_out) + static_cast<size_t>(it.row0 + row_local) * p.d;
  const int col0 = it.j * p.n_tile;
  float amax = 0.f;
  for (int cb = 0; cb < p.n_tile; cb += 64) {
    uint32_t packed[32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(taddr + cb + 32 * half, r);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float v0 = __uint_as_float(r[2 * i]) * scale;
        const float v1 = __uint_as_float(r[2 * i + 1]) * scale;
        amax = fmaxf(amax, fmaxf(fabsf(v0), fabsf(v1)));
        packed[16 * half + i] = pack_f16x2(v0, v1);
      }
    }
    store_box(st, packed, lane, full_box, valid, shared ? tm_s : tm_o, col0 + cb,
              it.row0 + q * 32, row_dst + col0 + cb);
  }
  if (valid && amax > kF16Max) record_status(p.status, MOE_ERR_DEVICE_BOUNDS, SITE_SLOT_FP16_RANGE);
}

// Row ids of one GEMM1 tile (this CTA's up to 128 rows): lane l reads rows
// 4l..4l+3.  Issued early (during the previous item), converted to token ids
// into a shared-memory table when the item starts.
__device__ __forceinline__ void tile_rows_fetch(const GemmParams &p, const Item &it, int lane,
                                                int (&v)[4]) {
  const bool shared = it.group == p.E;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int r = 4 * lane + q;
    v[q] = r < it.nrows ? (shared ? it.row0 + r : p.perm[it.row0 + r]) : -1;
  }
}

__device__ __forceinline__ void tile_tokens_store(const GemmParams &p, const Item &it, int lane,
                                                  const int (&v)[4], int *tok_s) {
  const bool shared = it.group == p.E;
#pragma unroll
  for (int q = 0; q < 4; ++q) tok_s[4 * lane + q] = v[q] < 0 ? -1 : (shared ? v[q] : v[q] / p.k);
  __syncwarp();
}

// The part of an item that one CTA of a pair owns: rows [128 r, 128 r + 128).
__device__ __forceinline__ Item pair_half(Item it, int rank) {
  it.row0 += rank * kBlockM;
  it.nrows = it.nrows - rank * kBlockM;
  if (it.nrows < 0) it.nrows = 0;
  if (it.nrows > kBlockM) it.nrows = kBlockM;
  return it;
}

}  // namespace gemm
}  // namespace moe
