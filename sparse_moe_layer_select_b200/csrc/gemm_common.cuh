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

__device__ __forceinline__ void swiglu_epilogue(const GemmParams &p, const Item &it,
                                                uint32_t taddr, int row_local) {
  const bool shared = it.group == p.E;
  const bool valid = row_local < it.nrows;
  uint16_t *dst = shared ? p.h_shared + static_cast<size_t>(it.row0 + row_local) * p.Fs
                         : p.h + static_cast<size_t>(it.row0 + row_local) * p.F;
  dst += it.j * p.n_half;
  for (int c = 0; c < p.n_half; c += 32) {
    uint32_t g[32], u[32];
    tmem_ld_32x32b_x32(taddr + c, g);
    tmem_ld_32x32b_x32(taddr + p.n_half + c, u);
    tmem_ld_wait();
    uint32_t packed[16];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
      const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
      const float h0 = g0 / (1.f + __expf(-g0)) * u0;
      const float h1 = g1 / (1.f + __expf(-g1)) * u1;
      amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
      packed[i] = pack_f16x2(h0, h1);
    }
    if (valid && amax > kF16Max) record_status(p.status, MOE_ERR_DEVICE_BOUNDS, SITE_H_FP16_RANGE);
    if (valid) {
      uint4 *d4 = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
      for (int v = 0; v < 4; ++v)
        d4[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
    }
  }
}

__device__ __forceinline__ void slot_epilogue(const GemmParams &p, const Item &it, uint32_t taddr,
                                              int row_local) {
  const bool shared = it.group == p.E;
  const bool valid = row_local < it.nrows;
  float scale = 1.f;
  size_t dst_row = 0;
  if (valid) {
    if (shared) {
      const size_t t = static_cast<size_t>(it.row0 + row_local);
      dst_row = t * p.slots + p.k;
    } else {
      const int pt = p.perm[it.row0 + row_local];
      const int t = pt / p.k;
      const int jslot = pt - t * p.k;
      scale = p.routed_scale * p.topk_w[pt];
      dst_row = static_cast<size_t>(t) * p.slots + jslot;
    }
  }
  uint16_t *dst = p.slot_out + dst_row * p.d + static_cast<size_t>(it.j) * p.n_tile;
  for (int c = 0; c < p.n_tile; c += 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr + c, r);
    tmem_ld_wait();
    if (valid) {
      uint32_t packed[16];
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float v0 = __uint_as_float(r[2 * i]) * scale;
        const float v1 = __uint_as_float(r[2 * i + 1]) * scale;
        amax = fmaxf(amax, fmaxf(fabsf(v0), fabsf(v1)));
        packed[i] = pack_f16x2(v0, v1);
      }
      if (amax > kF16Max) record_status(p.status, MOE_ERR_DEVICE_BOUNDS, SITE_SLOT_FP16_RANGE);
      uint4 *d4 = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
      for (int v = 0; v < 4; ++v)
        d4[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
    }
  }
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
