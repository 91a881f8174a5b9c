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
  int kb0;     // first K block (ROUTER K slices; 0 otherwise)
  bool skip;   // no work (N tile beyond this group's width)
};

// The tile record an item reads (zero for router items and past the end).
// Roles load the record of their next item one item ahead, so that the gap
// between two items holds no global-load round trip.
template <int MODE>
__device__ __forceinline__ int4 load_tile_rec(const GemmParams &p, int item, int n_items) {
  if ((MODE & 3) == MODE_ROUTER || item >= n_items) return make_int4(0, 0, 0, 0);
  return *reinterpret_cast<const int4 *>(&p.tiles[item / p.n_ntiles]);
}

template <int MODE>
__device__ __forceinline__ Item decode_tile(const GemmParams &p, int item, int4 t) {
  constexpr int BASE = MODE & 3;
  constexpr int KB = stage_k(MODE);
  Item it;
  if (BASE == MODE_ROUTER) {  // item = (128-token tile, block of n_tile experts, K slice)
    const int per_tile = p.n_ntiles * p.ksplit;
    const int ti = item / per_tile;
    const int r = item - ti * per_tile;
    it.group = -1;
    it.row0 = ti * kBlockM;
    it.nrows = min(kBlockM, p.T - it.row0);
    it.j = r / p.ksplit;
    it.nk = p.d / KB / p.ksplit;
    it.kb0 = (r - it.j * p.ksplit) * it.nk;
    it.skip = false;
    return it;
  }
  it.kb0 = 0;
  const int ti = item / p.n_ntiles;
  it.j = item - ti * p.n_ntiles;
  it.group = t.x;
  it.row0 = t.y;
  it.nrows = t.z;
  const bool shared = it.group == p.E;
  if (BASE == MODE_GEMM1) {
    const int width = shared ? p.Fs : p.F;
    it.skip = it.j * p.n_half >= width;
    it.nk = p.d / KB;
  } else {
    it.skip = false;
    it.nk = (shared ? p.Fs : p.F) / KB;
  }
  return it;
}

// Walks one role's items (item, item + step, ...) with a one-item look-ahead:
// current() decodes the role's next non-empty item from the tile record that
// was loaded while the previous item ran; prefetch() starts the loads of the
// record (and the status word) for the item after it; next() steps on.  A
// status word raised by any role is seen at most one item late (every wait
// in the pipeline is bounded on its own).
template <int MODE>
struct ItemWalk {
  int item, step, n_items;
  int4 rec;
  int stop;

  __device__ __forceinline__ ItemWalk(const GemmParams &p, int first, int step_, int n)
      : item(first), step(step_), n_items(n), stop(0) {
    rec = load_tile_rec<MODE>(p, item, n_items);
  }
  // false when this role has no item left (or an error was raised).
  __device__ __forceinline__ bool current(const GemmParams &p, Item &it) {
    for (;;) {
      if (item >= n_items || stop) return false;
      it = decode_tile<MODE>(p, item, rec);
      if (!it.skip) return true;
      item += step;
      rec = load_tile_rec<MODE>(p, item, n_items);
    }
  }
  // Issue the loads for the item after the current one (results consumed by
  // the next current()).
  __device__ __forceinline__ void prefetch(const GemmParams &p) {
    rec = load_tile_rec<MODE>(p, item + step, n_items);
    stop = *reinterpret_cast<const volatile int *>(p.status);
  }
  __device__ __forceinline__ void next() { item += step; }
};

// A 128-row GEMM1 operand part is gathered by kGatherWarps warps, each
// copying kGatherRows consecutive rows with 16-byte cp.async (one warp
// instruction moves 4 whole 128-byte rows).  One warp issues such copies at
// about one instruction per 15 ns, slower than the tensor cores consume a
// stage, so the rows are split across warps on all four SM sub-partitions.
// Even so the copies arrive at only ~16 KB per 0.5 us per SM, which bounds
// the gate/up GEMM at large batches.  (TMA tile::gather4 moves the same 4
// rows per instruction but was slower: with one gathering warp, gather4 for
// all or part of the rows took 2.34 to 2.99 ms for the gate/up GEMM of the
// skewed T=32768 prefill; beside these eight warps, gather4 for 32 or 64 of
// the 128 rows took 1.70 or 2.15 ms against 1.08 ms.)
#ifndef MOE_GATHER_WARPS
#define MOE_GATHER_WARPS 8
#endif
// Whether the TMA-issuing warp also gathers a share (1) or only issues TMA (0).
#ifndef MOE_TMA_WARP_GATHERS
#define MOE_TMA_WARP_GATHERS 0
#endif
constexpr int kGatherWarps = MOE_GATHER_WARPS;
constexpr bool kTmaWarpGathers = MOE_TMA_WARP_GATHERS != 0;
constexpr int kExtraGatherWarps = kGatherWarps - (kTmaWarpGathers ? 1 : 0);
constexpr int kGatherRows = kBlockM / kGatherWarps;
constexpr int kGatherGroups = kGatherRows / 4;  // cp.async instructions per lane per stage
static_assert(kBlockM % (4 * kGatherWarps) == 0 && kExtraGatherWarps >= 0, "gather split");

// Row ids (expert-order row -> token * k + slot, or the token itself for a
// shared-expert tile) of the rows lane `lane` of gather warp gw copies:
// rows gw * kGatherRows + (lane >> 3) + 4 i, i < kGatherGroups; -1 past the
// valid rows.  Issued during the previous item (plain loads whose results
// are first used when the item starts), so that no load, shuffle or
// shared-memory access sits between two items: on a gathering warp those
// would queue behind the in-flight copy instructions.
__device__ __forceinline__ void gather_rows_fetch(const GemmParams &p, const Item &it, int lane,
                                                  int gw, int (&raw)[kGatherGroups]) {
  const bool shared = it.group == p.E;
#pragma unroll
  for (int i = 0; i < kGatherGroups; ++i) {
    const int r = gw * kGatherRows + (lane >> 3) + 4 * i;
    raw[i] = r < it.nrows ? (shared ? it.row0 + r : p.perm[it.row0 + r]) : -1;
  }
}

// Token ids from row ids (arithmetic only).
__device__ __forceinline__ void gather_tokens(const GemmParams &p, const Item &it,
                                              const int (&raw)[kGatherGroups],
                                              int (&tok)[kGatherGroups]) {
  const bool shared = it.group == p.E;
#pragma unroll
  for (int i = 0; i < kGatherGroups; ++i)
    tok[i] = (raw[i] < 0 || shared) ? raw[i] : raw[i] / p.k;
}

// Issue this warp's share of one stage's A gather (GEMM1): the k-block
// starting at column kc, into the 128B-swizzled A buffer at a_dst; the
// lanes' completions arrive on bar (one arrival per lane).  Rows are bf16 x,
// or e4m3 xq for MODE_F8 (128 bytes of a row either way).
template <int MODE>
__device__ __forceinline__ void gather_a_stage(const GemmParams &p, const int (&tok)[kGatherGroups],
                                               int lane, int gw, uint8_t *a_dst, uint64_t *bar,
                                               int kc) {
  constexpr int ES = elem_bytes(MODE);
  // 128-byte swizzle: chunk c of row r sits at chunk (c ^ (r & 7)).
  const int c = lane & 7;
  const uint32_t a_base = smem_u32(a_dst);
  const char *xsrc = ((MODE & MODE_F8) ? reinterpret_cast<const char *>(p.xq)
                                       : reinterpret_cast<const char *>(p.x)) +
                     kc * ES + c * 16;
#pragma unroll
  for (int i = 0; i < kGatherGroups; ++i) {
    const int r = gw * kGatherRows + (lane >> 3) + 4 * i;
    if (tok[i] >= 0)
      cp_async_16(a_base + r * 128 + ((c ^ (r & 7)) << 4),
                  xsrc + static_cast<size_t>(tok[i]) * p.d * ES);
  }
  cp_async_arrive_noinc(bar);
}

// Width, in logit units, of the ambiguous band at the k-th/(k+1)-th boundary
// whose experts the select kernel re-decides on float64 logits (see
// router_cc.cu); far above twice the fp32 logit error of either logit path.
constexpr float kRefineBand = 2e-4f;

// Router epilogue: each thread owns one token row and writes its fp32
// logits of the item's experts as 16-byte vectors, into the plane of the
// item's K slice (the bias goes into slice 0's plane; zeros otherwise);
// selection happens in the warp-per-token select kernel that follows.
__device__ __forceinline__ void router_epilogue(const GemmParams &p, const Item &it,
                                                       uint32_t taddr, int row_local,
                                                       const float *bias_s) {
  if ((row_local >> 5) * 32 >= it.nrows) return;  // no valid row in this warp's quarter
  const bool valid = row_local < it.nrows;
  const int e0 = it.j * p.n_tile;  // this item's block of experts
  const int slice = it.kb0 / it.nk;
  float *dst = p.logits_out + static_cast<size_t>(slice) * p.T * p.E +
               static_cast<size_t>(it.row0 + row_local) * p.E + e0;
  // bias_s holds 512 entries, zero past E; E and n_tile are at most 256, so its
  // last n_tile entries are zeros for the slices after the first.
  const float *b = bias_s + (slice == 0 ? e0 : 512 - p.n_tile);
  for (int c = 0; c < p.n_tile; c += 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr + c, r);
    tmem_ld_wait();
    if (valid) {
      if (c + 32 <= p.n_tile) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4 *>(dst + c + i) =
              make_float4(__uint_as_float(r[i]) + b[c + i], __uint_as_float(r[i + 1]) + b[c + i + 1],
                          __uint_as_float(r[i + 2]) + b[c + i + 2],
                          __uint_as_float(r[i + 3]) + b[c + i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c + i < p.n_tile) dst[c + i] = __uint_as_float(r[i]) + b[c + i];
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

// MODE_F8 epilogues: the weight-row scales of an item's columns, 8 per lane
// (lane l holds columns 8l .. 8l+7 of a 256-column block, or 4l .. 4l+3 of
// a 128-column one), loaded once per item; a 16-column chunk takes its 16
// scales by warp shuffle.
struct ColScales {
  float4 a, b;
};

template <int PER_LANE>  // 4 or 8
__device__ __forceinline__ ColScales load_col_scales(const float *src, int lane) {
  ColScales c;
  c.a = *reinterpret_cast<const float4 *>(src + PER_LANE * lane);
  c.b = PER_LANE == 8 ? *reinterpret_cast<const float4 *>(src + PER_LANE * lane + 4) : c.a;
  return c;
}

__device__ __forceinline__ float pick(const ColScales &c, int e) {  // e: compile-time 0..7
  const float4 &v = e < 4 ? c.a : c.b;
  switch (e & 3) {
    case 0: return v.x;
    case 1: return v.y;
    case 2: return v.z;
    default: return v.w;
  }
}

// acc[i] *= rs * scale(column c0 + i), i < 16, c0 a multiple of 16.
template <int PER_LANE>
__device__ __forceinline__ void scale_chunk16(uint32_t (&acc)[16], float rs, const ColScales &c,
                                              int c0) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float sc = __shfl_sync(0xffffffffu, pick(c, i % PER_LANE), (c0 + i) / PER_LANE);
    acc[i] = __float_as_uint(__uint_as_float(acc[i]) * rs * sc);
  }
}

// GEMM1 epilogue: h = silu(gate) * up for this thread's row, fp16, 64
// columns per store box.  F8: the accumulators are first multiplied by the
// token row's scale and each column's weight-row scale.
template <bool F8>
__device__ __forceinline__ void swiglu_epilogue(const GemmParams &p, const Item &it,
                                                uint32_t taddr, int row_local, EpiStage &st,
                                                const CUtensorMap *tm_h, const CUtensorMap *tm_hsh) {
  const bool shared = it.group == p.E;
  const int q = row_local >> 5;
  if (q * 32 >= it.nrows) return;  // no valid row in this warp's quarter (warp-uniform)
  const int lane = row_local & 31;
  const bool valid = row_local < it.nrows;
  const bool full_box = (q + 1) * 32 <= it.nrows;
  uint16_t *row_dst = shared ? p.h_shared + static_cast<size_t>(it.row0 + row_local) * p.Fs
                             : p.h + static_cast<size_t>(it.row0 + row_local) * p.F;
  const int col0 = it.j * p.n_half;
  float rs = 1.f;
  ColScales cg{}, cu{};
  if (F8) {  // n_half = 128 columns of gate and of up: 4 scales of each per lane
    if (valid) {
      const int tok = shared ? it.row0 + row_local : p.perm[it.row0 + row_local] / p.k;
      rs = p.sx[tok];
    }
    cg = load_col_scales<4>((shared ? p.sb0_sh : p.sb0 + static_cast<size_t>(it.group) * p.F) + col0,
                            lane);
    cu = load_col_scales<4>((shared ? p.sb1_sh : p.sb1 + static_cast<size_t>(it.group) * p.F) + col0,
                            lane);
  }
  float amax = 0.f;
  for (int cb = 0; cb < p.n_half; cb += 64) {
    uint32_t packed[32];
#pragma unroll
    for (int qu = 0; qu < 4; ++qu) {  // 16 gate and 16 up columns at a time
      uint32_t g[16], u[16];
      tmem_ld_32x32b_x16(taddr + cb + 16 * qu, g);
      tmem_ld_32x32b_x16(taddr + p.n_half + cb + 16 * qu, u);
      tmem_ld_wait();
      if (F8) {
        scale_chunk16<4>(g, rs, cg, cb + 16 * qu);
        scale_chunk16<4>(u, rs, cu, cb + 16 * qu);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float h0 = swiglu(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i]));
        const float h1 = swiglu(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1]));
        amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
        packed[8 * qu + i] = pack_f16x2(h0, h1);
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
template <bool F8>
__device__ __forceinline__ void down_epilogue(const GemmParams &p, const Item &it, uint32_t taddr,
                                              int row_local, EpiStage &st,
                                              const CUtensorMap *tm_o, const CUtensorMap *tm_s) {
  const bool shared = it.group == p.E;
  const int q = row_local >> 5;
  if (q * 32 >= it.nrows) return;  // no valid row in this warp's quarter (warp-uniform)
  const int lane = row_local & 31;
  const bool valid = row_local < it.nrows;
  const bool full_box = (q + 1) * 32 <= it.nrows;
  float scale = 1.f;
  if (valid && !shared) scale = p.routed_scale * p.topk_w[p.perm[it.row0 + row_local]];
  uint16_t *row_dst = (shared ? p.s_out : p.o_out) + static_cast<size_t>(it.row0 + row_local) * p.d;
  const int col0 = it.j * p.n_tile;
  ColScales cd{};
  if (F8) {  // h row scale, then each column's weight-row scale (n_tile = 256: 8 per lane)
    if (valid) scale *= shared ? p.sa_sh[it.row0 + row_local] : p.sa[it.row0 + row_local];
    cd = load_col_scales<8>((shared ? p.sb0_sh : p.sb0 + static_cast<size_t>(it.group) * p.d) + col0,
                            lane);
  }
  float amax = 0.f;
  for (int cb = 0; cb < p.n_tile; cb += 64) {
    uint32_t packed[32];
#pragma unroll
    for (int qu = 0; qu < 4; ++qu) {  // 16 columns at a time
      uint32_t r[16];
      tmem_ld_32x32b_x16(taddr + cb + 16 * qu, r);
      tmem_ld_wait();
      if (F8) scale_chunk16<8>(r, 1.f, cd, cb + 16 * qu);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v0 = __uint_as_float(r[2 * i]) * scale;
        const float v1 = __uint_as_float(r[2 * i + 1]) * scale;
        amax = fmaxf(amax, fmaxf(fabsf(v0), fabsf(v1)));
        packed[8 * qu + i] = pack_f16x2(v0, v1);
      }
    }
    store_box(st, packed, lane, full_box, valid, shared ? tm_s : tm_o, col0 + cb,
              it.row0 + q * 32, row_dst + col0 + cb);
  }
  if (valid && amax > kF16Max) record_status(p.status, MOE_ERR_DEVICE_BOUNDS, SITE_SLOT_FP16_RANGE);
}

// GEMM2 epilogue of the reduce combine: each row's routed_scale * w * o (a
// shared-expert row: o) is added into its token's fp32 accumulator row.  The
// warp's 8 KB staging holds its 32 rows x 64 fp32 columns (256 bytes a row);
// every lane stages its own row and issues that row's bulk reduce-adds, which
// the L2 performs (the order of a token's k + 1 additions is not fixed).
// Within a row the sixteen 16-byte chunks are stored rotated by (lane & 7)
// places, so that the warp's shared-memory stores spread over all banks; the
// rotated row then goes out as two bulk reductions (the chunks from the
// rotation point on, then the wrapped ones).
__device__ __forceinline__ void down_epilogue_reduce_cols(const GemmParams &p, const Item &it,
                                                          uint32_t taddr, int row_local,
                                                          EpiStage &st, int col0, int ncols) {
  const bool shared = it.group == p.E;
  const int q = row_local >> 5;
  if (q * 32 >= it.nrows) return;  // no valid row in this warp's quarter (warp-uniform)
  const int lane = row_local & 31;
  const bool valid = row_local < it.nrows;
  float scale = 1.f;
  int tok = 0;
  if (valid) {
    if (shared) {
      tok = it.row0 + row_local;
    } else {
      const int pr = p.perm[it.row0 + row_local];
      tok = pr / p.k;
      scale = p.routed_scale * p.topk_w[pr];
    }
  }
  float *dst = p.yacc + static_cast<size_t>(tok) * p.d + col0;
  uint8_t *row_buf = st.buf + lane * 256;
  const int rot = lane & 7;
  for (int cb = 0; cb < ncols; cb += 64) {
    bulk_wait_read_all();  // this lane's previous reductions have read its staged row
#pragma unroll
    for (int qu = 0; qu < 4; ++qu) {  // 16 columns (four 16-byte chunks) at a time
      uint32_t r[16];
      tmem_ld_32x32b_x16(taddr + cb + 16 * qu, r);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int pos = (4 * qu + i + rot) & 15;
        *reinterpret_cast<float4 *>(row_buf + pos * 16) =
            make_float4(__uint_as_float(r[4 * i]) * scale, __uint_as_float(r[4 * i + 1]) * scale,
                        __uint_as_float(r[4 * i + 2]) * scale,
                        __uint_as_float(r[4 * i + 3]) * scale);
      }
    }
    if (valid) {
      fence_proxy_async_smem();  // the staged row is visible to the bulk copy
      // memory chunks rot..15 hold columns 0 .. 4 (16 - rot) - 1, chunks 0..rot-1 the rest
      bulk_reduce_add_f32(dst + cb, row_buf + rot * 16, static_cast<uint32_t>(16 - rot) * 16);
      if (rot) bulk_reduce_add_f32(dst + cb + 4 * (16 - rot), row_buf, static_cast<uint32_t>(rot) * 16);
      bulk_commit_group();
    }
  }
}

// The reduce epilogue of an item's N tile (GEMM2 with MODE_RED).
__device__ __forceinline__ void down_epilogue_reduce(const GemmParams &p, const Item &it,
                                                     uint32_t taddr, int row_local, EpiStage &st) {
  down_epilogue_reduce_cols(p, it, taddr, row_local, st, it.j * p.n_tile, p.n_tile);
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
