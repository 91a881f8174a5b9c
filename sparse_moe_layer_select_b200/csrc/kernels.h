// kernels.h -- internal launch interface between the C ABI (moe_api.cu) and
// the device kernels.  Not part of the public boundary.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace moe {

// Row tile of the grouped GEMMs: `nrows` (<= 128) consecutive rows starting
// at `row0` of group `group` (an expert id, or E for the shared expert,
// whose rows are token ids).
struct Tile {
  int group;
  int row0;
  int nrows;
  int pad;
};

constexpr int kBlockM = 128;        // rows per tile (tcgen05 M)
constexpr int kBlockK = 64;         // K elements per pipeline stage (one 128-byte swizzle row)
constexpr int kStages = 4;          // shared-memory pipeline depth
constexpr int kIndexChunk = 4096;   // (token, slot) entries per index-builder chunk (at most)

// Entries per index-builder chunk for a batch of n (token, slot) entries: one
// chunk up to kIndexChunk; above that a power of two from 1024 to kIndexChunk,
// so that mid-sized batches still spread over 32-48 CTAs (one per chunk).
__host__ __device__ inline int index_chunk_entries(int64_t n) {
  if (n <= kIndexChunk) return kIndexChunk;
  int c = 1024;
  while (c < kIndexChunk && static_cast<int64_t>(c) * 48 < n) c *= 2;
  return c;
}

enum GemmMode : int {
  MODE_ROUTER = 0,
  MODE_GEMM1 = 1,
  MODE_GEMM2 = 2,
  MODE_F8 = 4,  // mode bit: e4m3 operands (tcgen05 kind::f8f6f4), per-row scales
  MODE_GEMM1_F8 = MODE_GEMM1 | MODE_F8,
  MODE_GEMM2_F8 = MODE_GEMM2 | MODE_F8,
  // mode bit of GEMM2: the epilogue adds each scaled row into its token's fp32
  // accumulator row (bulk reduce-add) instead of writing fp16 contribution rows
  MODE_RED = 8,
  MODE_GEMM2_RED = MODE_GEMM2 | MODE_RED,
};
// K elements of one pipeline stage: one 128-byte swizzle row of A and B.
__host__ __device__ constexpr int stage_k(int mode) { return (mode & MODE_F8) ? 128 : kBlockK; }
__host__ __device__ constexpr int elem_bytes(int mode) { return (mode & MODE_F8) ? 1 : 2; }

struct GemmParams {
  int *status;              // workspace header (status word)
  const Tile *tiles;        // GEMM1/GEMM2: tile list
  const int *n_tiles_dev;   // GEMM1/GEMM2: number of tiles (device)
  int n_tiles_host;         // ROUTER: number of row tiles
  int n_ntiles;             // N tiles per row tile (max over groups)
  int ksplit;               // ROUTER: K slices; slice s writes partial logits at s * T * E
  int T, d, E, k, F, Fs;
  int n_half;               // GEMM1: gate (and up) columns per N tile
  int n_tile;               // MMA N of this launch
  uint32_t a_bytes;         // bytes of one A stage (ROUTER, GEMM2 routed rows)
  uint32_t a_sh_bytes;      // bytes of one A stage for shared-expert rows (GEMM2)
  float routed_scale;       // GEMM2: routed_scaling_factor
  const uint16_t *x;        // GEMM1: token rows [T, d] bf16 (gathered by cp.async)
  const int *perm;          // GEMM1/GEMM2: expert-order rows -> t * k + j
  const float *topk_w;      // GEMM2
  const float *bias;        // ROUTER (may be null)
  float *logits_out;        // ROUTER out: [ksplit][T, E] fp32 partial logits, bias in slice 0
  uint16_t *h;              // GEMM1 out: [T*k, F] fp16 (expert-order rows)
  uint16_t *h_shared;       // GEMM1 out: [T, Fs] fp16
  uint16_t *o_out;          // GEMM2 out: [T*k, d] fp16, routed_scale * w * o (expert-order rows)
  uint16_t *s_out;          // GEMM2 out: [T, d] fp16 shared-expert output
  float *yacc;              // MODE_GEMM2_RED / fused out: [T, d] fp32 accumulator (zeroed before)
  // fused expert kernel: the FFN width is cut into parts of fp (routed) / fp_sh
  // (shared) columns, n_parts / n_parts_sh of them; n_ntiles = the larger count
  int n_parts, n_parts_sh, fp, fp_sh;
  unsigned long long *trace;  // pipeline timestamps (builds with MOE_TRACE only), or null
  // MODE_F8 launches: e4m3 codes and float32 scales (one per row)
  const uint8_t *xq;        // GEMM1: token rows [T, d] e4m3 (gathered by cp.async)
  const float *sx;          // GEMM1: scale of each token row of xq
  const float *sa;          // GEMM2: scale of each expert-order row of h
  const float *sa_sh;       // GEMM2: scale of each token row of h_shared
  const float *sb0, *sb1;   // scales of the B rows (gate, up | down) of the routed experts
  const float *sb0_sh, *sb1_sh;  // same for the shared expert
};

// Pipeline trace layout (MOE_TRACE builds): trace[(cta * kTraceKinds + kind) * kTraceN + n].
constexpr int kTraceKinds = 8;
constexpr int kTraceN = 4096;
enum TraceKind : int {
  TR_ISSUE = 0,      // producer issued stage n (after its empty wait)
  TR_LANDED = 1,     // this CTA's loads of stage n complete (pair relay)
  TR_FULL = 2,       // MMA thread saw stage n full
  TR_MMA = 3,        // MMAs of stage n issued
  TR_EPI_START = 4,  // epilogue saw item n's accumulator
  TR_EPI_END = 5,    // epilogue released item n's accumulator
  TR_PWAIT = 6,      // producer starts waiting for stage n's buffer
  TR_PDONE = 7,      // producer finished issuing stage n
};

struct GemmMaps {
  CUtensorMap a, b0, b1, a_sh, b0_sh, b1_sh;
  CUtensorMap out, out_sh;  // epilogue TMA stores: 64 columns x 32 rows, 128-byte swizzle
};

// Tensor maps of the fused expert kernel (128-row boxes of 64 columns).
struct FusedMaps {
  CUtensorMap gate, up, down, gate_sh, up_sh, down_sh;
};

// The fused expert FFN (gate/up GEMM, SwiGLU into tensor memory, down GEMM with
// A from tensor memory, modulation and reduce combine into p.yacc); grid = SMs.
size_t gemm_fused_smem_bytes();
cudaError_t launch_gemm_fused(const GemmParams &p, const FusedMaps &m, int grid, cudaStream_t s);

size_t gemm_smem_bytes();
cudaError_t launch_gemm(int mode, const GemmParams &p, const GemmMaps &m, int grid,
                        cudaStream_t s);
// CTA-pair (cluster of 2, M = 256) variant of MODE_GEMM1 / MODE_GEMM2; grid even.
size_t gemm_pair_smem_bytes();
cudaError_t launch_gemm_pair(int mode, const GemmParams &p, const GemmMaps &m, int grid,
                             cudaStream_t s);

// CUDA-core router logits; sms: the device's SM count (grid shape choice).
cudaError_t launch_router_cc(const uint16_t *x, const uint16_t *w_router, const float *bias,
                             float *logits, int T, int d, int E, int sms, cudaStream_t s);
// Warp-per-token selection over the fp32 logits of every token.
// Expert id of a (token, slot) pair that is not routed (a padding token).
constexpr int kNotRouted = -1;

// token_mask (optional, [T]): 0 = padding token, which gets kNotRouted ids
// and zero weights.  bias: the logit bias (its float64 refinement adds it);
// sel_bias: a selection-only bias on the sigmoid scores (one of the two).
// nsplit > 1: logits holds nsplit partial [T, E] planes (K slices of the
// router GEMM); each token's logits are their sum in plane order, written
// back into plane 0 before the selection.
// ix (optional): the index builder's outputs; when the batch's T * k entries
// form one index chunk and E <= 256, the selection kernel also builds the
// index (expert order and tile lists) and *indexed is set.
struct SelectIndexOut {
  int with_shared;
  int *chunk_hist;
  int32_t *counts, *offsets, *perm, *inv;
  Tile *tiles, *tiles_pair;
  int *header;
};
cudaError_t launch_router_select(float *logits, int nsplit, const uint16_t *x,
                                 const uint16_t *w_router, const float *bias,
                                 const float *sel_bias, const uint8_t *token_mask, int T, int d,
                                 int E, int k, int norm_topk, int32_t *topk_idx, float *topk_w,
                                 cudaStream_t s, const SelectIndexOut *ix = nullptr,
                                 bool *indexed = nullptr);

cudaError_t launch_index(const int32_t *topk_idx, int T, int k, int E, int with_shared,
                         int *chunk_hist, Tile *tiles, int *status, int32_t *counts,
                         int32_t *offsets, int32_t *perm, cudaStream_t s, int *launches,
                         Tile *tiles_pair = nullptr, int32_t *inv = nullptr);
// x_perm[r] = x[perm[r] / k] for r < *n_valid (the routed rows, offsets[E]).
cudaError_t launch_gather_rows(const uint16_t *x, const int32_t *perm, const int32_t *n_valid,
                               int n_rows, int k, int d, uint16_t *x_perm, cudaStream_t s);
// y[t] = bf16( sum_j o[inv[t*k + j]] + s_out[t] ), fp32 sums in slot order; slots
// with inv < 0 (not routed) are skipped.
cudaError_t launch_combine(const uint16_t *o, const uint16_t *s_out, const int32_t *inv, int T,
                           int k, int d, uint16_t *y, cudaStream_t s);
// y = bf16(yacc), n elements (a multiple of 8).
cudaError_t launch_finalize(const float *yacc, size_t n, uint16_t *y, cudaStream_t s);
// Per-row e4m3 codes and float32 scales of a [rows, K] bf16 (or fp16) matrix;
// K % 8 == 0; rows from *n_valid on (if given) are skipped; pow2: power-of-two
// scales.
cudaError_t launch_quant_rows_e4m3(const uint16_t *src, bool is_f16, bool pow2, int rows,
                                  const int32_t *n_valid, int K, uint8_t *codes, float *scales,
                                  cudaStream_t s);
cudaError_t launch_bf16_to_f16(const uint16_t *src, size_t n, uint16_t *dst, int *status,
                               cudaStream_t s);
cudaError_t launch_selftest_wait(int *status, long long limit_cycles, cudaStream_t s);

// Sets what moe_last_launch_count() reports on this host thread (entry points
// implemented outside moe_api.cu).
void set_last_launch_count(int n);

}  // namespace moe
