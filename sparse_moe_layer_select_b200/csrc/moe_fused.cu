// moe_fused.cu -- the routed and shared expert FFNs as one persistent tcgen05
// kernel per layer call, with the SwiGLU activation kept in tensor memory.
//
// Per item (a 128-row tile of one expert's rows in expert order, or of the
// shared expert's token rows, and one part of the FFN width F):
//
//   phase 1  [gate | up] = X_tile . [W_gate | W_up]^T in 128-column chunks of F
//            (tcgen05.mma M=128 x N=256, A = the tile's x rows gathered through
//            the expert-order permutation by cp.async, B = 128 gate and 128 up
//            weight rows by TMA); the epilogue forms h = silu(gate) * up
//            (Laguna-M.1-base spec sheet, Feed-forward: SwiGLU, no bias),
//            rounds it to fp16 and stores it back into tensor memory
//            (tcgen05.st), so h never leaves the SM;
//   phase 2  o = h . W_down^T in 128-column tiles of d (tcgen05.mma M=128 x N=128
//            with the A operand read from tensor memory, B = fp16 W_down rows
//            by TMA, K = the part's width); the epilogue multiplies each row by
//            routed_scaling_factor * w (the 2.5 modulation of the routed sum,
//            Laguna M.1/XS.2 Technical Report summary, Key claims, report §3.1;
//            1 for the shared expert) and adds it into its token's fp32
//            accumulator row with bulk reduce-adds: the weighted combine and the
//            shared-expert add happen in this epilogue.
//
// Tensor memory (512 columns x 128 lanes): columns [0, 256) hold the phase-1
// accumulator (gate 0..127, up 128..255), in phase 2 two 128-column
// accumulators (double-buffered, so the epilogue of one d tile overlaps the
// MMAs of the next); columns [256, 256 + Fp/2) hold h as packed fp16 pairs.
// Fp <= 512 is the width of one part of F: a wider FFN is split into parts
// whose partial down projections add into the same token rows.
//
// Roles (one CTA per SM, persistent over items; all waits bounded):
//   warp 0      TMA loads of the B operands into a 4-stage ring of 48 KB
//               (phase 1: gate + up rows, 32 KB; phase 2: two 64-column K
//               boxes of 128 W_down rows, 32 KB);
//   warps 6..13 phase 1: gather the tile's x rows into the stage's A buffer
//               (16 KB, 128B-swizzled) with 16-byte cp.async; phase 2: arrive;
//   warp 1      TMEM allocation; lane 0 issues the MMAs and the commits;
//   warps 2..5  epilogues (each the 32 rows of its TMEM lane quarter).
// No TMA or bulk copy here uses cluster multicast.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gemm_common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "status.cuh"

namespace moe {

using namespace gemm;

namespace {

constexpr int kFStages = 4;
constexpr int kFABytes = kBlockM * kBlockK * 2;  // 16 KB: 128 rows x 64 bf16
constexpr int kFBBytes = 256 * kBlockK * 2;      // 32 KB: 256 rows x 64 16-bit values
constexpr int kFTmemCols = 512;
constexpr int kHCol = 256;                       // first tensor-memory column of h
constexpr int kFGather2Warp = 6;
constexpr int kFThreads = 192 + 32 * kGatherWarps;

struct FusedSmem {
  static constexpr int a_off = 0;
  static constexpr int b_off = a_off + kFStages * kFABytes;
  static constexpr int epi_off = b_off + kFStages * kFBBytes;  // 4 warps x 8 KB staging
  static constexpr int bar_off = epi_off + 4 * kEpiBytesPerWarp;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int n_bars = 2 * kFStages + 5;
  static constexpr int tmem_slot_off = bar_off + n_bars * 8;
  static constexpr int total = tmem_slot_off + 16;
};
static_assert(FusedSmem::total + 1024 <= 232448, "shared memory budget");

// One item: a row tile and a part of the FFN width.
struct FItem {
  int group;   // expert id, E = shared expert
  int row0;    // first expert-order row (token id for the shared expert)
  int nrows;   // valid rows (<= 128)
  int fbase;   // first column of F (of Fs) this part covers
  int fw;      // width of the part (a multiple of 128, <= 512)
  bool skip;   // part index beyond this group's parts
};

__device__ __forceinline__ int4 fused_rec(const GemmParams &p, int item, int n_items) {
  if (item >= n_items) return make_int4(0, 0, 0, 0);
  return *reinterpret_cast<const int4 *>(&p.tiles[item / p.n_ntiles]);
}

__device__ __forceinline__ FItem fused_decode(const GemmParams &p, int item, int4 t) {
  FItem it;
  const int part = item % p.n_ntiles;
  it.group = t.x;
  it.row0 = t.y;
  it.nrows = t.z;
  const bool shared = it.group == p.E;
  const int parts = shared ? p.n_parts_sh : p.n_parts;
  it.fw = shared ? p.fp_sh : p.fp;
  it.fbase = part * it.fw;
  it.skip = part >= parts;
  return it;
}

// A role's walk over its items (item, item + step, ...), loading the tile record
// and the status word of the next item one item ahead (as ItemWalk does).
struct FusedWalk {
  int item, step, n_items;
  int4 rec;
  int stop;
  __device__ __forceinline__ FusedWalk(const GemmParams &p, int first, int step_, int n)
      : item(first), step(step_), n_items(n), stop(0) {
    rec = fused_rec(p, item, n_items);
  }
  __device__ __forceinline__ bool current(const GemmParams &p, FItem &it) {
    for (;;) {
      if (item >= n_items || stop) return false;
      it = fused_decode(p, item, rec);
      if (!it.skip) return true;
      item += step;
      rec = fused_rec(p, item, n_items);
    }
  }
  __device__ __forceinline__ void prefetch(const GemmParams &p) {
    rec = fused_rec(p, item + step, n_items);
    stop = *reinterpret_cast<const volatile int *>(p.status);
  }
  __device__ __forceinline__ void next() { item += step; }
};

// The gather helpers of gemm_common.cuh take an Item; the fused item maps onto
// its group, first row and valid rows.
__device__ __forceinline__ Item as_item(const FItem &f) {
  Item it;
  it.group = f.group;
  it.row0 = f.row0;
  it.nrows = f.nrows;
  it.j = 0;
  it.nk = 0;
  it.kb0 = 0;
  it.skip = false;
  return it;
}

// Phase-1 epilogue: h = silu(gate) * up of this thread's row for the chunk's
// 128 columns, fp16, into tensor memory at h_col (64 packed columns).
__device__ __forceinline__ void swiglu_to_tmem(const GemmParams &p, bool valid, uint32_t taddr,
                                               uint32_t h_taddr) {
  float amax = 0.f;
#pragma unroll 1
  for (int cb = 0; cb < 128; cb += 32) {  // 32 gate and the matching 32 up columns
    uint32_t g[16], u[16], hp[16];
    tmem_ld_32x32b_x16(taddr + cb, g);
    tmem_ld_32x32b_x16(taddr + 128 + cb, u);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float h0 = swiglu(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i]));
      const float h1 = swiglu(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1]));
      amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
      hp[i] = pack_f16x2(h0, h1);
    }
    tmem_ld_32x32b_x16(taddr + cb + 16, g);
    tmem_ld_32x32b_x16(taddr + 128 + cb + 16, u);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float h0 = swiglu(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i]));
      const float h1 = swiglu(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1]));
      amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
      hp[8 + i] = pack_f16x2(h0, h1);
    }
    tmem_st_32x32b_x16(h_taddr + cb / 2, hp);
  }
  tmem_st_wait();
  if (valid && amax > kF16Max) record_status(p.status, MOE_ERR_DEVICE_BOUNDS, SITE_H_FP16_RANGE);
}

}  // namespace

__global__ void __launch_bounds__(kFThreads, 1)
    moe_fused_kernel(const __grid_constant__ GemmParams p,
                     const __grid_constant__ CUtensorMap tm_gate,
                     const __grid_constant__ CUtensorMap tm_up,
                     const __grid_constant__ CUtensorMap tm_down,
                     const __grid_constant__ CUtensorMap tm_gate_sh,
                     const __grid_constant__ CUtensorMap tm_up_sh,
                     const __grid_constant__ CUtensorMap tm_down_sh) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem + FusedSmem::a_off;
  uint8_t *sB = smem + FusedSmem::b_off;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + FusedSmem::bar_off);
  uint64_t *full = bars;
  uint64_t *empty = bars + kFStages;
  uint64_t *acc_full = bars + 2 * kFStages;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + FusedSmem::tmem_slot_off);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages; ++s) {
      // one expect_tx arrival for the B boxes plus one arrival from each
      // gathering lane (a cp.async completion in phase 1, a plain arrive in phase 2)
      mbar_init(&full[s], 1 + 32 * kGatherWarps);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4 * 32);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_gate);
    prefetch_tmap(&tm_up);
    prefetch_tmap(&tm_down);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kFTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_items = *p.n_tiles_dev * p.n_ntiles;
  const int nkd = p.d / kBlockK;   // phase-1 K stages (64 columns of d each)
  const int nd = p.d / 128;        // phase-2 d tiles
  int *status = p.status;

  if (warp == 0 || warp >= kFGather2Warp) {
    // ------------------------------------------------------------ loads
    const bool tma_warp = warp == 0;
    const int gw = warp - kFGather2Warp;  // gathering warp index (warps 6..)
    int s = 0;
    uint32_t ph = 0;
    long long issued = 0;
    bool ok = true;
    FusedWalk walk(p, blockIdx.x, gridDim.x, n_items);
    FItem fi;
    int raw[kGatherGroups];
    while (ok && walk.current(p, fi)) {
      const Item it = as_item(fi);
      const bool shared = fi.group == p.E;
      int tok[kGatherGroups];
      if (!tma_warp) {
        gather_rows_fetch(p, it, lane, gw, raw);
        gather_tokens(p, it, raw, tok);
      }
      walk.prefetch(p);
      const int nf = fi.fw / 128;
      const int nkf = fi.fw / 128;  // phase-2 K stages (128 columns of the part each)
      const int n_stages = nf * nkd + nd * nkf;
      for (int st = 0; st < n_stages && ok; ++st) {
        const bool ph1 = st < nf * nkd;
        int good = 1;
        if (lane == 0) {
          good = mbar_wait(&empty[s], ph ^ 1, status, SITE_GEMM_PRODUCER_EMPTY);
          if (good && tma_warp) mbar_arrive_expect_tx(&full[s], kFBBytes);
        }
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) {
          ok = false;
          break;
        }
        uint8_t *a_dst = sA + s * kFABytes;
        uint8_t *b_dst = sB + s * kFBBytes;
        if (ph1) {
          const int fc = st / nkd, kb = st - fc * nkd;
          const int kc = kb * kBlockK;
          if (tma_warp) {
            if (lane == 0) {
              const int brow = (shared ? 0 : fi.group * p.F) + fi.fbase + fc * 128;
              tma_load_2d(b_dst, shared ? &tm_gate_sh : &tm_gate, &full[s], kc, brow);
              tma_load_2d(b_dst + 128 * 128, shared ? &tm_up_sh : &tm_up, &full[s], kc, brow);
            }
          } else {
            gather_a_stage<MODE_GEMM1>(p, tok, lane, gw, a_dst, &full[s], kc);
          }
        } else {
          const int q = st - nf * nkd;
          const int dn = q / nkf, ks = q - dn * nkf;
          if (tma_warp) {
            if (lane == 0) {
              const int brow = (shared ? 0 : fi.group * p.d) + dn * 128;
              const int kc = fi.fbase + ks * 128;
              const CUtensorMap *tm = shared ? &tm_down_sh : &tm_down;
              tma_load_2d(b_dst, tm, &full[s], kc, brow);
              tma_load_2d(b_dst + 128 * 128, tm, &full[s], kc + 64, brow);
            }
          } else {
            mbar_arrive(&full[s]);
          }
        }
        ++issued;
        if (++s == kFStages) {
          s = 0;
          ph ^= 1;
        }
      }
      walk.next();
    }
    if (!tma_warp) cp_async_wait_all();
    if (tma_warp && lane == 0) {
      for (long long n = (issued > kFStages ? issued - kFStages : 0); n < issued; ++n)
        if (!mbar_wait(&full[n % kFStages], static_cast<uint32_t>((n / kFStages) & 1), status,
                       SITE_GEMM_DRAIN))
          break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_bf16_f32(kBlockM, 256);
      const uint32_t idesc2 = idesc_f16_f32(kBlockM, 128);
      int s = 0;
      uint32_t ph = 0;
      uint32_t eph[2] = {0, 0};  // phase of each half's acc_empty (uses so far)
      bool ok = true;
      FusedWalk walk(p, blockIdx.x, gridDim.x, n_items);
      FItem fi;
      auto wait_full = [&]() -> bool {
        if (!mbar_wait(&full[s], ph, status, SITE_GEMM_MMA_FULL)) return false;
        return true;
      };
      auto advance = [&]() {
        if (++s == kFStages) {
          s = 0;
          ph ^= 1;
        }
      };
      while (ok && walk.current(p, fi)) {
        walk.prefetch(p);
        walk.next();
        const int nf = fi.fw / 128;
        const int nkf = fi.fw / 128;
        // phase 1: each 128-column chunk of the part into the wide accumulator [0, 256)
        for (int fc = 0; fc < nf && ok; ++fc) {
          if (!mbar_wait(&acc_empty[0], eph[0] ^ 1, status, SITE_GEMM_MMA_ACC_EMPTY) ||
              !mbar_wait(&acc_empty[1], eph[1] ^ 1, status, SITE_GEMM_MMA_ACC_EMPTY)) {
            ok = false;
            break;
          }
          eph[0] ^= 1;
          eph[1] ^= 1;
          tc_fence_after();
          for (int kb = 0; kb < nkd; ++kb) {
            if (!wait_full()) {
              ok = false;
              break;
            }
            fence_proxy_async_smem();  // A was written by cp.async
            tc_fence_after();
            const uint32_t a0 = smem_u32(sA + s * kFABytes);
            const uint32_t b0 = smem_u32(sB + s * kFBBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f16_ss(tmem_base, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32),
                          idesc1, (kb | kk) != 0);
            umma_commit(&empty[s]);
            advance();
          }
          if (!ok) break;
          umma_commit(&acc_full[0]);
          umma_commit(&acc_full[1]);
        }
        // phase 2: d tiles of 128 columns, A = h in tensor memory, alternating halves
        for (int dn = 0; dn < nd && ok; ++dn) {
          const int hb = dn & 1;
          if (!mbar_wait(&acc_empty[hb], eph[hb] ^ 1, status, SITE_GEMM_MMA_ACC_EMPTY)) {
            ok = false;
            break;
          }
          eph[hb] ^= 1;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + hb * 128;
          for (int ks = 0; ks < nkf; ++ks) {
            if (!wait_full()) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t b0 = smem_u32(sB + s * kFBBytes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // K = 128: two 64-column boxes of W_down
              umma_f16_ts(d_tmem, tmem_base + kHCol + ks * 64 + kk * 8,
                          smem_desc_sw128(b0 + (kk >> 2) * (128 * 128) + (kk & 3) * 32), idesc2,
                          (ks | kk) != 0);
            umma_commit(&empty[s]);
            advance();
          }
          if (!ok) break;
          umma_commit(&acc_full[hb]);
        }
      }
      umma_commit(drain);
      mbar_wait(drain, 0, status, SITE_GEMM_DRAIN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q * 32 + lane;
    EpiStage st{smem + FusedSmem::epi_off + (warp - 2) * kEpiBytesPerWarp, 0};
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t fph[2] = {0, 0};
    FusedWalk walk(p, blockIdx.x, gridDim.x, n_items);
    FItem fi;
    bool ok = true;
    while (ok && walk.current(p, fi)) {
      walk.prefetch(p);
      walk.next();
      const Item it = as_item(fi);
      const bool valid = row_local < fi.nrows;
      const bool quarter = q * 32 < fi.nrows;  // this warp's quarter holds a valid row
      const int nf = fi.fw / 128;
      for (int fc = 0; fc < nf; ++fc) {
        if (!mbar_wait(&acc_full[0], fph[0], status, SITE_GEMM_EPI_ACC_FULL) ||
            !mbar_wait(&acc_full[1], fph[1], status, SITE_GEMM_EPI_ACC_FULL)) {
          ok = false;
          break;
        }
        fph[0] ^= 1;
        fph[1] ^= 1;
        tc_fence_after();
        // every warp stores its quarter's h (rows past the tile only feed rows the
        // phase-2 epilogue discards)
        swiglu_to_tmem(p, valid && quarter, lane_base, lane_base + kHCol + fc * 64);
        tc_fence_before();
        mbar_arrive(&acc_empty[0]);
        mbar_arrive(&acc_empty[1]);
      }
      for (int dn = 0; dn < nd && ok; ++dn) {
        const int hb = dn & 1;
        if (!mbar_wait(&acc_full[hb], fph[hb], status, SITE_GEMM_EPI_ACC_FULL)) {
          ok = false;
          break;
        }
        fph[hb] ^= 1;
        tc_fence_after();
        if (quarter) down_epilogue_reduce_cols(p, it, lane_base + hb * 128, row_local, st,
                                               dn * 128, 128);
        tc_fence_before();
        mbar_arrive(&acc_empty[hb]);
      }
    }
    bulk_wait_all();  // this thread's reductions have completed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kFTmemCols);
  }
}

size_t gemm_fused_smem_bytes() { return FusedSmem::total + 1024; }

cudaError_t launch_gemm_fused(const GemmParams &p, const FusedMaps &m, int grid, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = gemm_fused_smem_bytes();
  cfg.stream = s;
  return cudaLaunchKernelEx(&cfg, moe_fused_kernel, p, m.gate, m.up, m.down, m.gate_sh, m.up_sh,
                            m.down_sh);
}

cudaError_t gemm_fused_set_attributes() {
  return cudaFuncSetAttribute(moe_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(gemm_fused_smem_bytes()));
}

}  // namespace moe
