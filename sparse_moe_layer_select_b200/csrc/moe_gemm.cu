// moe_gemm.cu -- persistent, warp-specialised tcgen05 GEMM for the MoE layer.
//
// One kernel template serves the three contractions of the layer:
//
//   MODE_ROUTER  logits[128 tokens, n_tile experts] = x_tile . W_r^T (+ b), fp32 in TMEM,
//                written out for the warp-per-token selection (sigmoid router
//                with post-top-k normalisation: Laguna M.1/XS.2 Technical
//                Report summary, Key claims, report §3.1).
//   MODE_GEMM1   [gate | up] = X_perm . [W_gate | W_up]^T for one expert and
//                one column block; the rows of X_perm are gathered from x
//                through the expert-order permutation by 16-byte cp.async
//                copies written straight into the swizzled operand layout, so
//                the permuted activations are never written out.  The
//                epilogue applies SwiGLU, h = silu(gate) * up, and stores h in
//                fp16 (Laguna-M.1-base spec sheet, Feed-forward: SwiGLU, no bias).
//   MODE_GEMM2   o = h . W_down^T (fp16 operands, fp32 accumulation) for one
//                expert and one d-column block; the
//                epilogue multiplies each row by routed_scaling_factor * w
//                (the 2.5 modulation of the routed sum: Technical Report
//                summary, report §3.1) and writes it, in fp16, to its
//                expert-order row of O (the combine reads O through the
//                inverse permutation); shared-expert rows go, unscaled, to
//                the token's row of S.
//   MODE_F8 | *  the same two expert GEMMs on e4m3 operands (tcgen05
//                kind::f8f6f4, K=32 per instruction); the epilogues apply the
//                per-row activation scale and per-column weight scale.
//
// Roles inside a CTA (one CTA per SM, persistent over items):
//   warp 0      producer: fills a kStages-deep ring of (A, B) stages with
//               TMA tiles (GEMM1: the B tiles only).
//   warps 6..   GEMM1: kGatherWarps warps gather the A rows by cp.async
//               through the expert-order permutation, an equal share of the
//               128 rows each (gemm_common.cuh).
//   warp 1      allocates 512 TMEM columns; lane 0 issues tcgen05.mma
//               (M=128, N<=256, K=16 per instruction) into one of two
//               accumulator buffers and commits stage releases.
//   warps 2..5  epilogue: tcgen05.ld the finished accumulator (each thread
//               owns one row), compute, store; release the buffer, so the
//               MMA of the next item overlaps this epilogue.
// Every wait is bounded (status.cuh); on expiry the kernel records
// MOE_ERR_DEVICE_TIMEOUT, drains what it issued, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cfloat>

#include "gemm_common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "status.cuh"

namespace moe {

using namespace gemm;

namespace {

constexpr int kABytes = kBlockM * kBlockK * 2;  // 16 KB: 128 rows x 128 bytes
constexpr int kBBytesMax = 256 * kBlockK * 2;   // 32 KB: up to 256 rows
constexpr int kTmemCols = 512;                  // two accumulators of up to 256 columns
constexpr int kAccStride = 256;
// warps: 0 TMA loads, 1 MMA, 2-5 epilogue, 6.. gather (GEMM1)
constexpr int kGather2Warp = 6;
constexpr int kSingleThreads = 192 + 32 * kExtraGatherWarps;

struct SmemLayout {
  static constexpr int a_off = 0;
  static constexpr int b_off = a_off + kStages * kABytes;
  // epilogue output staging (4 warps x 8 KB); the router's bias table reuses it
  static constexpr int epi_off = b_off + kStages * kBBytesMax;
  static constexpr int bias_off = epi_off;
  static constexpr int bar_off = epi_off + 4 * kEpiBytesPerWarp;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int n_bars = 2 * kStages + 5;
  static constexpr int tmem_slot_off = bar_off + n_bars * 8;
  static constexpr int total = tmem_slot_off + 16;
};
static_assert(SmemLayout::total + 1024 <= 232448, "shared memory budget");

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kSingleThreads, 1)
    moe_gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b0,
                    const __grid_constant__ CUtensorMap tm_b1,
                    const __grid_constant__ CUtensorMap tm_a_sh,
                    const __grid_constant__ CUtensorMap tm_b0_sh,
                    const __grid_constant__ CUtensorMap tm_b1_sh,
                    const __grid_constant__ CUtensorMap tm_out,
                    const __grid_constant__ CUtensorMap tm_out_sh) {
  // BASE: the GEMM this launch computes; F8: e4m3 operands (MODE_F8 bit).
  constexpr int BASE = MODE & 3;
  constexpr bool F8 = (MODE & MODE_F8) != 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem + SmemLayout::a_off;
  uint8_t *sB = smem + SmemLayout::b_off;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SmemLayout::bar_off);
  uint64_t *full = bars;
  uint64_t *empty = bars + kStages;
  uint64_t *acc_full = bars + 2 * kStages;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout::tmem_slot_off);
  float *bias_s = reinterpret_cast<float *>(smem + SmemLayout::bias_off);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // GEMM1: one expect_tx arrival for the B tiles plus one cp.async
      // completion arrival from each lane of the gathering warps.
      mbar_init(&full[s], BASE == MODE_GEMM1 ? 1 + 32 * kGatherWarps : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4 * 32);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (BASE == MODE_ROUTER) {
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) bias_s[e] = p.bias ? p.bias[e] : 0.f;
    for (int e = p.E + threadIdx.x; e < 512; e += blockDim.x) bias_s[e] = 0.f;
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b0);
    if (BASE == MODE_GEMM1) prefetch_tmap(&tm_b1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_items = (BASE == MODE_ROUTER) ? p.n_tiles_host * p.n_ntiles * p.ksplit
                                            : *p.n_tiles_dev * p.n_ntiles;
  // The down projection multiplies fp16 h by fp16 W_down, the others bf16 operands; F8
  // launches e4m3 (whose format code equals fp16's).
  const uint32_t idesc = (BASE == MODE_GEMM2 || F8) ? idesc_f16_f32(kBlockM, p.n_tile)
                                                     : idesc_bf16_f32(kBlockM, p.n_tile);
  int *status = p.status;

  if (warp == 0 || warp >= kGather2Warp) {
    // ------------------------------------------------------------ loads
    // Warp 0 issues the TMA loads (and arms each stage's barrier); the
    // gathering warps (warp 0 too when kTmaWarpGathers) copy GEMM1's A rows,
    // kGatherRows each.
    const bool tma_warp = warp == 0;
    const int gw = tma_warp ? (kTmaWarpGathers ? 0 : -1)
                            : (kTmaWarpGathers ? 1 : 0) + (warp - kGather2Warp);
    const bool gathers = BASE == MODE_GEMM1 && gw >= 0;
    if (tma_warp || gathers) {
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      ItemWalk<MODE> walk(p, blockIdx.x, gridDim.x, n_items);
      Item it;
      // GEMM1: row ids of this warp's rows of item raw_item (loaded one item ahead).
      int raw[kGatherGroups];
      int raw_item = -1;
      while (ok && walk.current(p, it)) {
        const bool shared = it.group == p.E;
        int tok[kGatherGroups];
        if (gathers) {
          if (raw_item != walk.item) gather_rows_fetch(p, it, lane, gw, raw);
          gather_tokens(p, it, raw, tok);
        }
        walk.prefetch(p);
        // A boxes shorter than 128 rows (tensors with fewer rows) fill only
        // their rows; the rest of the stage feeds accumulator rows that the
        // epilogue discards.
        uint32_t bytes;
        if (BASE == MODE_ROUTER) bytes = p.a_bytes + p.n_tile * 128;
        else if (BASE == MODE_GEMM1) bytes = 2 * p.n_half * 128;  // A arrives by cp.async
        else bytes = (shared ? p.a_sh_bytes : p.a_bytes) + p.n_tile * 128;
        for (int kb = 0; kb < it.nk; ++kb) {
          int good = 1;
          if (tma_warp && lane == 0) MOE_TRACE_AT(p, TR_PWAIT, issued);
          if (lane == 0) {
            good = mbar_wait(&empty[s], ph ^ 1, status, SITE_GEMM_PRODUCER_EMPTY);
            if (good && tma_warp) mbar_arrive_expect_tx(&full[s], bytes);
          }
          good = __shfl_sync(0xffffffffu, good, 0);
          if (!good) {
            ok = false;
            break;
          }
          if (tma_warp && lane == 0) MOE_TRACE_AT(p, TR_ISSUE, issued);
          uint8_t *a_dst = sA + s * kABytes;
          uint8_t *b_dst = sB + s * kBBytesMax;
          const int kc = (it.kb0 + kb) * stage_k(MODE);
          if (tma_warp && lane == 0) {
            if (BASE == MODE_GEMM1) {
              const int brow = (shared ? 0 : it.group * p.F) + it.j * p.n_half;
              tma_load_2d(b_dst, shared ? &tm_b0_sh : &tm_b0, &full[s], kc, brow);
              tma_load_2d(b_dst + p.n_half * 128, shared ? &tm_b1_sh : &tm_b1, &full[s], kc, brow);
            } else if (BASE == MODE_ROUTER) {
              tma_load_2d(a_dst, &tm_a, &full[s], kc, it.row0);
              tma_load_2d(b_dst, &tm_b0, &full[s], kc, it.j * p.n_tile);
            } else {
              tma_load_2d(a_dst, shared ? &tm_a_sh : &tm_a, &full[s], kc, it.row0);
              const int brow = (shared ? 0 : it.group * p.d) + it.j * p.n_tile;
              tma_load_2d(b_dst, shared ? &tm_b0_sh : &tm_b0, &full[s], kc, brow);
            }
          }
          if (gathers) gather_a_stage<MODE>(p, tok, lane, gw, a_dst, &full[s], kc);
          if (tma_warp && lane == 0) MOE_TRACE_AT(p, TR_PDONE, issued);
          ++issued;
          if (++s == kStages) {
            s = 0;
            ph ^= 1;
          }
          if (gathers && kb == 0) {
            // Row ids of the next item; its tile record was loaded at this
            // item's start.  Skipped items are fetched when reached.
            const Item nx = decode_tile<MODE>(p, walk.item + walk.step, walk.rec);
            raw_item = -1;
            if (walk.item + walk.step < n_items && !nx.skip) {
              gather_rows_fetch(p, nx, lane, gw, raw);
              raw_item = walk.item + walk.step;
            }
          }
        }
        walk.next();
      }
      // Every stage filled must have landed before the CTA exits.
      if (gathers) cp_async_wait_all();
      if (tma_warp && lane == 0) {
        for (long long n = (issued > kStages ? issued - kStages : 0); n < issued; ++n)
          if (!mbar_wait(&full[n % kStages], static_cast<uint32_t>((n / kStages) & 1), status,
                         SITE_GEMM_DRAIN))
            break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      int consumed = 0;
      ItemWalk<MODE> walk(p, blockIdx.x, gridDim.x, n_items);
      Item it;
      while (ok && walk.current(p, it)) {
        walk.prefetch(p);
        walk.next();
        if (!mbar_wait(&acc_empty[acc], aph ^ 1, status, SITE_GEMM_MMA_ACC_EMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccStride;
        for (int kb = 0; kb < it.nk; ++kb) {
          if (!mbar_wait(&full[s], ph, status, SITE_GEMM_MMA_FULL)) {
            ok = false;
            break;
          }
          MOE_TRACE_AT(p, TR_FULL, consumed);
          if (BASE == MODE_GEMM1) fence_proxy_async_smem();  // A was written by cp.async
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kABytes);
          const uint32_t b0 = smem_u32(sB + s * kBBytesMax);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 4 x 32 bytes of the 128-byte rows
            if (F8)
              umma_f8_ss(d_tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32),
                         idesc, (kb | kk) != 0);
            else
              umma_f16_ss(d_tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32),
                          idesc, (kb | kk) != 0);
          }
          umma_commit(&empty[s]);
          MOE_TRACE_AT(p, TR_MMA, consumed);
          ++consumed;
          if (++s == kStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1;
        }
      }
      // All MMAs issued by this thread complete before TMEM is released.
      umma_commit(drain);
      mbar_wait(drain, 0, status, SITE_GEMM_DRAIN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    if (MODE == MODE_GEMM2_F8 && warp == 2 && lane == 0) {
      // The FP8 down epilogue multiplies by one scale per output column, read
      // from the [E, d] (and [d]) float32 tables as each item starts; each CTA
      // asks L2 for its share of the tables up front, so that those reads,
      // on the epilogue's critical path, find them there.
      const size_t total = static_cast<size_t>(p.E) * p.d * 4;
      const size_t share = ((total + gridDim.x - 1) / gridDim.x + 15) & ~static_cast<size_t>(15);
      const size_t off = static_cast<size_t>(blockIdx.x) * share;
      if (off < total)
        prefetch_l2_bulk(reinterpret_cast<const char *>(p.sb0) + off,
                         static_cast<uint32_t>(total - off < share ? total - off : share));
      if (blockIdx.x == 0 && p.Fs > 0 && p.sb0_sh != nullptr)
        prefetch_l2_bulk(p.sb0_sh, static_cast<uint32_t>(p.d) * 4);
    }
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q * 32 + lane;
    EpiStage st{smem + SmemLayout::epi_off + (warp - 2) * kEpiBytesPerWarp, 0};
    int acc = 0;
    uint32_t aph = 0;
    int done = 0;
    ItemWalk<MODE> walk(p, blockIdx.x, gridDim.x, n_items);
    Item it;
    while (walk.current(p, it)) {
      walk.prefetch(p);
      walk.next();
      if (!mbar_wait(&acc_full[acc], aph, status, SITE_GEMM_EPI_ACC_FULL)) break;
      if (warp == 2 && lane == 0) MOE_TRACE_AT(p, TR_EPI_START, done);
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccStride;
      if (BASE == MODE_ROUTER) {
        router_epilogue(p, it, taddr, row_local, bias_s);
      } else if (BASE == MODE_GEMM1) {
        swiglu_epilogue<F8>(p, it, taddr, row_local, st, &tm_out, &tm_out_sh);
      } else if (MODE & MODE_RED) {
        down_epilogue_reduce(p, it, taddr, row_local, st);
      } else {
        down_epilogue<F8>(p, it, taddr, row_local, st, &tm_out, &tm_out_sh);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (warp == 2 && lane == 0) MOE_TRACE_AT(p, TR_EPI_END, done);
      ++done;
      if (++acc == 2) {
        acc = 0;
        aph ^= 1;
      }
    }
    bulk_wait_all();  // this thread's output stores / reductions are complete
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

size_t gemm_smem_bytes() { return SmemLayout::total + 1024; }

cudaError_t launch_gemm(int mode, const GemmParams &p, const GemmMaps &m, int grid,
                        cudaStream_t s) {
  const size_t smem = gemm_smem_bytes();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSingleThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  switch (mode) {
    case MODE_ROUTER:
      return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<MODE_ROUTER>, p, m.a, m.b0, m.b1, m.a_sh,
                                m.b0_sh, m.b1_sh, m.out, m.out_sh);
    case MODE_GEMM1:
      return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<MODE_GEMM1>, p, m.a, m.b0, m.b1, m.a_sh,
                                m.b0_sh, m.b1_sh, m.out, m.out_sh);
    case MODE_GEMM2:
      return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<MODE_GEMM2>, p, m.a, m.b0, m.b1, m.a_sh,
                                m.b0_sh, m.b1_sh, m.out, m.out_sh);
    case MODE_GEMM1_F8:
      return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<MODE_GEMM1_F8>, p, m.a, m.b0, m.b1, m.a_sh,
                                m.b0_sh, m.b1_sh, m.out, m.out_sh);
    case MODE_GEMM2_F8:
      return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<MODE_GEMM2_F8>, p, m.a, m.b0, m.b1, m.a_sh,
                                m.b0_sh, m.b1_sh, m.out, m.out_sh);
    case MODE_GEMM2_RED:
      return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<MODE_GEMM2_RED>, p, m.a, m.b0, m.b1, m.a_sh,
                                m.b0_sh, m.b1_sh, m.out, m.out_sh);
    default:
      return cudaErrorInvalidValue;
  }
}

// Raise the dynamic shared-memory limit of the three instantiations (once per device).
cudaError_t gemm_set_attributes() {
  const int smem = static_cast<int>(gemm_smem_bytes());
  cudaError_t e;
  e = cudaFuncSetAttribute(moe_gemm_kernel<MODE_ROUTER>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_kernel<MODE_GEMM1>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_kernel<MODE_GEMM2>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_kernel<MODE_GEMM1_F8>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_kernel<MODE_GEMM2_RED>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(moe_gemm_kernel<MODE_GEMM2_F8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

}  // namespace moe
