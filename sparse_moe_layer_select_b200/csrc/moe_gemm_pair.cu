// moe_gemm_pair.cu -- the expert GEMMs on CTA pairs (clusters of two SMs).
//
// Same work as MODE_GEMM1 / MODE_GEMM2 of moe_gemm.cu (gate/up GEMM with
// the SwiGLU epilogue, down GEMM with the modulation epilogue), but each item
// is a 256-row tile computed by one tcgen05.mma.cta_group::2 per K step
// (M = 256, N <= 256): each SM of the pair holds its own 128 rows of A and
// half of the N rows of B, so a pipeline stage is 32 KB per SM instead of
// 48 KB and six stages fit, while every B byte brought into shared memory
// feeds 256 rows of tokens.  For the gate/up GEMM the leader CTA loads the
// gate rows and its peer the up rows of the same column block.
//
// Synchronisation (all waits bounded, as in moe_gemm.cu):
//   lfull[s]   GEMM1, per CTA: its own loads of stage s have landed (TMA bytes
//              and cp.async arrivals)
//   gather     GEMM1's A rows are copied by warps 7.. (each a share of the
//              128 rows, gemm_common.cuh); warp 0 issues the TMA loads
//   relay      GEMM1: warp 6 of the peer CTA forwards each of its completed
//              stages to the leader's full[s], after a proxy fence for the
//              cp.async-written rows (a cp.async completion can only arrive on
//              a barrier of its own CTA)
//   full[s]    GEMM1, leader: the peer's half of stage s is in shared memory
//              (the leader's MMA thread waits on its own lfull[s] for its
//              half).  GEMM2 (all loads by TMA), leader: both halves are in
//              shared memory -- each CTA's TMA loads complete on the leader's
//              full[s] (.cta_group::2), the leader arms it for both CTAs' bytes
//   empty[s]   per CTA: the leader's MMAs of stage s completed (commit
//              multicast to both CTAs)
//   acc_full   per CTA: an accumulator is complete (commit multicast)
//   acc_empty  leader: the eight epilogue warps of both CTAs drained it
// No TMA or bulk copy in this kernel uses cluster multicast.
#include <cuda_bf16.h>

#include "gemm_common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "status.cuh"

namespace moe {

using namespace gemm;

namespace {

constexpr int kPairStages = 6;
// warps: 0 TMA loads, 1 MMA, 2-5 epilogue, 6 relay, 7.. gather (GEMM1)
constexpr int kPairGather2Warp = 7;
constexpr int kPairThreads = 224 + 32 * kExtraGatherWarps;
constexpr int kPABytes = kBlockM * kBlockK * 2;  // 16 KB: this CTA's 128 rows of A
constexpr int kPBBytes = 128 * kBlockK * 2;      // 16 KB: this CTA's half of B (<= 128 rows)
constexpr int kPTmemCols = 512;
constexpr int kPAccStride = 256;

struct PairSmem {
  static constexpr int a_off = 0;
  static constexpr int b_off = a_off + kPairStages * kPABytes;
  static constexpr int epi_off = b_off + kPairStages * kPBBytes;  // 4 warps x 8 KB staging
  static constexpr int bar_off = epi_off + 4 * kEpiBytesPerWarp;
  // full[S], lfull[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int n_bars = 3 * kPairStages + 5;
  static constexpr int tmem_slot_off = bar_off + n_bars * 8;
  static constexpr int total = tmem_slot_off + 16;
};
static_assert(PairSmem::total + 1024 <= 232448, "shared memory budget");

}  // namespace

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    moe_gemm_pair_kernel(const __grid_constant__ GemmParams p,
                         const __grid_constant__ CUtensorMap tm_a,
                         const __grid_constant__ CUtensorMap tm_b0,
                         const __grid_constant__ CUtensorMap tm_b1,
                         const __grid_constant__ CUtensorMap tm_a_sh,
                         const __grid_constant__ CUtensorMap tm_b0_sh,
                         const __grid_constant__ CUtensorMap tm_b1_sh,
                         const __grid_constant__ CUtensorMap tm_out,
                         const __grid_constant__ CUtensorMap tm_out_sh) {
  constexpr int BASE = MODE & 3;  // the GEMM; MODE_RED: the reduce-combine epilogue
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem + PairSmem::a_off;
  uint8_t *sB = smem + PairSmem::b_off;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + PairSmem::bar_off);
  uint64_t *full = bars;
  uint64_t *lfull = bars + kPairStages;
  uint64_t *empty = bars + 2 * kPairStages;
  uint64_t *acc_full = bars + 3 * kPairStages;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + PairSmem::tmem_slot_off);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      // GEMM1: the peer's relayed arrival (the leader waits on its own lfull);
      // GEMM2: the leader's expect-tx arrival for both CTAs' bytes
      mbar_init(&full[s], 1);
      // own loads: one expect_tx arrival (+ one cp.async arrival per gathering lane)
      mbar_init(&lfull[s], BASE == MODE_GEMM1 ? 1 + 32 * kGatherWarps : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_b0);
    prefetch_tmap(&tm_b1);
    prefetch_tmap(&tm_a);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kPTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_items = (*p.n_tiles_dev) * p.n_ntiles;
  const int cluster_id = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  int *status = p.status;
  const int half_b_rows = BASE == MODE_GEMM1 ? p.n_half : p.n_tile / 2;

  if (warp == 0 || warp >= kPairGather2Warp) {
    // ------------------------------------------------------------ loads
    // Warp 0 issues the TMA loads (and arms each stage's barrier); the
    // gathering warps (warp 0 too when kTmaWarpGathers) copy GEMM1's A rows,
    // kGatherRows each.
    const bool tma_warp = warp == 0;
    const int gw = tma_warp ? (kTmaWarpGathers ? 0 : -1)
                            : (kTmaWarpGathers ? 1 : 0) + (warp - kPairGather2Warp);
    const bool gathers = BASE == MODE_GEMM1 && gw >= 0;
    if (tma_warp || gathers) {
      // GEMM2: both CTAs' TMA loads complete on the leader's full[s]
      const uint32_t leader_full0 = map_shared_rank(smem_u32(&full[0]), 0);
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      ItemWalk<MODE> walk(p, cluster_id, n_clusters, n_items);
      Item whole;
      // GEMM1: row ids of this warp's rows of item raw_item (loaded one item ahead).
      int raw[kGatherGroups];
      int raw_item = -1;
      while (ok && walk.current(p, whole)) {
        const Item it = pair_half(whole, rank);
        const bool shared = it.group == p.E;
        int tok[kGatherGroups];
        if (gathers) {
          if (raw_item != walk.item) gather_rows_fetch(p, it, lane, gw, raw);
          gather_tokens(p, it, raw, tok);
        }
        walk.prefetch(p);
        const uint32_t bytes = BASE == MODE_GEMM1
                                   ? static_cast<uint32_t>(half_b_rows * 128)
                                   : (shared ? p.a_sh_bytes : p.a_bytes) + half_b_rows * 128;
        for (int kb = 0; kb < whole.nk; ++kb) {
          int good = 1;
          if (tma_warp && lane == 0) MOE_TRACE_AT(p, TR_PWAIT, issued);
          if (lane == 0) {
            good = mbar_wait(&empty[s], ph ^ 1, status, SITE_GEMM_PRODUCER_EMPTY);
            if (good && tma_warp) {
              if (BASE == MODE_GEMM1) mbar_arrive_expect_tx(&lfull[s], bytes);
              else if (leader) mbar_arrive_expect_tx(&full[s], 2 * bytes);  // equal boxes per CTA
            }
          }
          good = __shfl_sync(0xffffffffu, good, 0);
          if (!good) {
            ok = false;
            break;
          }
          if (tma_warp && lane == 0) MOE_TRACE_AT(p, TR_ISSUE, issued);
          uint8_t *a_dst = sA + s * kPABytes;
          uint8_t *b_dst = sB + s * kPBBytes;
          const int kc = kb * kBlockK;
          if (tma_warp && lane == 0) {
            if (BASE == MODE_GEMM1) {
              // leader: gate rows; peer: up rows of the same column block
              const int brow = (shared ? 0 : it.group * p.F) + it.j * p.n_half;
              const CUtensorMap *tm =
                  leader ? (shared ? &tm_b0_sh : &tm_b0) : (shared ? &tm_b1_sh : &tm_b1);
              tma_load_2d(b_dst, tm, &lfull[s], kc, brow);
            } else {
              const uint32_t bar = leader_full0 + s * 8;
              tma_load_2d_pair(a_dst, shared ? &tm_a_sh : &tm_a, bar, kc, it.row0);
              const int brow = (shared ? 0 : it.group * p.d) + it.j * p.n_tile + rank * half_b_rows;
              tma_load_2d_pair(b_dst, shared ? &tm_b0_sh : &tm_b0, bar, kc, brow);
            }
          }
          if (gathers) gather_a_stage<MODE>(p, tok, lane, gw, a_dst, &lfull[s], kc);
          if (tma_warp && lane == 0) MOE_TRACE_AT(p, TR_PDONE, issued);
          ++issued;
          if (++s == kPairStages) {
            s = 0;
            ph ^= 1;
          }
          if (gathers && kb == 0) {
            // Row ids of the next item; its tile record was loaded at this
            // item's start.  Skipped items are fetched when reached.
            const Item nx = decode_tile<MODE>(p, walk.item + walk.step, walk.rec);
            raw_item = -1;
            if (walk.item + walk.step < n_items && !nx.skip) {
              gather_rows_fetch(p, pair_half(nx, rank), lane, gw, raw);
              raw_item = walk.item + walk.step;
            }
          }
        }
        walk.next();
      }
      // Every stage filled must have landed before the CTA exits.  GEMM2: the
      // leader's full[] counts both CTAs' bytes, and the peer stays until the
      // leader reaches the closing cluster barrier.
      if (gathers) cp_async_wait_all();
      if (tma_warp && lane == 0 && (BASE == MODE_GEMM1 || leader)) {
        uint64_t *landed = BASE == MODE_GEMM1 ? lfull : full;
        for (long long n = (issued > kPairStages ? issued - kPairStages : 0); n < issued; ++n)
          if (!mbar_wait(&landed[n % kPairStages], static_cast<uint32_t>((n / kPairStages) & 1),
                         status, SITE_GEMM_DRAIN))
            break;
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ relay (peer CTA)
    // The leader's MMA thread waits on the leader's own lfull; only the peer's
    // completed stages are forwarded, one remote arrival each on the leader's full.
    if (BASE == MODE_GEMM1 && lane == 0 && !leader) {
      const uint32_t leader_full0 = map_shared_rank(smem_u32(&full[0]), 0);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int relayed = 0;
      ItemWalk<MODE> walk(p, cluster_id, n_clusters, n_items);
      Item whole;
      while (ok && walk.current(p, whole)) {
        walk.prefetch(p);
        walk.next();
        for (int kb = 0; kb < whole.nk; ++kb) {
          if (!mbar_wait(&lfull[s], ph, status, SITE_GEMM_MMA_FULL)) {
            ok = false;
            break;
          }
          MOE_TRACE_AT(p, TR_LANDED, relayed);
          ++relayed;
          if (BASE == MODE_GEMM1) fence_proxy_async_smem();  // rows written by cp.async
          mbar_arrive_cluster(leader_full0 + s * 8);
          if (++s == kPairStages) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      const uint32_t idesc = BASE == MODE_GEMM2 ? idesc_f16_f32(2 * kBlockM, p.n_tile)
                                                : idesc_bf16_f32(2 * kBlockM, p.n_tile);
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      int consumed = 0;
      ItemWalk<MODE> walk(p, cluster_id, n_clusters, n_items);
      Item it;
      while (ok && walk.current(p, it)) {
        walk.prefetch(p);
        walk.next();
        if (!mbar_wait(&acc_empty[acc], aph ^ 1, status, SITE_GEMM_MMA_ACC_EMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kPAccStride;
        for (int kb = 0; kb < it.nk; ++kb) {
          // this CTA's half of the stage (its loads), then the peer's (relayed)
          if ((BASE == MODE_GEMM1 && !mbar_wait(&lfull[s], ph, status, SITE_GEMM_MMA_FULL)) ||
              !mbar_wait(&full[s], ph, status, SITE_GEMM_MMA_FULL)) {
            ok = false;
            break;
          }
          MOE_TRACE_AT(p, TR_FULL, consumed);
          if (BASE == MODE_GEMM1) fence_proxy_async_smem();  // own rows written by cp.async
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kPABytes);
          const uint32_t b0 = smem_u32(sB + s * kPBBytes);
#pragma unroll
          for (int kk = 0; kk < kBlockK / 16; ++kk)
            umma_f16_ss_pair(d_tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32),
                             idesc, (kb | kk) != 0);
          umma_commit_pair_multicast(&empty[s], 0x3);
          MOE_TRACE_AT(p, TR_MMA, consumed);
          ++consumed;
          if (++s == kPairStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair_multicast(&acc_full[acc], 0x3);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1;
        }
      }
      umma_commit_pair_multicast(drain, 0x1);
      mbar_wait(drain, 0, status, SITE_GEMM_DRAIN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    const uint32_t leader_acc_empty0 = map_shared_rank(smem_u32(&acc_empty[0]), 0);
    EpiStage st{smem + PairSmem::epi_off + (warp - 2) * kEpiBytesPerWarp, 0};
    int acc = 0;
    uint32_t aph = 0;
    int done = 0;
    ItemWalk<MODE> walk(p, cluster_id, n_clusters, n_items);
    Item whole;
    while (walk.current(p, whole)) {
      walk.prefetch(p);
      walk.next();
      if (!mbar_wait(&acc_full[acc], aph, status, SITE_GEMM_EPI_ACC_FULL)) break;
      if (warp == 2 && lane == 0) MOE_TRACE_AT(p, TR_EPI_START, done);
      tc_fence_after();
      const Item it = pair_half(whole, rank);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kPAccStride;
      if (BASE == MODE_GEMM1) swiglu_epilogue<false>(p, it, taddr, row_local, st, &tm_out, &tm_out_sh);
      else if (MODE & MODE_RED) down_epilogue_reduce(p, it, taddr, row_local, st);
      else down_epilogue<false>(p, it, taddr, row_local, st, &tm_out, &tm_out_sh);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_acc_empty0 + acc * 8);
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
  cluster_sync();  // no CTA leaves while its peer may still read its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kPTmemCols);
  }
}

size_t gemm_pair_smem_bytes() { return PairSmem::total + 1024; }

cudaError_t launch_gemm_pair(int mode, const GemmParams &p, const GemmMaps &m, int grid,
                             cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = gemm_pair_smem_bytes();
  cfg.stream = s;
  if (mode == MODE_GEMM1)
    return cudaLaunchKernelEx(&cfg, moe_gemm_pair_kernel<MODE_GEMM1>, p, m.a, m.b0, m.b1, m.a_sh,
                              m.b0_sh, m.b1_sh, m.out, m.out_sh);
  if (mode == MODE_GEMM2_RED)
    return cudaLaunchKernelEx(&cfg, moe_gemm_pair_kernel<MODE_GEMM2_RED>, p, m.a, m.b0, m.b1,
                              m.a_sh, m.b0_sh, m.b1_sh, m.out, m.out_sh);
  if (mode == MODE_GEMM2)
    return cudaLaunchKernelEx(&cfg, moe_gemm_pair_kernel<MODE_GEMM2>, p, m.a, m.b0, m.b1, m.a_sh,
                              m.b0_sh, m.b1_sh, m.out, m.out_sh);
  return cudaErrorInvalidValue;
}

cudaError_t gemm_pair_set_attributes() {
  const int smem = static_cast<int>(gemm_pair_smem_bytes());
  cudaError_t e = cudaFuncSetAttribute(moe_gemm_pair_kernel<MODE_GEMM1>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_pair_kernel<MODE_GEMM2_RED>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(moe_gemm_pair_kernel<MODE_GEMM2>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

// How many CTA pairs can be resident at once.  A pair needs two SMs of one
// GPC, so on a GPU whose GPCs have odd SM counts this is below SMs / 2; the
// persistent grid must not exceed it, or the surplus pairs run as a second
// wave after the others finish.
cudaError_t gemm_pair_max_clusters(int *clusters) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = gemm_pair_smem_bytes();
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n1 = 0, n2 = 0;
  cudaError_t e = cudaOccupancyMaxActiveClusters(&n1, moe_gemm_pair_kernel<MODE_GEMM1>, &cfg);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveClusters(&n2, moe_gemm_pair_kernel<MODE_GEMM2>, &cfg);
  if (e != cudaSuccess) return e;
  *clusters = n1 < n2 ? n1 : n2;
  return cudaSuccess;
}

}  // namespace moe
