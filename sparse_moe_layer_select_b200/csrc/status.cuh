// status.cuh -- device-side status word, site ids and the wait bound.
#pragma once
#include <cstdint>

#include "../../include/moe.h"

namespace moe {

// About one second at the B200's 1.9 GHz boost clock.
constexpr long long kWaitLimitCycles = 2000000000LL;

// Where a device-side error was detected (written next to the status code).
enum Site : int {
  SITE_NONE = 0,
  SITE_GEMM_PRODUCER_EMPTY = 10,
  SITE_GEMM_MMA_FULL = 11,
  SITE_GEMM_MMA_ACC_EMPTY = 12,
  SITE_GEMM_EPI_ACC_FULL = 13,
  SITE_GEMM_DRAIN = 14,
  SITE_PERMUTE_EXPERT_ID = 20,
  SITE_INDEX_GRID_BARRIER = 21,  // the one-launch index builder's wait for all chunk histograms
  SITE_H_FP16_RANGE = 30,        // SwiGLU activation beyond the fp16 range
  SITE_SLOT_FP16_RANGE = 31,     // scaled expert contribution beyond the fp16 range
  SITE_WEIGHT_FP16_RANGE = 32,   // down-projection weight beyond the fp16 range
  SITE_SELFTEST_FLAG = 90,
};

// Layout of the first 256 bytes of every workspace.
struct WsHeader {
  int status;     // first error code (0 = none)
  int site;       // Site of that error
  int n_tiles;    // 128-row tiles in the expert tile list (written by the index builder)
  int n_tiles_pair;  // 256-row tiles in the second list, when one is built
  int index_done;    // index builder: histogram CTAs finished (the last one scans)
  int index_arrived; // one-launch index builder: CTAs past their histogram (grid barrier)
  int pad[58];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte block");

// Keep the first error only.
__device__ __forceinline__ void record_status(int *status, int code, int site) {
  if (status == nullptr) return;
  if (atomicCAS(status, 0, code) == 0) {
    volatile int *s = status;
    s[1] = site;
    __threadfence();
  }
}

__device__ __forceinline__ bool status_is_set(const int *status) {
  return *reinterpret_cast<const volatile int *>(status) != 0;
}

}  // namespace moe
