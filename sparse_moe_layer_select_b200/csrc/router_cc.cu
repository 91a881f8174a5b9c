// router_cc.cu -- CUDA-core router logits (small token counts and shapes
// outside the tensor-core router's limits) and the selection kernel that
// both logit paths feed.
//
// Sigmoid router with post-top-k normalisation (Laguna M.1/XS.2 Technical
// Report summary, Key claims, report §3.1; Laguna-M.1-base spec sheet,
// Mixture of experts: sigmoid router scores, top-k renormalisation on).
//
//   router_logits_kernel  fp32 logits[T, E] = x . W_r^T (+ b): a CTA stages
//                         8 token rows in shared memory; each warp computes
//                         two experts' logits for those 8 tokens (16-byte
//                         loads of W_r, fp32 FMA, warp butterfly reduction).
//   router_select_kernel  one warp per token, for both logit paths: the E
//                         logits sit in registers (E/32 per lane) as
//                         order-preserving integer keys; each lane keeps the
//                         top three of its keys (rebuilt when all three are
//                         taken), and k+1 rounds of a warp arg-max over the
//                         lanes' heads (a max- then a min-reduction, ties to
//                         the lower expert index) pick the experts in
//                         descending order; tokens whose
//                         k-th and (k+1)-th logits are within kRefineBand get
//                         the experts near that boundary re-decided on float64
//                         logits; sigmoid and normalisation in fp32.  When
//                         the tensor-core router split d into K slices, the
//                         warp first sums the slices' partial logits (slice
//                         order) and writes the sum back to the first plane.
//   router_select_index_kernel  the same, then, for a batch whose T * k
//                         entries form one index chunk, the index builder
//                         (index_common.cuh) in whichever CTA finishes last.
#include <cuda_bf16.h>

#include <cfloat>

#include "gemm_common.cuh"
#include "index_common.cuh"
#include "kernels.h"
#include "status.cuh"

namespace moe {

using gemm::kRefineBand;

namespace {

constexpr int kTokPerCta = 8;
constexpr int kWarpsPerCta = 8;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// kExpPerWarp experts per warp: 2 when the whole grid fits on the SMs at one
// CTA each (small batches; 142 registers), else 1 (84 registers, several CTAs
// per SM to hide the memory round trips of many CTA waves).
template <int kExpPerWarp>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    router_logits_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ w_router,
                         const float *__restrict__ bias, float *__restrict__ logits, int T, int d,
                         int E) {
  extern __shared__ uint4 xs4[];  // [kTokPerCta][d] bf16
  const int t0 = blockIdx.x * kTokPerCta;
  const int nt = min(kTokPerCta, T - t0);
  const int vec_per_row = d / 8;
  const int n_vec = kTokPerCta * vec_per_row;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // This lane's weight vectors of the warp's kExpPerWarp expert rows,
  // kWLoads per row in flight at a time.
  constexpr int kWLoads = 8;
  uint4 wv[kExpPerWarp][kWLoads];
  auto load_w = [&](int e0, int c0) {
#pragma unroll
    for (int j = 0; j < kExpPerWarp; ++j) {
      const uint4 *wr = reinterpret_cast<const uint4 *>(w_router + static_cast<size_t>(e0 + j) * d);
#pragma unroll
      for (int u = 0; u < kWLoads; ++u) {
        const int c = c0 + 32 * u;
        wv[j][u] = (e0 + j < E && c < vec_per_row) ? wr[c] : make_uint4(0, 0, 0, 0);
      }
    }
  };
  // The first experts' first batch of weights is requested before the token
  // rows are staged, so that the two memory round trips overlap.
  const int e_first = (blockIdx.y * kWarpsPerCta + warp) * kExpPerWarp;
  if (e_first < E) load_w(e_first, lane);
  bool have_w = e_first < E;
  // Stage the tokens: each thread's loads are issued together (kStageLoads at
  // a time), then stored, so the staging costs about one memory round trip.
  constexpr int kStageLoads = 8;
  for (int i0 = threadIdx.x; i0 < n_vec; i0 += kStageLoads * blockDim.x) {
    uint4 v[kStageLoads];
#pragma unroll
    for (int u = 0; u < kStageLoads; ++u) {
      const int i = i0 + u * blockDim.x;
      const int r = i / vec_per_row;
      v[u] = (i < n_vec && r < nt)
                 ? reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t0 + r) * d)[i - r * vec_per_row]
                 : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kStageLoads; ++u)
      if (i0 + u * blockDim.x < n_vec) xs4[i0 + u * blockDim.x] = v[u];
  }
  __syncthreads();
  // Each staged x vector read from shared memory feeds all kExpPerWarp
  // experts (the reads, not the FMAs, bound this loop); every logit keeps the
  // same products in the same order.
  for (int e0 = e_first; e0 < E; e0 += gridDim.y * kWarpsPerCta * kExpPerWarp) {
    float acc[kExpPerWarp][kTokPerCta];
#pragma unroll
    for (int j = 0; j < kExpPerWarp; ++j)
#pragma unroll
      for (int r = 0; r < kTokPerCta; ++r) acc[j][r] = 0.f;
    for (int c0 = lane; c0 < vec_per_row; c0 += 32 * kWLoads) {
      if (!have_w) load_w(e0, c0);
      have_w = false;
#pragma unroll
      for (int u = 0; u < kWLoads; ++u) {
        const int c = c0 + 32 * u;
        if (c >= vec_per_row) break;
        float wf[kExpPerWarp][8];
#pragma unroll
        for (int j = 0; j < kExpPerWarp; ++j) bf16x8_to_f32(wv[j][u], wf[j]);
#pragma unroll
        for (int r = 0; r < kTokPerCta; ++r) {
          float xf[8];
          bf16x8_to_f32(xs4[r * vec_per_row + c], xf);
#pragma unroll
          for (int j = 0; j < kExpPerWarp; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[j][r] = fmaf(xf[i], wf[j][i], acc[j][r]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kExpPerWarp; ++j)
#pragma unroll
      for (int r = 0; r < kTokPerCta; ++r) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          acc[j][r] += __shfl_xor_sync(0xffffffffu, acc[j][r], off);
      }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < kExpPerWarp; ++j) {
        const int e = e0 + j;
        if (e >= E) break;
        const float b = bias ? bias[e] : 0.f;
        for (int r = 0; r < nt; ++r) logits[static_cast<size_t>(t0 + r) * E + e] = acc[j][r] + b;
      }
    }
  }
}

constexpr int kSelectWarps = 8;
// CTAs per SM the selection kernels are compiled for: four 8-warp CTAs (<= 64
// registers a thread) keep a 4096-token batch within one wave on 148 SMs.
constexpr int kSelectCtasPerSm = 4;

// kRefineBand (gemm_common.cuh): width of the ambiguous band around the
// k-th/(k+1)-th boundary, in logit units.  It is far above twice the largest
// fp32 logit error of either logit path at these widths (tensor-core
// accumulation up to 1.2e-5, CUDA-core FMA below 4e-6), so every expert
// outside the band is on the right side of the boundary, and the band is
// decided on float64 logits.

// float64 logits of up to four experts e[0..n) for one token: exact bf16
// products, float64 sums (lane-strided, then a butterfly in fixed order), plus
// the bias.  The token row is read once per group; the loads of a batch of
// chunks are issued before any is used (the register budget of the selection
// kernels bounds the batch).
__device__ __forceinline__ void logits_f64_x4(const uint16_t *__restrict__ x,
                                              const uint16_t *__restrict__ w_router,
                                              const float *__restrict__ bias, int t,
                                              const int (&e)[4], int n, int d, int lane,
                                              double (&out)[4]) {
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t) * d);
  const uint4 *wr[4];
#pragma unroll
  for (int g = 0; g < 4; ++g)
    wr[g] = reinterpret_cast<const uint4 *>(w_router + static_cast<size_t>(g < n ? e[g] : e[0]) * d);
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  const int nvec = d / 8;
  if (n <= 2) {
    // The usual band of one or two experts: four of the lane's chunks of the
    // three rows in flight at once (the loads of a batch are issued before any
    // is used), so the rows cost two memory round trips at d = 2048.
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
    for (int c0 = lane; c0 < nvec; c0 += 4 * 32) {
      uint4 xv[4], wv0[4], wv1[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int c = c0 + 32 * b;
        xv[b] = c < nvec ? xr[c] : zero;
        wv0[b] = c < nvec ? wr[0][c] : zero;
        wv1[b] = (c < nvec && n > 1) ? wr[1][c] : zero;
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float xf[8], wf0[8], wf1[8];
        bf16x8_to_f32(xv[b], xf);
        bf16x8_to_f32(wv0[b], wf0);
        bf16x8_to_f32(wv1[b], wf1);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          acc[0] = fma(static_cast<double>(xf[i]), static_cast<double>(wf0[i]), acc[0]);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          acc[1] = fma(static_cast<double>(xf[i]), static_cast<double>(wf1[i]), acc[1]);
      }
    }
  } else {
#pragma unroll 4
    for (int c = lane; c < nvec; c += 32) {
      float xf[8];
      bf16x8_to_f32(xr[c], xf);
      uint4 wv[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) wv[g] = wr[g][c];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float wf[8];
        bf16x8_to_f32(wv[g], wf);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          acc[g] = fma(static_cast<double>(xf[i]), static_cast<double>(wf[i]), acc[g]);
      }
    }
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], off);
    out[g] = acc[g] + ((bias && g < n) ? static_cast<double>(bias[e[g]]) : 0.0);
  }
}

// Order-preserving fp32 -> uint32 key (IEEE sign-magnitude to unsigned
// order); -0 is folded onto +0 and NaN onto 0, below every number.
__device__ __forceinline__ uint32_t logit_key(float f) {
  if (f != f) return 0u;
  const uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_logit(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// One warp per token: each lane keeps the top three of its NPL = E/32 logits
// (registers only); each of the k+1 rounds then takes the warp arg-max of the
// 32 list heads (ties to the lower expert id) and the winning lane pops its
// head, rebuilding its list from its remaining logits when it runs empty.  Tokens whose k-th and (k+1)-th logits are
// within kRefineBand get the experts near that boundary re-decided on
// float64 logits.  Then sigmoid scores and post-top-k normalisation (Laguna
// M.1/XS.2 Technical Report summary, Key claims, report §3.1; Laguna-M.1-base
// spec sheet, Mixture of experts).

// Per-warp scratch of the float64 re-decision: the band members' ids and
// values, then the places they take.
struct RefineScratch {
  double vals[32];
  int ids[32];
  int out_e[16];
  float out_l[16];
};

// The float64 re-decision of a token whose k-th and (k+1)-th selection values
// (lk, lk1) are within kRefineBand: the band's experts (nband of them, the
// first 32 in rs->ids in ascending id, found by the caller from the values it
// holds) are ranked on float64 values and fill the places after the experts
// above the band (my_l / my_e of lanes 0..k-1 are updated).  Kept out of line:
// it runs for few tokens, and inlined its float64 state would crowd the
// registers of every token's path.
__device__ __noinline__ void refine_band(int t, int lane, RefineScratch *rs, const float *row,
                                         const uint16_t *__restrict__ x,
                                         const uint16_t *__restrict__ w_router,
                                         const float *__restrict__ bias,
                                         const float *__restrict__ sel_bias, int d, int E, int k,
                                         float lk, float lk1, int nband, float &my_l, int &my_e) {
  auto sel_value = [&](int e) -> float {
    const float l = row[e];
    return sel_bias ? 1.f / (1.f + expf(-l)) + sel_bias[e] : l;
  };

    // The fp32 selection values are within kRefineBand / 4 of their float64
    // values, so with mid the midpoint of the k-th and (k+1)-th values:
    // experts above mid + kRefineBand are in the float64 top k, those below
    // mid - kRefineBand are not.  Only the experts inside the band are
    // re-decided on float64 values; they fill the places after the ones
    // above the band.
    const float mid = 0.5f * (lk + lk1);
    const float lo = mid - kRefineBand, hi = mid + kRefineBand;
    const int above = __popc(__ballot_sync(0xffffffffu, lane < k && my_l > hi));
    const int nslice = (E + 31) / 32;
    __syncwarp();
    if (nband <= 32) {
      for (int g0 = 0; g0 < nband; g0 += 4) {
        int eg[4];
        const int ng = min(4, nband - g0);
#pragma unroll
        for (int g = 0; g < 4; ++g) eg[g] = rs->ids[g0 + (g < ng ? g : 0)];
        double lg[4];
        logits_f64_x4(x, w_router, bias, t, eg, ng, d, lane, lg);
        if (lane < ng) {
          const double l = lane == 0 ? lg[0] : lane == 1 ? lg[1] : lane == 2 ? lg[2] : lg[3];
          rs->vals[g0 + lane] =
              sel_bias ? 1.0 / (1.0 + exp(-l)) + static_cast<double>(sel_bias[eg[lane]]) : l;
        }
      }
      __syncwarp();
      if (lane < nband) {  // rank: descending float64 value, lower id first on ties
        const double vc = rs->vals[lane];
        const int ec = rs->ids[lane];
        int rank = 0;
        for (int j = 0; j < nband; ++j) {
          const double vj = rs->vals[j];
          rank += (vj > vc || (vj == vc && rs->ids[j] < ec)) ? 1 : 0;
        }
        if (above + rank < k) {
          rs->out_e[above + rank] = ec;
          rs->out_l[above + rank] = static_cast<float>(vc);
        }
      }
      __syncwarp();
      if (lane >= above && lane < k) {
        my_e = rs->out_e[lane];
        my_l = rs->out_l[lane];
      }
      __syncwarp();
    } else {
      // More than 32 experts in the band (degenerate, e.g. many equal
      // logits): every expert from the lower band edge up is re-decided,
      // streamed four at a time into a sorted list on lane 0.
      double best_l[16];
      int best_e[16];
      int nbest = 0;
      int eg[4] = {0, 0, 0, 0};
      int ng = 0;
      for (int i = 0; i <= nslice; ++i) {
        unsigned m = 0;
        if (i < nslice) {
          const int e_lane = lane + 32 * i;
          m = __ballot_sync(0xffffffffu, e_lane < E && sel_value(e_lane) >= lo);
        }
        while (m || (i == nslice && ng > 0)) {
          while (m && ng < 4) {
            eg[ng++] = (__ffs(m) - 1) + 32 * i;
            m &= m - 1;
          }
          if (ng < 4 && i < nslice) break;  // group not full: take more from the next slice
          double lg[4];
          logits_f64_x4(x, w_router, bias, t, eg, ng, d, lane, lg);
          if (lane == 0) {
            for (int g = 0; g < ng; ++g) {
              // sorted insert, descending value, lower id first on ties (ids arrive ascending)
              const double l = sel_bias
                                   ? 1.0 / (1.0 + exp(-lg[g])) + static_cast<double>(sel_bias[eg[g]])
                                   : lg[g];
              int pos = nbest < k ? nbest : k;
              while (pos > 0 && l > best_l[pos - 1]) --pos;
              if (pos < k) {
                const int last = nbest < k ? nbest : k - 1;
                for (int q = last; q > pos; --q) {
                  best_l[q] = best_l[q - 1];
                  best_e[q] = best_e[q - 1];
                }
                best_l[pos] = l;
                best_e[pos] = eg[g];
                if (nbest < k) ++nbest;
              }
            }
          }
          ng = 0;
        }
      }
      for (int q = 0; q < k; ++q) {  // hand the list to lanes 0..k-1
        const float lq =
            __shfl_sync(0xffffffffu, lane == 0 ? static_cast<float>(best_l[q]) : 0.f, 0);
        const int eq = __shfl_sync(0xffffffffu, lane == 0 ? best_e[q] : 0, 0);
        if (lane == q) {
          my_l = lq;
          my_e = eq;
        }
      }
    }
  }

template <int NPL>
__device__ __forceinline__ void select_token(int t, int lane, RefineScratch *rs,
                                             float *__restrict__ logits, int nsplit, int T,
                                             const uint16_t *__restrict__ x,
                                             const uint16_t *__restrict__ w_router,
                                             const float *__restrict__ bias,
                                             const float *__restrict__ sel_bias, int d, int E,
                                             int k, int norm_topk, int32_t *__restrict__ topk_idx,
                                             float *__restrict__ topk_w) {
  float *row = logits + static_cast<size_t>(t) * E;
  // This lane's logits (experts lane + 32 i): all loads first, one memory
  // round trip.  With K slices (nsplit <= 4) the partial planes are summed in
  // slice order and the sum is written back into plane 0, where the rest of
  // the selection (and any later reader) finds the logits.
  float lv[NPL];
  if (nsplit == 1) {
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const int e = lane + 32 * i;
      lv[i] = e < E ? row[e] : 0.f;
    }
  } else {
    const size_t plane = static_cast<size_t>(T) * E;
    float part[4][NPL];
#pragma unroll
    for (int sl = 0; sl < 4; ++sl)
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        part[sl][i] = (sl < nsplit && e < E) ? row[sl * plane + e] : 0.f;
      }
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      float l = part[0][i];
#pragma unroll
      for (int sl = 1; sl < 4; ++sl)
        if (sl < nsplit) l += part[sl][i];
      lv[i] = l;
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (lane + 32 * i < E) row[lane + 32 * i] = lv[i];
    __syncwarp();
  }
  // The selection value of expert e with logit l: l, or with a selection-only
  // bias sigmoid(l) + b_e (the weights below always use the logit).
  auto sel_of = [&](int e, float l) -> float {
    return sel_bias ? 1.f / (1.f + expf(-l)) + sel_bias[e] : l;
  };
  auto sel_value = [&](int e) -> float { return sel_of(e, row[e]); };
  // Keys: an order-preserving map of the fp32 selection value to uint32, plus
  // one (larger value, larger key; +0 and -0 equal; NaN the lowest value, key
  // 1); 0 marks an empty entry (and the padding slots past E).
  uint32_t key[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? logit_key(sel_of(e, lv[i])) + 1u : 0u;
  }
  // Each lane keeps the top three of its remaining slots in (key descending,
  // slot ascending) order -- slot i holds expert lane + 32 i, so equal keys keep
  // the lower expert id first.  "Remaining" are the slots after the last one
  // this lane gave up; when all three are taken the list is rebuilt from them.
  uint32_t hk0, hk1, hk2;
  int hi0, hi1, hi2;
  auto build = [&](uint32_t last_k, int last_i) {
    hk0 = hk1 = hk2 = 0u;
    hi0 = hi1 = hi2 = NPL;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const uint32_t u = key[i];
      if (!(u < last_k || (u == last_k && i > last_i))) continue;
      if (u > hk0) {
        hk2 = hk1; hi2 = hi1;
        hk1 = hk0; hi1 = hi0;
        hk0 = u;   hi0 = i;
      } else if (u > hk1) {
        hk2 = hk1; hi2 = hi1;
        hk1 = u;   hi1 = i;
      } else if (u > hk2) {
        hk2 = u;   hi2 = i;
      }
    }
  };
  build(0xffffffffu, -1);
  float my_l = 0.f;  // lane j < k keeps the j-th selected logit and expert
  int my_e = 0;
  float lk = 0.f, lk1 = -INFINITY;
  const int rounds = k < E ? k + 1 : k;
  for (int j = 0; j < rounds; ++j) {
    // the largest head key, then the lowest expert id among the heads holding it
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, hk0);
    const uint32_t mine = (hk0 == kmax && hk0 != 0u) ? static_cast<uint32_t>(lane + 32 * hi0)
                                                     : 0xffffffffu;
    const uint32_t ewin = __reduce_min_sync(0xffffffffu, mine);
    if (mine == ewin) {  // this lane's head is taken
      const uint32_t tk = hk0;
      const int ti = hi0;
      hk0 = hk1; hi0 = hi1;
      hk1 = hk2; hi1 = hi2;
      hk2 = 0u;  hi2 = NPL;
      if (hk0 == 0u) build(tk, ti);
    }
    const float lj = key_logit(kmax - 1u);
    if (j < k && lane == j) {
      my_l = lj;
      my_e = static_cast<int>(ewin);
    }
    if (j == k - 1) lk = lj;
    if (j == k) lk1 = lj;
  }

  if (k < E && lk - lk1 < kRefineBand) {
    // The band's members in ascending id, from the selection values this lane
    // holds as keys (no memory round trip); the first 32 go to rs->ids.
    const float mid = 0.5f * (lk + lk1);
    const float lo = mid - kRefineBand, hi = mid + kRefineBand;
    const unsigned lt = (1u << lane) - 1u;
    int nband = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      const float v = key_logit(key[i] - 1u);
      const bool in = key[i] != 0u && v >= lo && v <= hi;
      const unsigned b = __ballot_sync(0xffffffffu, in);
      const int pos = nband + __popc(b & lt);
      if (in && pos < 32) rs->ids[pos] = lane + 32 * i;
      nband += __popc(b);
    }
    __syncwarp();
    refine_band(t, lane, rs, row, x, w_router, bias, sel_bias, d, E, k, lk, lk1, nband, my_l,
                my_e);
  }

  // With a selection-only bias the rounds carried sigmoid(l) + b: the weights
  // take the selected experts' own logits.
  if (sel_bias && lane < k) my_l = row[my_e];
  const float s = 1.f / (1.f + expf(-my_l));
  float sum = lane < k ? s : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < k) {
    const size_t o = static_cast<size_t>(t) * k + lane;
    topk_idx[o] = my_e;
    topk_w[o] = norm_topk ? s / sum : s;
  }
}

// Routes one token per warp (padding tokens get kNotRouted ids and zero weights).
template <int NPL>
__device__ __forceinline__ void select_or_pad(int t, int lane, RefineScratch *rs, float *logits,
                                              int nsplit, int T, const uint16_t *x,
                                              const uint16_t *w_router, const float *bias,
                                              const float *sel_bias, const uint8_t *token_mask,
                                              int d, int E, int k, int norm_topk,
                                              int32_t *topk_idx, float *topk_w) {
  if (token_mask != nullptr && token_mask[t] == 0) {
    if (lane < k) {
      topk_idx[static_cast<size_t>(t) * k + lane] = kNotRouted;
      topk_w[static_cast<size_t>(t) * k + lane] = 0.f;
    }
    return;
  }
  select_token<NPL>(t, lane, rs, logits, nsplit, T, x, w_router, bias, sel_bias, d, E, k,
                    norm_topk, topk_idx, topk_w);
}

template <int NPL>
__global__ void __launch_bounds__(kSelectWarps * 32, kSelectCtasPerSm)
    router_select_kernel(float *__restrict__ logits, int nsplit, const uint16_t *__restrict__ x,
                         const uint16_t *__restrict__ w_router, const float *__restrict__ bias,
                         const float *__restrict__ sel_bias,
                         const uint8_t *__restrict__ token_mask, int T, int d, int E, int k,
                         int norm_topk,
                         int32_t *__restrict__ topk_idx, float *__restrict__ topk_w) {
  __shared__ RefineScratch scratch[kSelectWarps];
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelectWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  select_or_pad<NPL>(t, lane, &scratch[threadIdx.x >> 5], logits, nsplit, T, x, w_router, bias,
                     sel_bias, token_mask, d, E, k, norm_topk, topk_idx, topk_w);
}

// The same selection, then, for a batch whose T * k entries form a single
// index chunk (decode-sized), the index builder in the CTA that finishes
// last (a ticket in the workspace header; the other CTAs simply exit): the
// expert order and tile lists come out of this launch, with no index launch
// and no second read of the routing from a cold kernel.  Needs E <= 256 (one
// scan thread per expert).
template <int NPL>
__global__ void __launch_bounds__(kSelectWarps * 32, kSelectCtasPerSm)
    router_select_index_kernel(float *__restrict__ logits, int nsplit,
                               const uint16_t *__restrict__ x,
                               const uint16_t *__restrict__ w_router,
                               const float *__restrict__ bias, const float *__restrict__ sel_bias,
                               const uint8_t *__restrict__ token_mask, int T, int d, int E, int k,
                               int norm_topk, int32_t *__restrict__ topk_idx,
                               float *__restrict__ topk_w, SelectIndexOut ix) {
  __shared__ RefineScratch scratch[kSelectWarps];
  __shared__ int h[idx::kIdxWarps * idx::kMaxE];
  __shared__ int warp_sums[32];
  __shared__ int totals[3];
  __shared__ int ticket;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelectWarps + (threadIdx.x >> 5);
  if (t < T)
    select_or_pad<NPL>(t, lane, &scratch[threadIdx.x >> 5], logits, nsplit, T, x, w_router, bias,
                       sel_bias, token_mask, d, E, k, norm_topk, topk_idx, topk_w);
  __threadfence();  // this CTA's routing is visible before its ticket is taken
  __syncthreads();
  if (threadIdx.x == 0)
    ticket = atomicAdd(&reinterpret_cast<WsHeader *>(ix.header)->index_done, 1);
  __syncthreads();
  if (ticket != static_cast<int>(gridDim.x) - 1) return;
  __threadfence();
  idx::index_single_cta(topk_idx, T * k, E, T, ix.with_shared, ix.chunk_hist, ix.counts,
                        ix.offsets, ix.perm, ix.inv, ix.tiles, ix.tiles_pair, ix.header, h,
                        warp_sums, totals);
}

template <int kExpPerWarp>
cudaError_t launch_router_logits(const uint16_t *x, const uint16_t *w_router, const float *bias,
                                 float *logits, int T, int d, int E, int gx, int gy,
                                 cudaStream_t s) {
  const size_t smem = static_cast<size_t>(kTokPerCta) * d * 2;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(router_logits_kernel<kExpPerWarp>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  router_logits_kernel<kExpPerWarp><<<dim3(gx, gy), kWarpsPerCta * 32, smem, s>>>(
      x, w_router, bias, logits, T, d, E);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_cc(const uint16_t *x, const uint16_t *w_router, const float *bias,
                             float *logits, int T, int d, int E, int sms, cudaStream_t s) {
  const int gx = (T + kTokPerCta - 1) / kTokPerCta;
  // spread experts over enough CTAs to fill the GPU when T is small
  const int gy2 = (E + 2 * kWarpsPerCta - 1) / (2 * kWarpsPerCta);
  if (static_cast<int64_t>(gx) * gy2 <= sms)
    return launch_router_logits<2>(x, w_router, bias, logits, T, d, E, gx, gy2, s);
  int gy = (E + kWarpsPerCta - 1) / kWarpsPerCta;
  if (gx >= 256) gy = 1;
  return launch_router_logits<1>(x, w_router, bias, logits, T, d, E, gx, gy, s);
}

cudaError_t launch_router_select(float *logits, int nsplit, const uint16_t *x,
                                 const uint16_t *w_router, const float *bias,
                                 const float *sel_bias, const uint8_t *token_mask, int T, int d,
                                 int E, int k, int norm_topk, int32_t *topk_idx, float *topk_w,
                                 cudaStream_t s, const SelectIndexOut *ix, bool *indexed) {
  const int blocks = (T + kSelectWarps - 1) / kSelectWarps;
  const int threads = kSelectWarps * 32;
  const int npl = (E + 31) / 32;
  const bool fuse = ix != nullptr && static_cast<int64_t>(T) * k <= kIndexChunk &&
                    E <= threads && E <= idx::kMaxE;
  if (indexed) *indexed = fuse;
#define MOE_SELECT(N)                                                                           \
  do {                                                                                          \
    if (fuse)                                                                                   \
      router_select_index_kernel<N><<<blocks, threads, 0, s>>>(                                 \
          logits, nsplit, x, w_router, bias, sel_bias, token_mask, T, d, E, k, norm_topk,       \
          topk_idx, topk_w, *ix);                                                               \
    else                                                                                        \
      router_select_kernel<N><<<blocks, threads, 0, s>>>(logits, nsplit, x, w_router, bias,     \
                                                         sel_bias, token_mask, T, d, E, k,      \
                                                         norm_topk, topk_idx, topk_w);          \
  } while (0)
  if (npl <= 1) MOE_SELECT(1);
  else if (npl <= 2) MOE_SELECT(2);
  else if (npl <= 4) MOE_SELECT(4);
  else if (npl <= 8) MOE_SELECT(8);
  else MOE_SELECT(16);
#undef MOE_SELECT
  return cudaGetLastError();
}

}  // namespace moe
