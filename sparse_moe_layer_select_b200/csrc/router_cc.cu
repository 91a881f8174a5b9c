// router_cc.cu -- CUDA-core router for small token counts and shapes outside
// the tensor-core router's limits (E not a multiple of 16, or E > 256).
//
// Sigmoid router with post-top-k normalisation (Laguna M.1/XS.2 Technical
// Report summary, Key claims, report §3.1; Laguna-M.1-base spec sheet,
// Mixture of experts: "Router score: sigmoid", "Renormalize top-k: Yes").
//
//   router_logits_kernel  fp32 logits[T, E] = x . W_r^T (+ b): a CTA stages
//                         8 token rows in shared memory; each warp computes
//                         one expert's logits for those 8 tokens (16-byte
//                         loads of W_r, fp32 FMA, warp butterfly reduction).
//   topk_kernel           one warp per token: the E logits sit in registers
//                         (E/32 per lane); k rounds of a warp arg-max (ties to
//                         the lower expert index) pick the experts in
//                         descending order; sigmoid and normalisation in fp32.
#include <cuda_bf16.h>

#include <cfloat>

#include "kernels.h"

namespace moe {

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

__global__ void __launch_bounds__(kWarpsPerCta * 32)
    router_logits_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ w_router,
                         const float *__restrict__ bias, float *__restrict__ logits, int T, int d,
                         int E) {
  extern __shared__ uint4 xs4[];  // [kTokPerCta][d] bf16
  const int t0 = blockIdx.x * kTokPerCta;
  const int nt = min(kTokPerCta, T - t0);
  const int vec_per_row = d / 8;
  for (int i = threadIdx.x; i < kTokPerCta * vec_per_row; i += blockDim.x) {
    const int r = i / vec_per_row;
    const int c = i - r * vec_per_row;
    xs4[i] = r < nt ? reinterpret_cast<const uint4 *>(x + static_cast<size_t>(t0 + r) * d)[c]
                    : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int e = blockIdx.y * kWarpsPerCta + warp; e < E; e += gridDim.y * kWarpsPerCta) {
    const uint4 *wr = reinterpret_cast<const uint4 *>(w_router + static_cast<size_t>(e) * d);
    float acc[kTokPerCta];
#pragma unroll
    for (int r = 0; r < kTokPerCta; ++r) acc[r] = 0.f;
    for (int c = lane; c < vec_per_row; c += 32) {
      float wf[8];
      bf16x8_to_f32(wr[c], wf);
#pragma unroll
      for (int r = 0; r < kTokPerCta; ++r) {
        float xf[8];
        bf16x8_to_f32(xs4[r * vec_per_row + c], xf);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[r] = fmaf(xf[i], wf[i], acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kTokPerCta; ++r) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], off);
    }
    if (lane == 0) {
      const float b = bias ? bias[e] : 0.f;
      for (int r = 0; r < nt; ++r) logits[static_cast<size_t>(t0 + r) * E + e] = acc[r] + b;
    }
  }
}

constexpr int kMaxPerLane = 16;  // E <= 512

__global__ void __launch_bounds__(256)
    topk_kernel(const float *__restrict__ logits, int T, int E, int k, int norm_topk,
                int32_t *__restrict__ topk_idx, float *__restrict__ topk_w) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const float *row = logits + static_cast<size_t>(warp) * E;
  float v[kMaxPerLane];
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? row[e] : __int_as_float(0x7fc00000);  // NaN: never selected
  }
  float my_s = 0.f;
  int my_e = 0;
  float sum = 0.f;
  for (int j = 0; j < k; ++j) {
    // lane-local best (lowest index on ties: i ascending means e ascending)
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (v[i] > bv || (v[i] == bv && e < be)) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    // remove the winner (NaN compares false, so it is never picked again)
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i)
      if (lane + 32 * i == be) v[i] = __int_as_float(0x7fc00000);
    const float s = 1.f / (1.f + expf(-bv));
    sum += s;
    if (lane == j) {
      my_s = s;
      my_e = be;
    }
  }
  if (lane < k) {
    const size_t o = static_cast<size_t>(warp) * k + lane;
    topk_idx[o] = my_e;
    topk_w[o] = norm_topk ? my_s / sum : my_s;
  }
}

}  // namespace

cudaError_t launch_router_cc(const uint16_t *x, const uint16_t *w_router, const float *bias,
                             float *logits, int T, int d, int E, cudaStream_t s) {
  const int gx = (T + kTokPerCta - 1) / kTokPerCta;
  // spread experts over enough CTAs to fill the GPU when T is small
  int gy = (E + kWarpsPerCta - 1) / kWarpsPerCta;
  if (gx >= 256) gy = 1;
  const size_t smem = static_cast<size_t>(kTokPerCta) * d * 2;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(router_logits_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  router_logits_kernel<<<dim3(gx, gy), kWarpsPerCta * 32, smem, s>>>(x, w_router, bias, logits,
                                                                      T, d, E);
  return cudaGetLastError();
}

cudaError_t launch_topk_from_logits(const float *logits, int T, int E, int k, int norm_topk,
                                    int32_t *topk_idx, float *topk_w, cudaStream_t s) {
  const int threads = 256;
  const int blocks = (T * 32 + threads - 1) / threads;
  topk_kernel<<<blocks, threads, 0, s>>>(logits, T, E, k, norm_topk, topk_idx, topk_w);
  return cudaGetLastError();
}

}  // namespace moe
