// elementwise.cu -- the HBM-bound kernels of the layer.
//
//   gather_rows_kernel  x_perm[r, :] = x[perm[r] / k, :]   (materialised expert-order
//                       activations; the forward pass fuses this gather into the GEMM
//                       operand load instead)
//   combine_kernel      y[t, :] = bf16( sum_j o[inv[t*k + j], :] + s[t, :] ) in fp32 over
//                       the k routed fp16 rows (a padding token's slots have inv = -1
//                       and add nothing) (already scaled by routed_scaling_factor *
//                       w_t,j, stored in expert order) and the shared-expert row: the
//                       combine of the routed sum with the always-on shared expert
//                       (Laguna M.1/XS.2 Technical Report summary, Key claims, report §3.1)
//   finalize_kernel     y = bf16(yacc): the fp32 token rows of the reduce combine
//                       (the down GEMM added every scaled contribution and the
//                       shared-expert row into them) rounded once
//   bf16_to_f16_kernel  fp16 copy of the down-projection weights (round to nearest
//                       even; values beyond the fp16 range are reported)
//   selftest_wait_kernel  a bounded wait on a flag nothing sets (timeout self-test)
//
// All three move 16-byte vectors with one thread per vector, grid-stride.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.h"
#include "status.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ perm,
                       const int32_t *__restrict__ n_valid, int n_rows, int k, int vec_per_row,
                       uint4 *__restrict__ x_perm) {
  const size_t total = static_cast<size_t>(min(*n_valid, n_rows)) * vec_per_row;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / vec_per_row);
    const int c = static_cast<int>(i - static_cast<size_t>(r) * vec_per_row);
    const int t = perm[r] / k;
    x_perm[i] = x[static_cast<size_t>(t) * vec_per_row + c];
  }
}

// One CTA per token row at a time (grid-stride over tokens), one thread per
// 8 output columns: the k routed rows o[inv[t*k + j]] (already scaled by
// routed_scaling_factor * w) are added in slot order, then the shared-expert
// row, all in fp32; one RNE rounding to bf16.  The token's k row indices are
// staged in shared memory one token ahead, so a thread's row loads never
// wait on an index load.
constexpr int kCombineThreads = 256;

template <int KMAX>  // k <= KMAX
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const uint4 *__restrict__ o, const uint4 *__restrict__ s_out,
                   const int32_t *__restrict__ inv, int T, int k, int vec_per_row,
                   uint4 *__restrict__ y) {
  __shared__ int rows[2][16];
  int t = blockIdx.x;
  if (threadIdx.x < k && t < T) rows[0][threadIdx.x] = inv[static_cast<size_t>(t) * k + threadIdx.x];
  __syncthreads();
  int buf = 0;
  for (; t < T; t += gridDim.x) {
    const int tn = t + gridDim.x;
    if (threadIdx.x < k && tn < T)
      rows[buf ^ 1][threadIdx.x] = inv[static_cast<size_t>(tn) * k + threadIdx.x];
    for (int c = threadIdx.x; c < vec_per_row; c += kCombineThreads) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      auto add = [&](const uint4 v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[q]));
          acc[2 * q] += f.x;
          acc[2 * q + 1] += f.y;
        }
      };
      uint4 v[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {  // all row loads first (independent)
        const int r = j < k ? rows[buf][j] : -1;
        v[j] = r >= 0 ? o[static_cast<size_t>(r) * vec_per_row + c] : make_uint4(0, 0, 0, 0);
      }
      const uint4 sv = s_out ? s_out[static_cast<size_t>(t) * vec_per_row + c] : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && rows[buf][j] >= 0) add(v[j]);
      if (s_out) add(sv);
      uint32_t out[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        out[q] = *reinterpret_cast<uint32_t *>(&b2);
      }
      y[static_cast<size_t>(t) * vec_per_row + c] = make_uint4(out[0], out[1], out[2], out[3]);
    }
    __syncthreads();  // next token's indices staged; this token's reads done
    buf ^= 1;
  }
}

// y = bf16(yacc): the reduce combine's fp32 accumulator rounded once (RNE), 8
// values per thread (two 16-byte loads, one 16-byte store), grid-stride.
__global__ void __launch_bounds__(256)
    finalize_kernel(const float4 *__restrict__ yacc, size_t n_vec8, uint4 *__restrict__ y) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_vec8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = __ldcs(&yacc[2 * i]);
    const float4 b = __ldcs(&yacc[2 * i + 1]);
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y);
    const __nv_bfloat162 p1 = __floats2bfloat162_rn(a.z, a.w);
    const __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y);
    const __nv_bfloat162 p3 = __floats2bfloat162_rn(b.z, b.w);
    y[i] = make_uint4(*reinterpret_cast<const uint32_t *>(&p0),
                      *reinterpret_cast<const uint32_t *>(&p1),
                      *reinterpret_cast<const uint32_t *>(&p2),
                      *reinterpret_cast<const uint32_t *>(&p3));
  }
}

// Per-row e4m3 quantization (FP8 experts): one warp per row of K 16-bit
// values (bf16 or fp16 by `is_f16`), s = amax / 448 (1 for an all-zero
// row; rounded up to a power of two for h rows), r = 1 / s, codes = e4m3(v * r) with round to nearest even and
// saturation to +-448; division, reciprocal and product are correctly
// rounded float32 operations.  Rows from *n_valid on (if given) are skipped.
// pow2 != 0: the scale is rounded up to a power of two (exact scaling, so an
// element's code depends on that element alone).
__device__ __forceinline__ float row_scale(float amax, int pow2) {
  if (!(amax > 0.f)) return 1.f;
  const float t = __fdiv_rn(amax, 448.f);
  if (!pow2) return t;
  const uint32_t u = __float_as_uint(t);
  if (u < 0x00800000u) return __uint_as_float(0x00800000u);  // below the normal range: 2^-126
  return (u & 0x007fffffu) ? __uint_as_float((u & 0x7f800000u) + 0x00800000u) : t;
}

__global__ void __launch_bounds__(256)
    quant_rows_e4m3_kernel(const uint16_t *__restrict__ src, int is_f16, int pow2, int rows,
                           const int32_t *__restrict__ n_valid, int K,
                           uint8_t *__restrict__ codes, float *__restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int nrows = n_valid ? min(rows, *n_valid) : rows;
  auto to_f32 = [&](uint16_t b) -> float {
    return is_f16 ? __half2float(__ushort_as_half(b)) : __uint_as_float(static_cast<uint32_t>(b) << 16);
  };
  auto vec_amax = [&](const uint4 v, float m) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      m = fmaxf(m, fmaxf(fabsf(to_f32(w[q] & 0xffffu)), fabsf(to_f32(w[q] >> 16))));
    return m;
  };
  auto vec_codes = [&](const uint4 v, float rcp) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = make_float2(__fmul_rn(to_f32(w[q] & 0xffffu), rcp),
                                   __fmul_rn(to_f32(w[q] >> 16), rcp));
      const uint32_t two = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
      packed[q >> 1] |= (two & 0xffffu) << (16 * (q & 1));
    }
    return make_uint2(packed[0], packed[1]);
  };
  constexpr int kRegVec = 16;  // rows of up to 32 * 16 * 8 = 4096 values stay in registers
  const int nvec = K / 8;
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < nrows; r += warps) {
    const uint4 *row = reinterpret_cast<const uint4 *>(src + static_cast<size_t>(r) * K);
    uint2 *out = reinterpret_cast<uint2 *>(codes + static_cast<size_t>(r) * K);
    float amax = 0.f;
    if (nvec <= 32 * kRegVec) {  // one read of the row
      uint4 v[kRegVec];
#pragma unroll
      for (int j = 0; j < kRegVec; ++j) {
        const int c = lane + 32 * j;
        v[j] = c < nvec ? row[c] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < kRegVec; ++j) amax = vec_amax(v[j], amax);
      // amax >= 0: its bits order as unsigned integers
      amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
      const float scale = row_scale(amax, pow2);
      const float rcp = __frcp_rn(scale);
#pragma unroll
      for (int j = 0; j < kRegVec; ++j) {
        const int c = lane + 32 * j;
        if (c < nvec) out[c] = vec_codes(v[j], rcp);
      }
      if (lane == 0) scales[r] = scale;
    } else {  // longer rows: read twice
      for (int c = lane; c < nvec; c += 32) amax = vec_amax(row[c], amax);
      amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
      const float scale = row_scale(amax, pow2);
      const float rcp = __frcp_rn(scale);
      for (int c = lane; c < nvec; c += 32) out[c] = vec_codes(row[c], rcp);
      if (lane == 0) scales[r] = scale;
    }
  }
}

__global__ void __launch_bounds__(256)
    bf16_to_f16_kernel(const uint4 *__restrict__ src, size_t n_vec, uint4 *__restrict__ dst,
                       int *status) {
  bool over = false;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a = __uint_as_float(w[q] << 16);
      const float b = __uint_as_float(w[q] & 0xFFFF0000u);
      over |= fabsf(a) > 65504.f || fabsf(b) > 65504.f;
      __half2 h = __floats2half2_rn(a, b);
      o[q] = *reinterpret_cast<uint32_t *>(&h);
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (over) record_status(status, MOE_ERR_DEVICE_BOUNDS, SITE_WEIGHT_FP16_RANGE);
}

__global__ void selftest_wait_kernel(int *status, long long limit_cycles) {
  // The flag lives in this CTA's shared memory and nothing ever sets it.
  __shared__ volatile int flag;
  if (threadIdx.x == 0) flag = 0;
  __syncthreads();
  if (threadIdx.x != 0) return;
  const long long t0 = clock64();
  while (flag == 0) {
    if (clock64() - t0 > limit_cycles) {
      record_status(status, MOE_ERR_DEVICE_TIMEOUT, SITE_SELFTEST_FLAG);
      return;
    }
  }
}

int grid_for(size_t work, int threads) {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int sms = (dev >= 0 && dev < 64) ? cached[dev] : 0;
  if (sms == 0) {
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 0 && dev < 64) cached[dev] = sms;
  }
  const size_t want = (work + threads - 1) / threads;
  const size_t cap = static_cast<size_t>(sms) * 8;
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_gather_rows(const uint16_t *x, const int32_t *perm, const int32_t *n_valid,
                               int n_rows, int k, int d, uint16_t *x_perm, cudaStream_t s) {
  const int vpr = d / 8;
  const size_t work = static_cast<size_t>(n_rows) * vpr;
  gather_rows_kernel<<<grid_for(work, 256), 256, 0, s>>>(reinterpret_cast<const uint4 *>(x), perm,
                                                         n_valid, n_rows, k, vpr,
                                                         reinterpret_cast<uint4 *>(x_perm));
  return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t *o, const uint16_t *s_out, const int32_t *inv, int T,
                           int k, int d, uint16_t *y, cudaStream_t s) {
  const int vpr = d / 8;
  const size_t work = static_cast<size_t>(T) * kCombineThreads;  // one CTA per token
  const int grid = grid_for(work, kCombineThreads);
  const uint4 *o4 = reinterpret_cast<const uint4 *>(o);
  const uint4 *s4 = reinterpret_cast<const uint4 *>(s_out);
  uint4 *y4 = reinterpret_cast<uint4 *>(y);
  if (k <= 4)
    combine_kernel<4><<<grid, kCombineThreads, 0, s>>>(o4, s4, inv, T, k, vpr, y4);
  else if (k <= 8)
    combine_kernel<8><<<grid, kCombineThreads, 0, s>>>(o4, s4, inv, T, k, vpr, y4);
  else
    combine_kernel<16><<<grid, kCombineThreads, 0, s>>>(o4, s4, inv, T, k, vpr, y4);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const float *yacc, size_t n, uint16_t *y, cudaStream_t s) {
  const size_t n_vec8 = n / 8;
  finalize_kernel<<<grid_for(n_vec8, 256), 256, 0, s>>>(reinterpret_cast<const float4 *>(yacc),
                                                        n_vec8, reinterpret_cast<uint4 *>(y));
  return cudaGetLastError();
}

cudaError_t launch_bf16_to_f16(const uint16_t *src, size_t n, uint16_t *dst, int *status,
                               cudaStream_t s) {
  const size_t n_vec = n / 8;  // n is a multiple of 64 (d and F are)
  bf16_to_f16_kernel<<<grid_for(n_vec, 256), 256, 0, s>>>(reinterpret_cast<const uint4 *>(src),
                                                          n_vec, reinterpret_cast<uint4 *>(dst),
                                                          status);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(int *status, long long limit_cycles, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status, limit_cycles);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows_e4m3(const uint16_t *src, bool is_f16, bool pow2, int rows,
                                  const int32_t *n_valid, int K, uint8_t *codes, float *scales,
                                  cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const size_t threads = static_cast<size_t>(rows) * 32;
  quant_rows_e4m3_kernel<<<grid_for(threads, 256), 256, 0, s>>>(src, is_f16 ? 1 : 0, pow2 ? 1 : 0,
                                                               rows, n_valid, K, codes, scales);
  return cudaGetLastError();
}

}  // namespace moe
