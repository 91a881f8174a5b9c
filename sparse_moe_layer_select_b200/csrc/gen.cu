// gen.cu -- CUDA implementation of the seeded input generator (built as its
// own library, libmoe_gen.so; it holds none of the layer's arithmetic).
//
// Same definition as the host implementation in inputs.py:
//   Philox4x32-10 (Salmon et al., SC'11), key = 64-bit seed, counter =
//   (block_lo, block_hi, tensor_id, 0) with block = element_index / 2;
//   element 2*block + h uses words (2h, 2h+1) as uniforms (w + 0.5) / 2^32;
//   z = sqrt(-2 ln u_a) * cos(2 pi u_b) in double; v = z * sigma (double);
//   v rounded once, to nearest even, to bfloat16.
#include <cuda_runtime.h>

#include <cstdint>

namespace {

__device__ __forceinline__ void philox4x32_10(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += W0;
      k1 += W1;
    }
    const uint64_t p0 = static_cast<uint64_t>(M0) * c[0];
    const uint64_t p1 = static_cast<uint64_t>(M1) * c[2];
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c[1] ^ k0;
    const uint32_t n1 = static_cast<uint32_t>(p1);
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c[3] ^ k1;
    const uint32_t n3 = static_cast<uint32_t>(p0);
    c[0] = n0;
    c[1] = n1;
    c[2] = n2;
    c[3] = n3;
  }
}

__device__ __forceinline__ uint16_t f64_to_bf16_rne(double v) {
  if (fabs(v) < 0x1p-126) {
    const uint32_t b = __float_as_uint(static_cast<float>(v));
    return static_cast<uint16_t>((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
  }
  const uint64_t bits = static_cast<uint64_t>(__double_as_longlong(v));
  const uint64_t lsb = (bits >> 45) & 1ull;
  const uint64_t r = (bits + 0x0FFFFFFFFFFFull + lsb) & ~0x1FFFFFFFFFFFull;
  const float f = static_cast<float>(__longlong_as_double(static_cast<long long>(r)));
  return static_cast<uint16_t>(__float_as_uint(f) >> 16);
}

__global__ void gen_normal_bf16_kernel(uint16_t *dst, int64_t n, uint64_t seed, uint32_t tid,
                                       double sigma, int64_t start) {
  const double inv = 1.0 / 4294967296.0;
  const double two_pi = 6.283185307179586;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint64_t e = static_cast<uint64_t>(start + i);
    const uint64_t blk = e >> 1;
    uint32_t c[4] = {static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), tid, 0u};
    philox4x32_10(c, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
    const int h = static_cast<int>(e & 1);
    const double ua = (static_cast<double>(c[2 * h]) + 0.5) * inv;
    const double ub = (static_cast<double>(c[2 * h + 1]) + 0.5) * inv;
    const double z = sqrt(-2.0 * log(ua)) * cos(two_pi * ub);
    dst[i] = f64_to_bf16_rne(z * sigma);
  }
}

}  // namespace

extern "C" int moe_gen_normal_bf16(void *dst, int64_t n, uint64_t seed, uint32_t tensor_id,
                                   double sigma, int64_t start, void *stream) {
  if (n <= 0) return 0;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + 255) / 256;
  const int grid = static_cast<int>(want < sms * 16 ? want : sms * 16);
  gen_normal_bf16_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint16_t *>(dst), n, seed, tensor_id, sigma, start);
  return static_cast<int>(cudaGetLastError());
}
