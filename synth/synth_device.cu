// synth_device.cu - CUDA implementation of the seeded input generator.
// The recipe is stated in synth.h; synth_host.c implements the same recipe
// on the CPU.  All steps are integer arithmetic up to one IEEE double
// multiply and one round-to-nearest-even conversion, so both sides agree
// bit for bit.
#include "synth.h"

#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;

__device__ __forceinline__ void draw(uint64_t seed, uint32_t tid, uint64_t i, uint32_t r[4]) {
  uint32_t c0 = (uint32_t)i, c1 = (uint32_t)(i >> 32), c2 = tid, c3 = SYNTH_CTR_TAG;
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t lo0 = kM0 * c0, hi0 = __umulhi(kM0, c0);
    const uint32_t lo1 = kM1 * c2, hi1 = __umulhi(kM1, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    k0 += kW0; k1 += kW1;
  }
  r[0] = c0; r[1] = c1; r[2] = c2; r[3] = c3;
}

__device__ __forceinline__ double centred_value(uint64_t seed, uint32_t tid, uint64_t i, double scale) {
  uint32_t r[4];
  draw(seed, tid, i, r);
  const long long s = (long long)r[0] + (long long)r[1] + (long long)r[2] + (long long)r[3];
  const long long c = s - 2ll * 0xFFFFFFFFll;
  return __dmul_rn((double)c, scale);
}

__device__ __forceinline__ uint16_t bf16_from_double(double x) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(x);
  const uint32_t sign = (uint32_t)(b >> 63);
  const unsigned long long mag = b & 0x7FFFFFFFFFFFFFFFull;
  if (mag == 0) return (uint16_t)(sign << 15);
  const int e = (int)(mag >> 52) - 1023;
  if (e < -126) return (uint16_t)(sign << 15);
  const unsigned long long mant = mag & ((1ull << 52) - 1);
  uint32_t v = ((uint32_t)(e + 127) << 7) | (uint32_t)(mant >> 45);
  const unsigned long long rem = mant & ((1ull << 45) - 1), half = 1ull << 44;
  if (rem > half || (rem == half && (v & 1u))) v += 1u;
  return (uint16_t)((sign << 15) | v);
}

__global__ void fill_bf16_kernel(uint16_t* dst, int64_t row0, int64_t rows, int64_t cols, int64_t sr,
                                 int64_t sc, uint64_t seed, uint32_t tid, double scale) {
  const int64_t n = rows * cols;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cols, c = i - r * cols;
    dst[r * sr + c * sc] =
        bf16_from_double(centred_value(seed, tid, (uint64_t)(i + row0 * cols), scale));
  }
}

__global__ void fill_f32_kernel(float* dst, int64_t n, uint64_t seed, uint32_t tid, double scale) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = __double2float_rn(centred_value(seed, tid, (uint64_t)i, scale));
}

__global__ void fill_tokens_kernel(int32_t* dst, int64_t n, uint64_t seed, uint32_t tid, uint32_t V) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint32_t r[4];
    draw(seed, tid, (uint64_t)i, r);
    dst[i] = (int32_t)(((unsigned long long)r[0] * V) >> 32);
  }
}

double value_scale(double std) { return std * 0x1.bb67ae8584caap+0 * 0x1p-32; }

unsigned grid_for(int64_t n) {
  const int64_t blocks = (n + 255) / 256;
  return (unsigned)(blocks < 148 * 64 ? (blocks > 0 ? blocks : 1) : 148 * 64);
}

}  // namespace

extern "C" int synth_fill_bf16_device(uint16_t* dst, int64_t row0, int64_t rows, int64_t cols,
                                      int64_t stride_r, int64_t stride_c, uint64_t seed,
                                      uint32_t tid, double std, void* stream) {
  if (!dst || row0 < 0 || rows < 0 || cols <= 0) return (int)cudaErrorInvalidValue;
  if (rows == 0) return 0;
  fill_bf16_kernel<<<grid_for(rows * cols), 256, 0, (cudaStream_t)stream>>>(
      dst, row0, rows, cols, stride_r, stride_c, seed, tid, value_scale(std));
  return (int)cudaGetLastError();
}

extern "C" int synth_fill_f32_device(float* dst, int64_t n, uint64_t seed, uint32_t tid, double std,
                                     void* stream) {
  if (!dst || n < 0) return (int)cudaErrorInvalidValue;
  if (n == 0) return 0;
  fill_f32_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(dst, n, seed, tid, value_scale(std));
  return (int)cudaGetLastError();
}

extern "C" int synth_fill_tokens_device(int32_t* dst, int64_t n, uint64_t seed, uint32_t tid,
                                        int32_t V, void* stream) {
  if (!dst || n < 0 || V <= 0) return (int)cudaErrorInvalidValue;
  if (n == 0) return 0;
  fill_tokens_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(dst, n, seed, tid, (uint32_t)V);
  return (int)cudaGetLastError();
}
