// Device filler for seeded synthetic tables (input generation only).
//
// Writes element (row, col) of a [rows x width] table as the value that
// synth/gen.py computes on the host for the same (seed, tag, row, col):
//   z      = SplitMix64 output number (row * width + col) of the stream whose
//            seed is output number `tag` of the stream seeded with `seed`
//   s      = sum of the four 16-bit lanes of z               (Irwin-Hall(4))
//   value  = float(s - 131070) * scale                       (one fp32 multiply)
//   stored = value as fp32, or its bf16 round-to-nearest-even bit pattern.
// SplitMix64 is from Steele, Lea and Flood, OOPSLA 2014.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t splitmix_at(uint64_t base, uint64_t i) {
  return mix64(base + (i + 1) * kGamma);
}

__device__ inline float ih4_value(uint64_t z, float scale) {
  const int s = int(z & 0xFFFF) + int((z >> 16) & 0xFFFF) + int((z >> 32) & 0xFFFF) + int(z >> 48);
  return float(s - 131070) * scale;
}

__device__ inline uint16_t f32_to_bf16_rne_bits(float f) {
  uint32_t b = __float_as_uint(f);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return uint16_t(b >> 16);
}

// Each thread writes 8 consecutive elements (one 16-byte store for bf16).
__global__ void fill_bf16(uint16_t* __restrict__ dst, uint64_t n, uint64_t base, float scale) {
  const uint64_t stride = uint64_t(gridDim.x) * blockDim.x * 8;
  for (uint64_t i = (uint64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < n; i += stride) {
    if (i + 8 <= n) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint16_t lo = f32_to_bf16_rne_bits(ih4_value(splitmix_at(base, i + 2 * j), scale));
        const uint16_t hi = f32_to_bf16_rne_bits(ih4_value(splitmix_at(base, i + 2 * j + 1), scale));
        w[j] = uint32_t(lo) | (uint32_t(hi) << 16);
      }
      *reinterpret_cast<uint4*>(dst + i) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      for (uint64_t k = i; k < n; ++k) dst[k] = f32_to_bf16_rne_bits(ih4_value(splitmix_at(base, k), scale));
    }
  }
}

__global__ void fill_f32(float* __restrict__ dst, uint64_t n, uint64_t base, float scale) {
  const uint64_t stride = uint64_t(gridDim.x) * blockDim.x;
  for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    dst[i] = ih4_value(splitmix_at(base, i), scale);
}

}  // namespace

extern "C" {

// Fill a dense row-major [rows x width] table. dtype: 0 = bf16, 1 = fp32.
// dst must be 16-byte aligned for bf16. Returns 0 or a cudaError_t value.
int synth_fill_table(void* dst, int64_t rows, int32_t width, uint64_t seed, int32_t tag,
                     float scale, int32_t dtype, void* stream) {
  if (!dst || rows < 0 || width <= 0) return int(cudaErrorInvalidValue);
  if (dtype == 0 && (reinterpret_cast<uintptr_t>(dst) & 15)) return int(cudaErrorMisalignedAddress);
  const uint64_t n = uint64_t(rows) * uint64_t(width);
  if (n == 0) return 0;
  const uint64_t base = splitmix_at(seed, uint64_t(tag));
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 256;
  const uint64_t per = dtype == 0 ? 8 : 1;
  uint64_t want = (n / per + threads - 1) / threads;
  const uint64_t cap = uint64_t(sms) * 32;
  const int blocks = int(want < cap ? (want ? want : 1) : cap);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == 0)
    fill_bf16<<<blocks, threads, 0, s>>>(static_cast<uint16_t*>(dst), n, base, scale);
  else if (dtype == 1)
    fill_f32<<<blocks, threads, 0, s>>>(static_cast<float*>(dst), n, base, scale);
  else
    return int(cudaErrorInvalidValue);
  return int(cudaGetLastError());
}

}  // extern "C"
