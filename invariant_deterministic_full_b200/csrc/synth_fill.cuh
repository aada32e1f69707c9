// Device implementation of the synthetic-input generator (not the method):
// SplitMix64 counters (Steele, Lea, Flood, OOPSLA 2014), Irwin-Hall sum of
// twelve 16-bit uniforms for an approximately normal deviate, bf16(f32(z*std)).
// Integer arithmetic plus one IEEE division and two IEEE roundings, so it is
// bit-identical to any IEEE host implementation of the same definition.
#pragma once
#include "common.cuh"
#include "norm_rope.cuh"

namespace bi {

__device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__global__ void synth_fill_kernel(uint16_t* __restrict__ dst, int64_t rows, int64_t cols, uint64_t key, double std,
                                  int interleave, int phase) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = rows * cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    int64_t s = 0;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const uint64_t d = sm64_mix(key + ((uint64_t)(3 * i + j) + 1) * 0x9E3779B97F4A7C15ULL);
      s += (int64_t)(d & 0xFFFF) + (int64_t)((d >> 16) & 0xFFFF) + (int64_t)((d >> 32) & 0xFFFF) + (int64_t)(d >> 48);
    }
    const double z = __ddiv_rn((double)(s - 393210), 65535.99999237060546875);
    const float f = __double2float_rn(__dmul_rn(z, std));
    const int64_t r = i / cols, c = i % cols;
    int64_t dr = r;
    if (interleave > 0) dr = (r / interleave) * 2 * interleave + (int64_t)phase * interleave + r % interleave;
    if (interleave < 0) {  // paired RoPE row order of heads of size -interleave
      const int hd = -interleave;
      dr = (r / hd) * hd + paired_row((int)(r % hd), hd);
    }
    dst[dr * cols + c] = f32_to_bf16_bits(f);
  }
}

}  // namespace bi
