// Device side of the seeded input generator (see moe_synth.h).  Integer and
// correctly rounded IEEE float64 operations only (explicit _rn intrinsics, so no
// multiply-add contraction), which the host generator reproduces bit for bit.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

__device__ __forceinline__ uint64_t splitmix_word(uint64_t seed, uint64_t j) {
  uint64_t z = seed + (j + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void k_synth_normal(uint16_t* __restrict__ out, int64_t n, uint64_t start, uint64_t seed,
                               double stddev) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const uint64_t idx = start + uint64_t(i);
  int64_t sum = 0;
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const uint64_t w = splitmix_word(seed, idx * 3ull + uint64_t(m));
#pragma unroll
    for (int q = 0; q < 4; ++q) sum += int64_t((w >> (16 * q)) & 0xFFFFull);
  }
  const double z = double(sum - 393210) / 65536.0;  // exact
  const float f = __double2float_rn(__dmul_rn(z, stddev));
  out[i] = float_to_bf16_bits(f);
}

__global__ void k_synth_uniform(uint16_t* __restrict__ out, int64_t n, uint64_t start, uint64_t seed, double lo,
                                double d) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const uint64_t w = splitmix_word(seed, start + uint64_t(i));
  const double u = double(w >> 11) * 0x1.0p-53;
  const float f = __double2float_rn(__dadd_rn(lo, __dmul_rn(d, u)));
  out[i] = float_to_bf16_bits(f);
}

cudaError_t launch_synth_normal(uint16_t* out, int64_t n, int64_t start, uint64_t seed, double stddev,
                                cudaStream_t st) {
  const int threads = 256;
  k_synth_normal<<<dim3(unsigned((n + threads - 1) / threads)), threads, 0, st>>>(out, n, uint64_t(start), seed,
                                                                                  stddev);
  return cudaGetLastError();
}

cudaError_t launch_synth_uniform(uint16_t* out, int64_t n, int64_t start, uint64_t seed, double lo, double hi,
                                 cudaStream_t st) {
  const int threads = 256;
  k_synth_uniform<<<dim3(unsigned((n + threads - 1) / threads)), threads, 0, st>>>(out, n, uint64_t(start), seed,
                                                                                   lo, hi - lo);
  return cudaGetLastError();
}

}  // namespace moe
