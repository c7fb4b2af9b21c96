// Offline weight preparation: INT4 g128, 8-bitplane and NVFP4 quantisers.
//
// Each integer decision is taken with IEEE fp32 round-to-nearest-even division
// (__fdiv_rn) and rintf, so the packed bytes equal a plain CPU evaluation of the
// same formulas bit for bit.  Layouts are documented in moe.h.
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// Loads 8 consecutive bf16 (16 bytes) as floats.
MOE_DEVICE void load8(const uint16_t* p, float (&f)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_lo(u[i]);
    f[2 * i + 1] = bf16_hi(u[i]);
  }
}

// Per-group symmetric scale for a group spread over 16 consecutive lanes that
// hold 8 elements each: bf16(max|w| / qmax); returns the fp32 value of the bf16
// scale and writes its bits to *sbits.
MOE_DEVICE float group_scale16(const float (&f)[8], float qmax, uint16_t* sbits) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const uint16_t sb = float_to_bf16_bits(__fdiv_rn(amax, qmax));
  *sbits = sb;
  return bf16_bits_to_float(sb);
}

// One thread per 8 elements (one output word); a group of 128 is 16 lanes.
__global__ void k_quant_w4g128(const uint16_t* __restrict__ w, int64_t nwords, uint32_t* __restrict__ packed,
                               uint16_t* __restrict__ scales) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  const bool valid = i < nwords;  // nwords % 16 == 0: a group is all-valid or all-invalid
  float f[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (valid) load8(w + i * 8, f);
  uint16_t sbits;
  const float s = group_scale16(f, 7.0f, &sbits);
  uint32_t word = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float q = (s == 0.f) ? 0.f : rintf(__fdiv_rn(f[j], s));
    q = fminf(fmaxf(q, -8.f), 7.f);
    word |= uint32_t(int(q) + 8) << (4 * j);
  }
  if (valid) {
    packed[i] = word;
    if ((i & 15) == 0) scales[i >> 4] = sbits;
  }
}

// One thread per 8 elements; 4 consecutive lanes form one 32-element plane word.
__global__ void k_pack_bitplanes(const uint16_t* __restrict__ w, int64_t nchunks, int64_t N, int64_t K,
                                 uint32_t* __restrict__ planes, uint16_t* __restrict__ scales) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  const bool valid = i < nchunks;
  float f[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (valid) load8(w + i * 8, f);
  uint16_t sbits;
  const float s = group_scale16(f, 127.0f, &sbits);
  uint32_t u[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float q = (s == 0.f) ? 0.f : rintf(__fdiv_rn(f[j], s));
    q = fminf(fmaxf(q, -127.f), 127.f);
    u[j] = uint32_t(int(q) + 128);
  }
  const int sub = int(i & 3);  // which 8-bit slice of the 32-bit plane word
  uint32_t word[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) m |= ((u[j] >> (7 - p)) & 1u) << j;
    m <<= 8 * sub;
    m |= __shfl_xor_sync(0xffffffffu, m, 1);
    m |= __shfl_xor_sync(0xffffffffu, m, 2);
    word[p] = m;
  }
  if (!valid) return;
  const int64_t elem = i * 8;
  const int64_t row = elem / K;  // over E*N
  const int64_t kk = elem % K;
  const int64_t e = row / N, n = row % N;
  const int64_t kw = K / 32;
  // lane sub writes planes 2*sub and 2*sub+1
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int p = 2 * sub + q;
    planes[((e * 8 + p) * N + n) * kw + kk / 32] = word[p];
  }
  if ((i & 15) == 0) scales[i >> 4] = sbits;
}

// ---------------------------------------------------------------- NVFP4
// Eight consecutive elements as fp32: bf16 weights or activations, or fp32 activations.
MOE_DEVICE void load8(const float* p, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}

// amax of each expert matrix (or activation tensor), accumulated as fp32 bits (non-negative
// floats order like their bit patterns) into gscale[e], which the caller zeroed.
template <typename In>
__global__ void k_nvfp4_amax(const In* __restrict__ w, int64_t per_expert, float* __restrict__ gscale) {
  const int e = blockIdx.y;
  const In* base = w + int64_t(e) * per_expert;
  float amax = 0.f;
  for (int64_t c = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) * 8; c < per_expert;
       c += int64_t(gridDim.x) * blockDim.x * 8) {
    float f[8];
    load8(base + c, f);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned*>(gscale + e), __float_as_uint(amax));
}

MOE_DEVICE float e4m3_to_float(uint8_t c) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(c, __NV_E4M3);
  return __half2float(__half(h));
}

// One thread per block of 16 elements.  gscale holds amax here (see k_nvfp4_amax).
template <typename In>
__global__ void k_quant_nvfp4(const In* __restrict__ w, int64_t nblocks, int64_t blocks_per_expert,
                              const float* __restrict__ amax_e, uint8_t* __restrict__ codes,
                              uint8_t* __restrict__ block_scales) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= nblocks) return;
  const int64_t e = i / blocks_per_expert;
  const float g = __fdiv_rn(amax_e[e], 2688.0f);  // 6 * 448
  float f[16];
  float fa[8], fb[8];
  load8(w + i * 16, fa);
  load8(w + i * 16 + 8, fb);
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    f[j] = fa[j];
    f[8 + j] = fb[j];
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(f[j]));
  uint8_t sb = 0;
  const float denom = __fmul_rn(6.0f, g);
  if (denom != 0.f) sb = __nv_cvt_float_to_fp8(__fdiv_rn(amax, denom), __NV_SATFINITE, __NV_E4M3);
  const float prod = __fmul_rn(e4m3_to_float(sb), g);
  uint32_t lo = 0, hi = 0;
  if (prod != 0.f) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint32_t c = uint32_t(__nv_cvt_float_to_fp4(__fdiv_rn(f[j], prod), __NV_E2M1, cudaRoundNearest)) & 0xFu;
      if ((c & 7u) == 0) c = 0;  // one encoding of zero: +0
      if (j < 8)
        lo |= c << (4 * j);
      else
        hi |= c << (4 * (j - 8));
    }
  }
  *reinterpret_cast<uint2*>(codes + i * 8) = make_uint2(lo, hi);
  block_scales[i] = sb;
}

__global__ void k_nvfp4_finalize(float* __restrict__ gscale, int E) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) gscale[e] = __fdiv_rn(gscale[e], 2688.0f);
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_quantize_w4g128(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint32_t* packed,
                                   uint16_t* scales, cudaStream_t st) {
  const int64_t nwords = E * N * K / 8;
  const int threads = 256;
  const int64_t blocks = (nwords + threads - 1) / threads;
  k_quant_w4g128<<<dim3(unsigned(blocks)), threads, 0, st>>>(w, nwords, packed, scales);
  return cudaGetLastError();
}

cudaError_t launch_pack_bitplanes(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint32_t* planes,
                                  uint16_t* scales, cudaStream_t st) {
  const int64_t nchunks = E * N * K / 8;
  const int threads = 256;
  const int64_t blocks = (nchunks + threads - 1) / threads;
  k_pack_bitplanes<<<dim3(unsigned(blocks)), threads, 0, st>>>(w, nchunks, N, K, planes, scales);
  return cudaGetLastError();
}

cudaError_t launch_quantize_nvfp4(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint8_t* codes,
                                  uint8_t* block_scales, float* gscale, cudaStream_t st) {
  cudaError_t err = cudaMemsetAsync(gscale, 0, size_t(E) * sizeof(float), st);
  if (err != cudaSuccess) return err;
  const int64_t per_expert = N * K;
  const int threads = 256;
  int64_t bx = (per_expert / 8 + threads - 1) / threads;
  if (bx > 1024) bx = 1024;
  k_nvfp4_amax<uint16_t><<<dim3(unsigned(bx), unsigned(E)), threads, 0, st>>>(w, per_expert, gscale);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int64_t nblocks = E * N * K / 16;
  k_quant_nvfp4<uint16_t><<<dim3(unsigned((nblocks + threads - 1) / threads)), threads, 0, st>>>(
      w, nblocks, N * K / 16, gscale, codes, block_scales);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  k_nvfp4_finalize<<<dim3(unsigned((E + 255) / 256)), 256, 0, st>>>(gscale, int(E));
  return cudaGetLastError();
}

// Activations in NVFP4 for the W4A4 prefill path (the weights' recipe with the whole
// tensor as one scale unit): amax of `a` into *amax (zeroed here), then codes and block
// scales; *amax keeps the amax (the scale g = amax / 2688 is taken where it is used).
template <typename In>
cudaError_t launch_act_nvfp4(const In* a, int64_t n, uint8_t* codes, uint8_t* block_scales, float* amax,
                             cudaStream_t st) {
  cudaError_t err = cudaMemsetAsync(amax, 0, sizeof(float), st);
  if (err != cudaSuccess) return err;
  const int threads = 256;
  int64_t bx = (n / 8 + threads - 1) / threads;
  if (bx > 2048) bx = 2048;
  if (bx < 1) bx = 1;
  k_nvfp4_amax<In><<<dim3(unsigned(bx), 1u), threads, 0, st>>>(a, n, amax);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int64_t nblocks = n / 16;
  k_quant_nvfp4<In><<<dim3(unsigned((nblocks + threads - 1) / threads)), threads, 0, st>>>(a, nblocks, nblocks, amax,
                                                                                           codes, block_scales);
  return cudaGetLastError();
}
template cudaError_t launch_act_nvfp4<uint16_t>(const uint16_t*, int64_t, uint8_t*, uint8_t*, float*, cudaStream_t);
template cudaError_t launch_act_nvfp4<float>(const float*, int64_t, uint8_t*, uint8_t*, float*, cudaStream_t);

// The codes and block scales only, for a tensor whose amax is already in *amax.
template <typename In>
cudaError_t launch_act_nvfp4_codes(const In* a, int64_t n, uint8_t* codes, uint8_t* block_scales, const float* amax,
                                   cudaStream_t st) {
  const int threads = 256;
  const int64_t nblocks = n / 16;
  k_quant_nvfp4<In><<<dim3(unsigned((nblocks + threads - 1) / threads)), threads, 0, st>>>(a, nblocks, nblocks, amax,
                                                                                           codes, block_scales);
  return cudaGetLastError();
}
template cudaError_t launch_act_nvfp4_codes<float>(const float*, int64_t, uint8_t*, uint8_t*, const float*,
                                                   cudaStream_t);

cudaError_t launch_quantize_nvfp4_f32(const float* a, int64_t n, uint8_t* codes, uint8_t* block_scales,
                                      float* gscale, cudaStream_t st) {
  const cudaError_t err = launch_act_nvfp4<float>(a, n, codes, block_scales, gscale, st);
  if (err != cudaSuccess) return err;
  k_nvfp4_finalize<<<1, 32, 0, st>>>(gscale, 1);
  return cudaGetLastError();
}

}  // namespace moe
