// Routing-weighted combine: out[t] = bf16( sum_j w[t][j] * y_rows[pair_to_row[t*k+j]] (+ residual[t]) ),
// fp32 accumulation in slot order j, residual added last.  One thread per 8
// consecutive hidden elements (16-byte loads and stores).
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

__global__ void k_combine(const uint16_t* __restrict__ y, const int32_t* __restrict__ p2r,
                          const float* __restrict__ w, const uint16_t* residual, int H, int k, uint16_t* out) {
  const int t = blockIdx.x;
  const int h = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (h >= H) return;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int j = 0; j < k; ++j) {
    const float wj = w[size_t(t) * k + j];
    const int row = p2r[size_t(t) * k + j];
    const uint4 v = *reinterpret_cast<const uint4*>(y + size_t(row) * H + h);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(wj, bf16_lo(u[i]), acc[2 * i]);
      acc[2 * i + 1] = fmaf(wj, bf16_hi(u[i]), acc[2 * i + 1]);
    }
  }
  if (residual) {
    const uint4 v = *reinterpret_cast<const uint4*>(residual + size_t(t) * H + h);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += bf16_lo(u[i]);
      acc[2 * i + 1] += bf16_hi(u[i]);
    }
  }
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    o[i] = uint32_t(float_to_bf16_bits(acc[2 * i])) | (uint32_t(float_to_bf16_bits(acc[2 * i + 1])) << 16);
  *reinterpret_cast<uint4*>(out + size_t(t) * H + h) = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t launch_combine(const uint16_t* y_rows, const moe_routing_t& r, const uint16_t* residual, int T,
                           int H, int k, uint16_t* out, cudaStream_t st) {
  const int threads = 256;
  const int per_block = threads * 8;
  dim3 grid(unsigned(T), unsigned((H + per_block - 1) / per_block));
  k_combine<<<grid, threads, 0, st>>>(y_rows, r.pair_to_row, r.topk_w, residual, H, k, out);
  return cudaGetLastError();
}

}  // namespace moe
