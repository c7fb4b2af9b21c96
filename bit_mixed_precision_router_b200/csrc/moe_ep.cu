// Expert parallelism, the device side of the exchange: rows gathered by an index list
// (into send order, and back into arrival order), and each received row's local expert
// from the per-(source, local expert) counts.  After "Every Expert Counts: ExactMoE for
// Memory-Efficient W4A16 Inference", abstract (every selected expert executed, wherever
// it is placed); the exchange order is: senders in sorted-row order, owners in
// source-rank order, rows of one source grouped by local expert.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

// dst[i] = src[idx[i] / div] (rows of H bf16), one warp per row, 16-byte vectors
__global__ void k_gather_rows_by(const uint4* __restrict__ src, const int32_t* __restrict__ idx, int n, int div,
                                 int h16, uint4* __restrict__ dst) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int i = w; i < n; i += nw) {
    const size_t srow = size_t(idx[i] / div);
    for (int c = lane; c < h16; c += 32) dst[size_t(i) * h16 + c] = src[srow * h16 + c];
  }
}

// counts [S][El] (row-major); ids[r] = j for the rows r of source s and local expert j,
// rows ordered by s then j.  One CTA: an exclusive scan of the S*El counts, then each
// (s, j) fills its range.
__global__ void __launch_bounds__(1024) k_ids_from_counts(const int32_t* __restrict__ counts, int S, int El,
                                                          int32_t* __restrict__ ids) {
  __shared__ int part[1024];
  const int n = S * El;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b = threadIdx.x * per, e = min(n, b + per);
  int sum = 0;
  for (int i = b; i < e; ++i) sum += counts[i];
  part[threadIdx.x] = sum;
  __syncthreads();
  // inclusive scan over the 1024 partial sums (Hillis-Steele in shared memory)
  for (int d = 1; d < int(blockDim.x); d <<= 1) {
    const int v = threadIdx.x >= unsigned(d) ? part[threadIdx.x - d] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int run = part[threadIdx.x] - sum;
  for (int i = b; i < e; ++i) {
    const int j = i % El;
    for (int r = 0; r < counts[i]; ++r) ids[run + r] = j;
    run += counts[i];
  }
}

}  // namespace

cudaError_t launch_gather_rows_by(const uint16_t* src, const int32_t* idx, int n, int div, int H, uint16_t* dst,
                                  cudaStream_t st) {
  const int threads = 256;
  int64_t blocks = (int64_t(n) * 32 + threads - 1) / threads;
  blocks = blocks < 1 ? 1 : (blocks > 4096 ? 4096 : blocks);
  k_gather_rows_by<<<unsigned(blocks), threads, 0, st>>>(reinterpret_cast<const uint4*>(src), idx, n, div, H / 8,
                                               reinterpret_cast<uint4*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_ids_from_counts(const int32_t* counts, int S, int El, int32_t* ids, cudaStream_t st) {
  k_ids_from_counts<<<1, 1024, 0, st>>>(counts, S, El, ids);
  return cudaGetLastError();
}

}  // namespace moe
