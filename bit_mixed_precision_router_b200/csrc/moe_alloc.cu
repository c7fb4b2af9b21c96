// Budgeted per-expert bit allocation for bitplane experts (a Lagrangian
// rate-distortion choice per expert with a bisection to a routing-weighted read
// budget, after "DuoRate: Two-Rate Per-Expert Precision Allocation for
// Mixture-of-Experts Serving", key concepts "DuoRate Pipeline Stages" and "Routing
// Frequency Cancellation").
//   k_bitplane_distortion  offline: delta[e][b-1][k] = sum_n (s * (u'_b - u))^2 over the
//                          rows n of the gate/up matrix, fp64, rows in order;
//   k_act_moments          profiling: m[k] = mean_t x[t][k]^2, fp64, tokens in order;
//   k_allocate             one CTA: D[e][c] = m . delta[e][choice_c - 1] (one warp per
//                          dot product), f_e from the routing offsets, then a fixed
//                          number of bisection steps on the multiplier lam, each taking
//                          per expert argmin_c D[e][c] + lam * choice_c (ties to the larger
//                          width); "within the budget" is the exact integer sum_e n_e * b_e
//                          (n_e pairs routed to e) against the fp64 product budget * sum_e n_e;
//   k_expand_bits          bits[p] = bits_e[topk_ids[p]].
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kAllocThreads = 1024;
constexpr int kBisectSteps = 100;

__global__ void k_bitplane_distortion(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ scales,
                                      int E, int N, int K, double* __restrict__ delta) {
  const int64_t q = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (q >= int64_t(E) * K) return;
  const int e = int(q / K), k = int(q - int64_t(e) * K);
  const int KW = K / 32, KG = K / 128;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int n = 0; n < N; ++n) {
    int u = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p)
      u |= int((planes[((size_t(e) * 8 + p) * N + n) * KW + k / 32] >> (k % 32)) & 1u) << (7 - p);
    const double s = double(bf16_bits_to_float(scales[(size_t(e) * N + n) * KG + k / 128]));
#pragma unroll
    for (int b = 1; b <= 8; ++b) {
      const int ub = ((u >> (8 - b)) << (8 - b)) + (b < 8 ? (1 << (7 - b)) : 0);
      const double err = s * double(ub - u);
      acc[b - 1] += err * err;
    }
  }
#pragma unroll
  for (int b = 0; b < 8; ++b) delta[(size_t(e) * 8 + b) * K + k] = acc[b];
}

__global__ void k_act_moments(const uint16_t* __restrict__ x, int T, int H, double* __restrict__ m) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= H) return;
  double acc = 0.0;
  for (int t = 0; t < T; ++t) {
    const double v = double(bf16_bits_to_float(x[size_t(t) * H + k]));
    acc += v * v;
  }
  m[k] = acc / double(T);
}

struct Choices {
  int n;
  int v[8];
};

// Block sum of one integer per thread (exact), and block max of one double.
__device__ long long block_sum_i(long long v, long long* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < nw ? red[lane] : 0;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) w += __shfl_xor_sync(0xffffffffu, w, d);
    if (lane == 0) red[32] = w;
  }
  __syncthreads();
  return red[32];
}
__device__ double block_max(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, d));
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    double w = lane < nw ? red[lane] : 0.0;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) w = fmax(w, __shfl_xor_sync(0xffffffffu, w, d));
    if (lane == 0) red[32] = w;
  }
  __syncthreads();
  return red[32];
}

// index into ch of argmin_c D[c] + lam * ch[c], ties to the larger width
__device__ int choose_one(const double* D, const Choices& ch, double lam) {
  int bi = 0;
  double bc = D[0] + lam * double(ch.v[0]);
  for (int i = 1; i < ch.n; ++i) {
    const double c = D[i] + lam * double(ch.v[i]);
    if (c < bc || (c == bc && ch.v[i] > ch.v[bi])) {
      bi = i;
      bc = c;
    }
  }
  return bi;
}

__global__ void __launch_bounds__(kAllocThreads) k_allocate(const double* __restrict__ delta,
                                                            const double* __restrict__ m,
                                                            const int32_t* __restrict__ offsets, int E, int K,
                                                            Choices ch, double budget, uint8_t* __restrict__ bits_e,
                                                            double* lam_out) {
  extern __shared__ double smem_d[];
  double* D = smem_d;  // [E][8]
  __shared__ double red[33];
  __shared__ long long redi[33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  // one dot product per expert and candidate: lane partials over k = lane + 32 j, then a butterfly
  for (int q = warp; q < E * ch.n; q += nw) {
    const int e = q / ch.n, c = q - e * ch.n;
    const double* row = delta + (size_t(e) * 8 + (ch.v[c] - 1)) * K;
    double acc = 0.0;
    for (int k = lane; k < K; k += 32) acc = fma(m[k], row[k], acc);
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, d);
    if (lane == 0) D[size_t(e) * 8 + c] = acc;
  }
  __syncthreads();
  const double limit = budget * double(offsets[E] - offsets[0]);  // budget * sum_e n_e
  int i0 = 0;
  for (int i = 1; i < ch.n; ++i)
    if (ch.v[i] < ch.v[i0]) i0 = i;
  // within the budget at lam? (every thread takes part: the reduction synchronises the block)
  auto within = [&](double lam) -> bool {
    long long part = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      part += (long long)(offsets[e + 1] - offsets[e]) * ch.v[choose_one(D + size_t(e) * 8, ch, lam)];
    return double(block_sum_i(part, redi)) <= limit;
  };
  // upper multiplier: every expert at the smallest width
  double part = 0.0;
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    for (int i = 0; i < ch.n; ++i)
      if (ch.v[i] > ch.v[i0])
        part = fmax(part, (D[size_t(e) * 8 + i0] - D[size_t(e) * 8 + i]) / double(ch.v[i] - ch.v[i0]));
  double lo = 0.0, hi = 2.0 * block_max(part, red) + 1.0, lam;
  bool fixed_min = false;
  if (within(lo)) {
    lam = lo;
  } else if (!within(hi)) {
    lam = hi;
    fixed_min = true;
  } else {
    for (int s = 0; s < kBisectSteps; ++s) {
      const double mid = 0.5 * (lo + hi);
      if (within(mid)) hi = mid;
      else lo = mid;
    }
    lam = hi;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const bool unread = offsets[e + 1] == offsets[e];
    const int idx = (fixed_min || unread) ? i0 : choose_one(D + size_t(e) * 8, ch, lam);
    bits_e[e] = uint8_t(ch.v[idx]);
  }
  if (threadIdx.x == 0 && lam_out) *lam_out = lam;
}

__global__ void k_expand_bits(const int32_t* __restrict__ ids, const uint8_t* __restrict__ bits_e, int64_t n,
                              uint8_t* __restrict__ bits) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) bits[i] = bits_e[ids[i]];
}

}  // namespace

cudaError_t launch_bitplane_distortion(const uint32_t* planes, const uint16_t* scales, int E, int N, int K,
                                       double* delta, cudaStream_t st) {
  const int64_t n = int64_t(E) * K;
  k_bitplane_distortion<<<unsigned((n + 127) / 128), 128, 0, st>>>(planes, scales, E, N, K, delta);
  return cudaGetLastError();
}

cudaError_t launch_act_moments(const uint16_t* x, int T, int H, double* m, cudaStream_t st) {
  k_act_moments<<<unsigned((H + 255) / 256), 256, 0, st>>>(x, T, H, m);
  return cudaGetLastError();
}

cudaError_t launch_allocate_bits(const double* delta, const double* m, const int32_t* offsets, int E, int K,
                                 const uint8_t* choices, int nchoices, double budget, uint8_t* bits_e,
                                 double* lam_out, cudaStream_t st) {
  Choices ch{};
  ch.n = nchoices;
  for (int i = 0; i < nchoices; ++i) ch.v[i] = choices[i];
  const size_t smem = size_t(E) * 8 * sizeof(double);
  if (smem > 48 * 1024) {
    const cudaError_t err =
        cudaFuncSetAttribute(k_allocate, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
  }
  k_allocate<<<1, kAllocThreads, smem, st>>>(delta, m, offsets, E, K, ch, budget, bits_e, lam_out);
  return cudaGetLastError();
}

cudaError_t launch_expand_bits(const int32_t* ids, const uint8_t* bits_e, int64_t n, uint8_t* bits,
                               cudaStream_t st) {
  k_expand_bits<<<unsigned((n + 255) / 256), 256, 0, st>>>(ids, bits_e, n, bits);
  return cudaGetLastError();
}

}  // namespace moe
