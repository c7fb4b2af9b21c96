// Host-side launchers behind the C ABI (moe_api.cu).  Arguments are validated by
// the caller; each launcher only enqueues kernels and returns cudaGetLastError().
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

cudaError_t launch_quantize_w4g128(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint32_t* packed,
                                   uint16_t* scales, cudaStream_t st);
cudaError_t launch_pack_bitplanes(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint32_t* planes,
                                  uint16_t* scales, cudaStream_t st);
cudaError_t launch_quantize_nvfp4(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint8_t* codes,
                                  uint8_t* block_scales, float* gscale, cudaStream_t st);

// Routing: logits into `logits` (fp32 [T][E]), then top-k and the permutation.  The
// single-launch router elects its last CTA with `counter` (a 32-bit word that must be 0
// before the launch; the launch leaves it 0).  A workspace holds the counter in its
// first kRouteCounterBytes and the logits after it.
constexpr size_t kRouteCounterBytes = 256;
size_t route_workspace_bytes(int64_t T, int64_t E, int64_t k);
cudaError_t route_prepare_device();  // per-device kernel attributes; idempotent
cudaError_t launch_route(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H, int E, int k,
                         const moe_routing_t& out, float* logits, unsigned* counter, cudaStream_t st);
cudaError_t launch_route_ws(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H, int E, int k,
                            const moe_routing_t& out, void* ws, cudaStream_t st);
cudaError_t launch_select_bits(const float* w, int64_t n, const float thr[3], const uint8_t ch[4],
                               uint8_t* bits, cudaStream_t st);

// Grouped FFN.
bool ffn_shape_supported(int64_t H, int64_t I, moe_format_t fmt);
size_t ffn_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, moe_format_t fmt);
cudaError_t launch_grouped_ffn(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex,
                               const uint8_t* bits, int T, int H, int I, int E, int k, uint16_t* y_rows,
                               void* ws, cudaStream_t st);

// Tensor-core (tcgen05) grouped GEMM path, used by launch_grouped_ffn when the
// experts see enough rows on average (use_umma_path); W4 group-128 weights.
bool use_umma_path(int64_t T, int64_t E, int64_t k, moe_format_t fmt);
size_t umma_h_bytes(int64_t T, int64_t I, int64_t k);
size_t umma_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t k);
// the weight-streaming pass over the experts with at most max_rows routed rows (GEMM batches)
cudaError_t launch_gemv_small(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex, int T, int H, int I,
                              int E, int k, void* hbuf, uint16_t* y_rows, bool down, int max_rows, cudaStream_t st);
cudaError_t launch_grouped_ffn_umma(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex, int T,
                                    int H, int I, int E, int k, uint16_t* y_rows, void* hbuf, cudaStream_t st);

// NVFP4 activations (moe_quant.cu): amax of the tensor into *amax (zeroed first), codes
// and E4M3 block scales; the _codes form takes an amax already computed.  n % 16 == 0.
template <typename In>
cudaError_t launch_act_nvfp4(const In* a, int64_t n, uint8_t* codes, uint8_t* block_scales, float* amax,
                             cudaStream_t st);
template <typename In>
cudaError_t launch_act_nvfp4_codes(const In* a, int64_t n, uint8_t* codes, uint8_t* block_scales, const float* amax,
                                   cudaStream_t st);
cudaError_t launch_quantize_nvfp4_f32(const float* a, int64_t n, uint8_t* codes, uint8_t* block_scales,
                                      float* gscale, cudaStream_t st);

// W4A4 prefill (moe_ffn_umma.cu): NVFP4 weights and NVFP4 activations on the block-scaled
// FP4 tensor cores; the weight scales first laid out once in the tensor-memory copy order.
size_t w4a4_scale_tiles_bytes(int64_t H, int64_t I, int64_t E);
cudaError_t launch_w4a4_prepare(const moe_experts_t& ex, int H, int I, int E, uint8_t* tiles, cudaStream_t st);
size_t w4a4_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k);
cudaError_t launch_grouped_ffn_w4a4(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex,
                                    const uint8_t* tiles, int T, int H, int I, int E, int k, uint16_t* y_rows,
                                    void* ws, cudaStream_t st);

// Budgeted per-expert bit allocation (moe_alloc.cu).
cudaError_t launch_bitplane_distortion(const uint32_t* planes, const uint16_t* scales, int E, int N, int K,
                                       double* delta, cudaStream_t st);
cudaError_t launch_act_moments(const uint16_t* x, int T, int H, double* m, cudaStream_t st);
cudaError_t launch_allocate_bits(const double* delta, const double* m, const int32_t* offsets, int E, int K,
                                 const uint8_t* choices, int nchoices, double budget, uint8_t* bits_e,
                                 double* lam_out, cudaStream_t st);
cudaError_t launch_expand_bits(const int32_t* ids, const uint8_t* bits_e, int64_t n, uint8_t* bits,
                               cudaStream_t st);

// Slot cache on the device (moe_cache.cu) and the permutation alone (moe_route.cu).
cudaError_t launch_permute(const int32_t* ids, int P, int E, const moe_routing_t& out, cudaStream_t st);
cudaError_t launch_cache_step(void* state, const moe_routing_t& r, const uint8_t* bits, int P, int32_t* slot_ids,
                              const moe_cache_plan_t& plan, cudaStream_t st);
cudaError_t launch_cache_fetch(const moe_cache_plan_t& plan, int E, const moe_experts_t& host,
                               const moe_experts_t& slots, int H, int I, cudaStream_t st);

// Expert parallelism, device side of the exchange (moe_ep.cu).
cudaError_t launch_gather_rows_by(const uint16_t* src, const int32_t* idx, int n, int div, int H, uint16_t* dst,
                                  cudaStream_t st);
cudaError_t launch_ids_from_counts(const int32_t* counts, int S, int El, int32_t* ids, cudaStream_t st);

cudaError_t launch_combine(const uint16_t* y_rows, const moe_routing_t& r, const uint16_t* residual, int T,
                           int H, int k, uint16_t* out, cudaStream_t st);

cudaError_t launch_synth_normal(uint16_t* out, int64_t n, int64_t start, uint64_t seed, double stddev,
                                cudaStream_t st);
cudaError_t launch_synth_uniform(uint16_t* out, int64_t n, int64_t start, uint64_t seed, double lo, double hi,
                                 cudaStream_t st);

}  // namespace moe
