// The C ABI (moe.h, moe_synth.h): host-side argument validation, then dispatch to
// the launchers.  Nothing here allocates device memory or synchronises, except
// moe_check_device_errors.
#include <atomic>
#include <stdint.h>

#include <climits>

#include "moe_cache_core.cuh"
#include "moe_common.cuh"
#include "moe_internal.h"
#include "moe_synth.h"

// The device error word (one per device, bit kErrWaitTimeout set by a kernel
// whose bounded wait ran out).
__device__ unsigned g_moe_error_word;

namespace moe {

unsigned* device_error_word() {
  // per-device lookup cached on first use (host threads may race to store the same value)
  static std::atomic<unsigned*> cached[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  unsigned* w = cached[dev].load(std::memory_order_relaxed);
  if (!w) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moe_error_word) != cudaSuccess) return nullptr;
    w = static_cast<unsigned*>(p);
    cached[dev].store(w, std::memory_order_relaxed);
  }
  return w;
}

}  // namespace moe

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

cudaStream_t as_stream(moe_stream_t s) { return static_cast<cudaStream_t>(s); }

moe_status_t check_quant_args(const void* w, int64_t E, int64_t N, int64_t K, const void* o1, const void* o2,
                              int64_t kmult) {
  if (!w || !o1 || !o2) return MOE_ERR_INVALID_ARG;
  if (E < 1 || N < 1 || K < 1) return MOE_ERR_INVALID_ARG;
  if (K % kmult != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (E > INT_MAX || N > INT_MAX || E * N > (int64_t(1) << 40) / K) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(w) || !aligned16(o1) || !aligned16(o2)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

moe_status_t check_routing(const moe_routing_t* r) {
  if (!r) return MOE_ERR_INVALID_ARG;
  const void* ps[] = {r->topk_ids, r->topk_w, r->expert_offsets, r->sorted_pair, r->pair_to_row, r->expert_list};
  for (const void* p : ps)
    if (!p) return MOE_ERR_INVALID_ARG;
  for (const void* p : ps)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

moe_status_t check_route_shape(int64_t T, int64_t E, int64_t k) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (k < 1 || k > E || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T > INT_MAX / k) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case MOE_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
  }
  return "unknown status";
}

int moe_abi_version(void) { return MOE_ABI_VERSION; }

moe_status_t moe_quantize_w4g128(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint32_t* packed,
                                 uint16_t* scales, moe_stream_t stream) {
  moe_status_t s = check_quant_args(w, E, N, K, packed, scales, 128);
  if (s != MOE_OK) return s;
  return from_cuda(moe::launch_quantize_w4g128(w, E, N, K, packed, scales, as_stream(stream)));
}

moe_status_t moe_pack_bitplanes(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint32_t* planes,
                                uint16_t* scales, moe_stream_t stream) {
  moe_status_t s = check_quant_args(w, E, N, K, planes, scales, 128);
  if (s != MOE_OK) return s;
  return from_cuda(moe::launch_pack_bitplanes(w, E, N, K, planes, scales, as_stream(stream)));
}

moe_status_t moe_quantize_nvfp4(const uint16_t* w, int64_t E, int64_t N, int64_t K, uint8_t* codes,
                                uint8_t* block_scales, float* gscale, moe_stream_t stream) {
  moe_status_t s = check_quant_args(w, E, N, K, codes, block_scales, 32);
  if (s != MOE_OK) return s;
  if (!gscale) return MOE_ERR_INVALID_ARG;
  if (!aligned16(gscale)) return MOE_ERR_MISALIGNED;
  if (E > 65535) return MOE_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(moe::launch_quantize_nvfp4(w, E, N, K, codes, block_scales, gscale, as_stream(stream)));
}

moe_status_t moe_quantize_nvfp4_f32(const float* a, int64_t R, int64_t C, uint8_t* codes, uint8_t* block_scales,
                                    float* gscale, moe_stream_t stream) {
  if (!a || !codes || !block_scales || !gscale) return MOE_ERR_INVALID_ARG;
  if (R < 1 || C < 1) return MOE_ERR_INVALID_ARG;
  if (C % 16 != 0 || R > (int64_t(1) << 40) / C) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(a) || !aligned16(codes) || !aligned16(block_scales) || !aligned16(gscale)) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_quantize_nvfp4_f32(a, R * C, codes, block_scales, gscale, as_stream(stream)));
}

size_t moe_route_workspace_bytes(int64_t T, int64_t E, int64_t k) {
  if (T < 0 || E < 1 || k < 1) return 0;
  return moe::route_workspace_bytes(T, E, k);
}

moe_status_t moe_route_topk(const uint16_t* x, const uint16_t* w_router, const float* bias, int64_t T, int64_t H,
                            int64_t E, int64_t k, const moe_routing_t* out, void* workspace,
                            size_t workspace_bytes, moe_stream_t stream) {
  moe_status_t s = check_route_shape(T, E, k);
  if (s != MOE_OK) return s;
  if (H < 256 || H % 256 != 0 || H > INT_MAX / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;  // nothing to route; no pointer is read
  if (!x || !w_router) return MOE_ERR_INVALID_ARG;
  if ((s = check_routing(out)) != MOE_OK) return s;
  if (!aligned16(x) || !aligned16(w_router) || (bias && !aligned16(bias))) return MOE_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < moe::route_workspace_bytes(T, E, k)) return MOE_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_route_ws(x, w_router, bias, int(T), int(H), int(E), int(k), *out, workspace,
                                     as_stream(stream)));
}

moe_status_t moe_bitplane_distortion(const uint32_t* planes, const uint16_t* scales, int64_t E, int64_t N,
                                     int64_t K, double* delta, moe_stream_t stream) {
  if (!planes || !scales || !delta) return MOE_ERR_INVALID_ARG;
  if (E < 1 || N < 1 || K < 1) return MOE_ERR_INVALID_ARG;
  if (K % 128 != 0 || E > INT_MAX || N > INT_MAX || K > INT_MAX || E * K > INT_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(planes) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(delta) & 7u)) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_bitplane_distortion(planes, scales, int(E), int(N), int(K), delta, as_stream(stream)));
}

moe_status_t moe_activation_moments(const uint16_t* x, int64_t T, int64_t H, double* m, moe_stream_t stream) {
  if (!x || !m) return MOE_ERR_INVALID_ARG;
  if (T < 1 || H < 1) return MOE_ERR_INVALID_ARG;
  if (T > INT_MAX || H > INT_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(x) & 1u) || (reinterpret_cast<uintptr_t>(m) & 7u)) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_act_moments(x, int(T), int(H), m, as_stream(stream)));
}

moe_status_t moe_allocate_bits(const double* delta, const double* m, const int32_t* expert_offsets, int64_t E,
                               int64_t K, const uint8_t* choices, int64_t nchoices, double budget,
                               uint8_t* bits_e, double* lambda, moe_stream_t stream) {
  if (!delta || !m || !expert_offsets || !choices || !bits_e) return MOE_ERR_INVALID_ARG;
  if (nchoices < 1 || nchoices > 8 || !(budget >= 0.0) || budget > 1e300) return MOE_ERR_INVALID_ARG;
  for (int64_t i = 0; i < nchoices; ++i) {
    if (choices[i] < 1 || choices[i] > 8) return MOE_ERR_INVALID_ARG;
    for (int64_t j = 0; j < i; ++j)
      if (choices[j] == choices[i]) return MOE_ERR_INVALID_ARG;
  }
  if (E < 1 || E > MOE_MAX_EXPERTS || K < 1 || K > INT_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(delta) & 7u) || (reinterpret_cast<uintptr_t>(m) & 7u) ||
      (reinterpret_cast<uintptr_t>(expert_offsets) & 3u) || (lambda && (reinterpret_cast<uintptr_t>(lambda) & 7u)))
    return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_allocate_bits(delta, m, expert_offsets, int(E), int(K), choices, int(nchoices),
                                             budget, bits_e, lambda, as_stream(stream)));
}

moe_status_t moe_expand_bits(const int32_t* topk_ids, const uint8_t* bits_e, int64_t T, int64_t k,
                             uint8_t* bits, moe_stream_t stream) {
  if (T < 0 || k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!topk_ids || !bits_e || !bits) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(topk_ids) & 3u) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_expand_bits(topk_ids, bits_e, T * k, bits, as_stream(stream)));
}

size_t moe_cache_state_bytes(int64_t E, int64_t S) {
  if (E < 1 || E > MOE_MAX_EXPERTS || S < 1 || S > E) return 0;
  return moe::cache_state_bytes(int(E), int(S));
}

moe_status_t moe_cache_init(void* state, size_t state_bytes, int64_t E, int64_t S, int64_t planes) {
  if (!state) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > MOE_MAX_EXPERTS || S < 1 || S > E || planes < 1 || planes > 8) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(state) & 7u) return MOE_ERR_MISALIGNED;
  if (state_bytes < moe::cache_state_bytes(int(E), int(S))) return MOE_ERR_WORKSPACE;
  moe::cache_reset(moe::cache_view(state, int(E), int(S)), int(E), int(S), int(planes));
  return MOE_OK;
}

static moe_status_t cache_header(const void* state, const moe::CacheHeader** h) {
  if (!state) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(state) & 7u) return MOE_ERR_MISALIGNED;
  *h = static_cast<const moe::CacheHeader*>(state);
  if ((*h)->magic != moe::kCacheMagic) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status_t moe_cache_plan(void* state, const uint8_t* need, int32_t* served_expert, int32_t* served_slot,
                            uint8_t* fetch_lo, uint8_t* fetch_hi, int32_t* round_start, int32_t* nrounds) {
  const moe::CacheHeader* h = nullptr;
  const moe_status_t st = cache_header(state, &h);
  if (st != MOE_OK) return st;
  if (!need || !served_expert || !served_slot || !fetch_lo || !fetch_hi || !round_start || !nrounds)
    return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < h->E; ++e)  // validated before the state changes
    if (need[e] > h->P) return MOE_ERR_INVALID_ARG;
  *nrounds = moe::cache_plan(moe::cache_view(state, h->E, h->S), need, served_expert, served_slot, fetch_lo,
                             fetch_hi, round_start);
  return MOE_OK;
}

moe_status_t moe_cache_slots(const void* state, int32_t* expert_of, uint8_t* planes) {
  const moe::CacheHeader* h = nullptr;
  const moe_status_t st = cache_header(state, &h);
  if (st != MOE_OK) return st;
  if (!expert_of || !planes) return MOE_ERR_INVALID_ARG;
  const moe::CacheView v = moe::cache_view(const_cast<void*>(state), h->E, h->S);
  for (int s = 0; s < h->S; ++s) {
    expert_of[s] = v.expert_of[s];
    planes[s] = v.planes[s];
  }
  return MOE_OK;
}

moe_status_t moe_cache_step(void* state, int64_t E, int64_t S, const moe_routing_t* routing, const uint8_t* bits,
                            int64_t T, int64_t k, int32_t* slot_ids, const moe_cache_plan_t* plan,
                            moe_stream_t stream) {
  if (!state || !routing || !slot_ids || !plan) return MOE_ERR_INVALID_ARG;
  if (!plan->served_expert || !plan->served_slot || !plan->fetch_lo || !plan->fetch_hi || !plan->nserved ||
      !plan->overflow)
    return MOE_ERR_INVALID_ARG;
  const moe_status_t rs = check_route_shape(T, E, k);
  if (rs != MOE_OK) return rs;
  if (S < 1 || S > E) return MOE_ERR_INVALID_ARG;
  if (S < (T * k < E ? T * k : E)) return MOE_ERR_UNSUPPORTED_SHAPE;  // one round only
  const moe_status_t rc = check_routing(routing);
  if (rc != MOE_OK) return rc;
  if ((reinterpret_cast<uintptr_t>(state) & 7u) || (reinterpret_cast<uintptr_t>(slot_ids) & 3u))
    return MOE_ERR_MISALIGNED;
  if (T == 0) return MOE_OK;
  return from_cuda(moe::launch_cache_step(state, *routing, bits, int(T * k), slot_ids, *plan, as_stream(stream)));
}

moe_status_t moe_cache_fetch(const moe_cache_plan_t* plan, int64_t E, const moe_experts_t* host_store,
                             const moe_experts_t* slots, int64_t H, int64_t I, moe_stream_t stream) {
  if (!plan || !host_store || !slots) return MOE_ERR_INVALID_ARG;
  if (host_store->fmt != slots->fmt) return MOE_ERR_INVALID_ARG;
  const void* ps[] = {host_store->w13, host_store->w13_scale, host_store->w2, host_store->w2_scale,
                      slots->w13, slots->w13_scale, slots->w2, slots->w2_scale};
  for (const void* p : ps)
    if (!p) return MOE_ERR_INVALID_ARG;
  if (host_store->fmt == MOE_FMT_NVFP4 &&
      (!host_store->w13_gscale || !host_store->w2_gscale || !slots->w13_gscale || !slots->w2_gscale))
    return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > MOE_MAX_EXPERTS || H % 256 != 0 || I % 128 != 0 || H < 256 || I < 128)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  for (const void* p : ps)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_cache_fetch(*plan, int(E), *host_store, *slots, int(H), int(I), as_stream(stream)));
}

moe_status_t moe_permute(const int32_t* ids, int64_t T, int64_t k, int64_t E, const moe_routing_t* out,
                         moe_stream_t stream) {
  const moe_status_t rs = check_route_shape(T, E, k);
  if (rs != MOE_OK) return rs;
  if (!ids || !out || !out->expert_offsets || !out->sorted_pair || !out->pair_to_row || !out->expert_list)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(ids) || !aligned16(out->expert_offsets) || !aligned16(out->sorted_pair) ||
      !aligned16(out->pair_to_row) || !aligned16(out->expert_list))
    return MOE_ERR_MISALIGNED;
  if (T == 0) return MOE_OK;  // as moe_route_topk: nothing to permute, no pointer is read
  return from_cuda(moe::launch_permute(ids, int(T * k), int(E), *out, as_stream(stream)));
}

moe_status_t moe_select_bits(const float* topk_w, int64_t T, int64_t k, const float thresholds[3],
                             const uint8_t choices[4], uint8_t* bits, moe_stream_t stream) {
  if (!topk_w || !thresholds || !choices || !bits) return MOE_ERR_INVALID_ARG;
  if (T < 0 || k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_INVALID_ARG;
  if (!(thresholds[0] <= thresholds[1] && thresholds[1] <= thresholds[2])) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (choices[i] < 1 || choices[i] > 8) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_w) || !aligned16(bits)) return MOE_ERR_MISALIGNED;
  if (T == 0) return MOE_OK;
  return from_cuda(moe::launch_select_bits(topk_w, T * k, thresholds, choices, bits, as_stream(stream)));
}

size_t moe_ffn_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, moe_format_t fmt) {
  if (T < 0 || H < 1 || I < 1 || k < 1) return 0;
  return moe::ffn_workspace_bytes(T, H, I, E, k, fmt);
}

moe_status_t moe_grouped_ffn(const uint16_t* x, const moe_routing_t* routing, const moe_experts_t* experts,
                             const uint8_t* bits, int64_t T, int64_t H, int64_t I, int64_t E, int64_t k,
                             uint16_t* y_rows, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  if (!experts) return MOE_ERR_INVALID_ARG;
  moe_status_t s = check_route_shape(T, E, k);
  if (s != MOE_OK) return s;
  const moe_experts_t& ex = *experts;
  if (ex.fmt != MOE_FMT_W4G128 && ex.fmt != MOE_FMT_BITPLANE8 && ex.fmt != MOE_FMT_NVFP4)
    return MOE_ERR_INVALID_ARG;
  if (!ex.w13 || !ex.w13_scale || !ex.w2 || !ex.w2_scale) return MOE_ERR_INVALID_ARG;
  if (ex.fmt == MOE_FMT_NVFP4 && (!ex.w13_gscale || !ex.w2_gscale)) return MOE_ERR_INVALID_ARG;
  if (H < 256 || H % 256 != 0 || I < 128 || I % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (H > 65536 || I > 65536 || !moe::ffn_shape_supported(H, I, ex.fmt)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (int64_t(E) * 2 * I > INT_MAX || T * k > INT_MAX / (H > I ? H : I)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;  // no pairs; no activation or output pointer is read
  if (!x || !y_rows) return MOE_ERR_INVALID_ARG;
  if (ex.fmt == MOE_FMT_BITPLANE8 && !bits) return MOE_ERR_INVALID_ARG;
  if ((s = check_routing(routing)) != MOE_OK) return s;
  const void* ps[] = {x, ex.w13, ex.w13_scale, ex.w2, ex.w2_scale, y_rows};
  for (const void* p : ps)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  if ((bits && !aligned16(bits)) || (ex.w13_gscale && !aligned16(ex.w13_gscale)) ||
      (ex.w2_gscale && !aligned16(ex.w2_gscale)))
    return MOE_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < moe::ffn_workspace_bytes(T, H, I, E, k, ex.fmt)) return MOE_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MOE_ERR_MISALIGNED;
  if (!moe::device_error_word()) return MOE_ERR_CUDA;
  return from_cuda(moe::launch_grouped_ffn(x, *routing, ex, bits, int(T), int(H), int(I), int(E), int(k), y_rows,
                                           workspace, as_stream(stream)));
}

// shape rules of the W4A4 path: K stages of 256 elements (H), 64-element K blocks and
// 64-row gate/up weight tiles (I), 128-row down weight tiles (H)
static moe_status_t w4a4_shape(int64_t H, int64_t I, int64_t E) {
  if (H < 256 || H % 256 != 0 || I < 128 || I % 128 != 0 || H > 65536 || I > 65536) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (E < 1 || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (int64_t(E) * 2 * I > INT_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

static moe_status_t w4a4_experts(const moe_experts_t* experts) {
  if (!experts) return MOE_ERR_INVALID_ARG;
  const moe_experts_t& ex = *experts;
  if (ex.fmt != MOE_FMT_NVFP4) return MOE_ERR_INVALID_ARG;
  if (!ex.w13 || !ex.w13_scale || !ex.w2 || !ex.w2_scale || !ex.w13_gscale || !ex.w2_gscale) return MOE_ERR_INVALID_ARG;
  const void* ps[] = {ex.w13, ex.w13_scale, ex.w2, ex.w2_scale, ex.w13_gscale, ex.w2_gscale};
  for (const void* p : ps)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

size_t moe_w4a4_scale_tiles_bytes(int64_t H, int64_t I, int64_t E) {
  if (H < 1 || I < 1 || E < 1) return 0;
  return moe::w4a4_scale_tiles_bytes(H, I, E);
}

moe_status_t moe_w4a4_prepare(const moe_experts_t* experts, int64_t H, int64_t I, int64_t E, void* scale_tiles,
                              size_t scale_tiles_bytes, moe_stream_t stream) {
  moe_status_t s = w4a4_shape(H, I, E);
  if (s != MOE_OK) return s;
  if ((s = w4a4_experts(experts)) != MOE_OK) return s;
  if (!scale_tiles) return MOE_ERR_INVALID_ARG;
  if (!aligned16(scale_tiles)) return MOE_ERR_MISALIGNED;
  if (scale_tiles_bytes < moe::w4a4_scale_tiles_bytes(H, I, E)) return MOE_ERR_WORKSPACE;
  return from_cuda(moe::launch_w4a4_prepare(*experts, int(H), int(I), int(E), static_cast<uint8_t*>(scale_tiles),
                                            as_stream(stream)));
}

size_t moe_ffn_w4a4_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
  if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1) return 0;
  return moe::w4a4_workspace_bytes(T, H, I, E, k);
}

moe_status_t moe_grouped_ffn_w4a4(const uint16_t* x, const moe_routing_t* routing, const moe_experts_t* experts,
                                  const void* scale_tiles, int64_t T, int64_t H, int64_t I, int64_t E, int64_t k,
                                  uint16_t* y_rows, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  moe_status_t s = check_route_shape(T, E, k);
  if (s != MOE_OK) return s;
  if ((s = w4a4_shape(H, I, E)) != MOE_OK) return s;
  if ((s = w4a4_experts(experts)) != MOE_OK) return s;
  if (T * k > INT_MAX / (H > I ? H : I)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!x || !y_rows || !scale_tiles) return MOE_ERR_INVALID_ARG;
  if ((s = check_routing(routing)) != MOE_OK) return s;
  if (!aligned16(x) || !aligned16(y_rows) || !aligned16(scale_tiles)) return MOE_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < moe::w4a4_workspace_bytes(T, H, I, E, k)) return MOE_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MOE_ERR_MISALIGNED;
  if (!moe::device_error_word()) return MOE_ERR_CUDA;
  return from_cuda(moe::launch_grouped_ffn_w4a4(x, *routing, *experts, static_cast<const uint8_t*>(scale_tiles),
                                                int(T), int(H), int(I), int(E), int(k), y_rows, workspace,
                                                as_stream(stream)));
}

moe_status_t moe_combine(const uint16_t* y_rows, const moe_routing_t* routing, const uint16_t* residual,
                         int64_t T, int64_t H, int64_t k, uint16_t* out, moe_stream_t stream) {
  if (T < 0 || k < 1 || k > MOE_MAX_TOPK || H < 8) return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T > INT_MAX / k || T * k > INT64_MAX / H) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;  // no tokens; no pointer is read
  if (!y_rows || !out) return MOE_ERR_INVALID_ARG;
  moe_status_t s = check_routing(routing);
  if (s != MOE_OK) return s;
  if (!aligned16(y_rows) || !aligned16(out) || (residual && !aligned16(residual))) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_combine(y_rows, *routing, residual, int(T), int(H), int(k), out, as_stream(stream)));
}

moe_status_t moe_gather_rows(const uint16_t* src, const int32_t* idx, int64_t n, int64_t div, int64_t H,
                             uint16_t* dst, moe_stream_t stream) {
  if (n < 0 || div < 1 || H < 8) return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0 || n > INT_MAX || H > INT_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return MOE_OK;
  if (!src || !idx || !dst) return MOE_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst) || (reinterpret_cast<uintptr_t>(idx) & 3u)) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_gather_rows_by(src, idx, int(n), int(div), int(H), dst, as_stream(stream)));
}

moe_status_t moe_ids_from_counts(const int32_t* counts, int64_t S, int64_t El, int32_t* ids, moe_stream_t stream) {
  if (!counts || !ids || S < 1 || El < 1) return MOE_ERR_INVALID_ARG;
  if (S * El > (int64_t(1) << 20)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(counts) & 3u) || (reinterpret_cast<uintptr_t>(ids) & 3u)) return MOE_ERR_MISALIGNED;
  return from_cuda(moe::launch_ids_from_counts(counts, int(S), int(El), ids, as_stream(stream)));
}

moe_status_t moe_check_device_errors(moe_stream_t stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpyFromSymbol(&word, g_moe_error_word, sizeof(word)) != cudaSuccess) return MOE_ERR_CUDA;
  if (word != 0) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_moe_error_word, &zero, sizeof(zero)) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_ERR_DEVICE_TIMEOUT;
  }
  return MOE_OK;
}

moe_status_t moe_synth_normal_bf16(uint16_t* out, int64_t n, int64_t start, uint64_t seed, double stddev,
                                   moe_stream_t stream) {
  if (!out || n < 0 || start < 0) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (n / 256 >= int64_t(INT_MAX)) return MOE_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(moe::launch_synth_normal(out, n, start, seed, stddev, as_stream(stream)));
}

moe_status_t moe_synth_uniform_bf16(uint16_t* out, int64_t n, int64_t start, uint64_t seed, double lo, double hi,
                                    moe_stream_t stream) {
  if (!out || n < 0 || start < 0) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (n / 256 >= int64_t(INT_MAX)) return MOE_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(moe::launch_synth_uniform(out, n, start, seed, lo, hi, as_stream(stream)));
}

}  // extern "C"
