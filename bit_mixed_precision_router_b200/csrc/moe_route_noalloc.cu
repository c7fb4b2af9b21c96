// moe_route_topk_noalloc: the router (logits, top-k, permutation) for callers that
// cannot hand the library any device workspace.
//
// Some callers have no way to allocate: an engine whose device memory is planned
// once up front and handed out as fixed buffers (any cudaMalloc from inside a
// layer would break its plan or fail outright), a custom-op host that passes only
// the op's inputs and outputs, or code that runs while a stream is being captured
// into a CUDA graph in global mode, where cudaMalloc is not allowed.  For them the
// router's fp32 logits scratch lives in a fixed device array that is part of this
// library image instead of a caller-provided workspace.
//
// Limits and sharing:
//   - the array holds kMaxLogits = MOE_NOALLOC_MAX_LOGITS floats (256 KiB) for the
//     logits, then 256 bytes whose first word is the one-launch router's completion
//     counter; a call with T * E above kMaxLogits is rejected with
//     MOE_ERR_UNSUPPORTED_SHAPE;
//   - the counter sits at the same place for every shape, after every logit any call
//     can write, so calls of different shapes in any order find it at zero;
//   - every GPU that loads the library holds the array until the process exits;
//   - all calls share it: two calls whose kernels overlap on the same GPU (for
//     example on two streams) race on it and give undefined routing;
//   - the logits need no clearing (each call writes every logit it later reads); the
//     counter starts at zero because device variables are zero-initialised when the
//     module loads, and every call that uses it leaves it at zero.
// Set-up: the first call on a device looks up the array's device address with
// cudaGetSymbolAddress (the host-side name is only a stand-in, never a device
// address) while that device is current, caches it per device, and sets the router
// kernels' shared-memory attributes for that device.  Make that first call before
// capturing a stream into a graph; later calls make no set-up call.
#include <atomic>
#include <climits>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace {

constexpr int64_t kMaxLogits = MOE_NOALLOC_MAX_LOGITS;

static __device__ __align__(256) float g_route_logits_scratch[kMaxLogits + 64];

// Device address of g_route_logits_scratch on the current device, or nullptr.  The
// first call per device also prepares the router kernels for that device.
float* scratch_on_current_device() {
  static std::atomic<float*> cached[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  float* s = cached[dev].load(std::memory_order_acquire);
  if (!s) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_logits_scratch) != cudaSuccess || !p) return nullptr;
    if (moe::route_prepare_device() != cudaSuccess) return nullptr;
    s = static_cast<float*>(p);
    cached[dev].store(s, std::memory_order_release);
  }
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" moe_status_t moe_route_topk_noalloc(const uint16_t* x, const uint16_t* w_router, const float* bias,
                                               int64_t T, int64_t H, int64_t E, int64_t k,
                                               const moe_routing_t* out, moe_stream_t stream) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > MOE_MAX_EXPERTS || k < 1 || k > E || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (H < 256 || H % 256 != 0 || H > INT_MAX / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T > kMaxLogits / E) return MOE_ERR_UNSUPPORTED_SHAPE;  // logits would not fit the fixed array
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !out) return MOE_ERR_INVALID_ARG;
  const void* ps[] = {out->topk_ids,    out->topk_w,      out->expert_offsets,
                      out->sorted_pair, out->pair_to_row, out->expert_list};
  for (const void* p : ps)
    if (!p) return MOE_ERR_INVALID_ARG;
  for (const void* p : ps)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  if (!aligned16(x) || !aligned16(w_router) || (bias && !aligned16(bias))) return MOE_ERR_MISALIGNED;
  float* logits = scratch_on_current_device();
  if (!logits) return MOE_ERR_CUDA;
  unsigned* counter = reinterpret_cast<unsigned*>(logits + kMaxLogits);  // never reached by a logit write
  const cudaError_t err = moe::launch_route(x, w_router, bias, int(T), int(H), int(E), int(k), *out, logits,
                                            counter, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
