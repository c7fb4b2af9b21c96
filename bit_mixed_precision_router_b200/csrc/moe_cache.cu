// Expert slot cache on the device: one step's plan from the routing (single round) and
// the copy of the planned planes from pinned host memory into the slots.
//
// After "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference" (abstract:
// experts in pinned host memory run through a GPU-resident slot cache) and "PagedMoE:
// Cross-Precision Expert Caching for Token-Level Dynamic Precision in SSD-Resident MoE
// Inference" (abstract: a cached plane prefix is reused or extended by fetching only the
// missing planes).
//
// With at least as many slots as the step routes experts to, the sequential plan
// (moe_cache_core.cuh) never evicts a routed expert: a miss always finds a slot holding
// no routed expert.  It then reduces to: resident routed experts are hits or extensions;
// misses, in ascending id, take free slots by index, then slots of non-routed experts by
// (last step used, slot index).  k_cache_step computes exactly that in one CTA, in
// parallel, and rewrites every pair's expert id as its slot id for the permutation.
#include "moe_cache_core.cuh"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kStepThreads = 1024;


// block-wide exclusive scan of one int per thread (1024 threads)
__device__ int block_excl_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = sh[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += y;
    }
    sh[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int base = warp ? sh[warp - 1] : 0;
  *total = sh[31];
  __syncthreads();
  return base + x - v;
}

// One CTA: need[] from the routing, hits and extensions, victims for the misses, state
// update, the plan, and each pair's slot id.  E <= 1024, S <= E.
__global__ void __launch_bounds__(kStepThreads) k_cache_step(void* state, const int32_t* __restrict__ offsets,
                                                             const int32_t* __restrict__ sorted_pair,
                                                             const uint8_t* __restrict__ bits,
                                                             const int32_t* __restrict__ topk_ids, int npairs,
                                                             int32_t* __restrict__ slot_ids, moe_cache_plan_t out) {
  __shared__ int s_need[MOE_MAX_EXPERTS];
  __shared__ int s_scan[32];
  CacheHeader* h = static_cast<CacheHeader*>(state);
  const int E = h->E, S = h->S, P = h->P;
  CacheView v = cache_view(state, E, S);
  const int t = threadIdx.x;

  // demand per expert
  int need = 0;
  if (t < E) {
    for (int r = offsets[t]; r < offsets[t + 1]; ++r) {
      const int w = bits ? int(bits[sorted_pair[r]]) : 1;
      need = max(need, min(P, max(1, w)));
    }
    s_need[t] = need;
  }
  __syncthreads();
  const bool routed = t < E && need > 0;
  const int my_slot = routed ? v.slot_of[t] : -1;
  const bool miss = routed && my_slot < 0;

  // candidates: free slots first (by index), then slots of non-routed experts by (last_use, slot)
  bool cand = false;
  int64_t key_use = 0;
  int key_grp = 0;
  if (t < S) {
    const int x = v.expert_of[t];
    cand = x < 0 || s_need[x] == 0;
    key_grp = x < 0 ? 0 : 1;
    key_use = x < 0 ? 0 : v.last_use[t];
  }
  int total_miss = 0, total_cand = 0;
  const int miss_rank = block_excl_scan(miss ? 1 : 0, s_scan, &total_miss);
  (void)block_excl_scan(cand ? 1 : 0, s_scan, &total_cand);
  const bool overflow = total_miss > total_cand;
  if (t == 0) {
    *out.overflow = overflow ? 1 : 0;
    if (overflow) *out.nserved = 0;  // a fetch of this plan copies nothing
  }
  if (overflow) return;  // uniform across the block

  // rank of each candidate slot by (group, last_use, slot): count smaller keys
  __shared__ int s_victim[MOE_MAX_EXPERTS];  // candidate rank -> slot
  if (cand) {
    int rank = 0;
    for (int s = 0; s < S; ++s) {
      const int x = v.expert_of[s];
      const bool c = x < 0 || s_need[x] == 0;
      if (!c || s == t) continue;
      const int g = x < 0 ? 0 : 1;
      const int64_t u = x < 0 ? 0 : v.last_use[s];
      if (g < key_grp || (g == key_grp && (u < key_use || (u == key_use && s < t)))) ++rank;
    }
    s_victim[rank] = t;
  }
  __syncthreads();

  const int64_t step = h->step + 1;
  // each miss reads its victim and that victim's previous expert before anyone writes
  int vslot = -1, vold = -1;
  if (miss) {
    vslot = s_victim[miss_rank];
    vold = v.expert_of[vslot];
  }
  int have = 0;
  if (routed && !miss) have = v.planes[my_slot];
  __syncthreads();
  if (miss && vold >= 0) v.slot_of[vold] = -1;
  __syncthreads();
  int served_rank = 0, nserved = 0;
  served_rank = block_excl_scan(routed ? 1 : 0, s_scan, &nserved);
  if (routed) {
    const int s = miss ? vslot : my_slot;
    int lo = need, hi = need;
    if (miss) {
      v.expert_of[s] = t;
      v.slot_of[t] = s;
      v.planes[s] = uint8_t(need);
      lo = 0;
    } else if (have < need) {
      v.planes[s] = uint8_t(need);
      lo = have;
    }
    v.last_use[s] = step;
    out.served_expert[served_rank] = t;
    out.served_slot[served_rank] = s;
    out.fetch_lo[served_rank] = uint8_t(lo);
    out.fetch_hi[served_rank] = uint8_t(hi);
  }
  if (t == 0) {
    h->step = step;
    h->mark += 1;
    *out.nserved = nserved;
  }
  __syncthreads();
  // the pairs' slot ids (every routed expert is resident now)
  for (int p = t; p < npairs; p += kStepThreads) slot_ids[p] = v.slot_of[topk_ids[p]];
}

// Copies planes [lo, hi) of each served expert (and its scales on a miss) from the host
// store (pinned, device-accessible) into its slot.  grid.y = served index; grid.x splits
// the bytes; 16-byte vectors, four in flight per thread.
struct StoreDims {
  const uint8_t* host_w;   // [E][P][plane_bytes] (whole experts: P = 1)
  const uint8_t* host_s;   // [E][scale_bytes]
  uint8_t* slot_w;         // [S][P][plane_bytes]
  uint8_t* slot_s;         // [S][scale_bytes]
  const float* host_g;     // NVFP4: [E] per-expert scale, else null
  float* slot_g;           // NVFP4: [S]
  int64_t plane_bytes, scale_bytes;  // multiples of 16
  int P;
};

__global__ void k_cache_fetch(moe_cache_plan_t plan, StoreDims d) {
  const int i = blockIdx.y;
  if (i >= *plan.nserved) return;
  const int e = plan.served_expert[i], s = plan.served_slot[i];
  const int lo = plan.fetch_lo[i], hi = plan.fetch_hi[i];
  if (lo == hi) return;
  if (d.host_g && lo == 0 && blockIdx.x == 0 && threadIdx.x == 0) d.slot_g[s] = d.host_g[e];
  const int64_t wbytes = int64_t(hi - lo) * d.plane_bytes;
  const int64_t sbytes = lo == 0 ? d.scale_bytes : 0;
  const uint4* wsrc = reinterpret_cast<const uint4*>(d.host_w + (int64_t(e) * d.P + lo) * d.plane_bytes);
  uint4* wdst = reinterpret_cast<uint4*>(d.slot_w + (int64_t(s) * d.P + lo) * d.plane_bytes);
  const uint4* ssrc = reinterpret_cast<const uint4*>(d.host_s + int64_t(e) * d.scale_bytes);
  uint4* sdst = reinterpret_cast<uint4*>(d.slot_s + int64_t(s) * d.scale_bytes);
  const int64_t nw = wbytes / 16, ns = sbytes / 16, n = nw + ns;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t q0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; q0 < n; q0 += 4 * stride) {
    uint4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t q = q0 + u * stride;
      if (q < n) r[u] = q < nw ? wsrc[q] : ssrc[q - nw];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t q = q0 + u * stride;
      if (q < n) {
        if (q < nw)
          wdst[q] = r[u];
        else
          sdst[q - nw] = r[u];
      }
    }
  }
}

}  // namespace

size_t cache_state_bytes_dev(int E, int S) { return cache_state_bytes(E, S); }

cudaError_t launch_cache_step(void* state, const moe_routing_t& r, const uint8_t* bits, int P, int32_t* slot_ids,
                              const moe_cache_plan_t& plan, cudaStream_t st) {
  k_cache_step<<<1, kStepThreads, 0, st>>>(state, r.expert_offsets, r.sorted_pair, bits, r.topk_ids, P, slot_ids,
                                           plan);
  return cudaGetLastError();
}

// one matrix (w13 or w2) of the served experts; grid.y covers every possible served entry
static cudaError_t fetch_matrix(const moe_cache_plan_t& plan, int E, const StoreDims& d, cudaStream_t st) {
  const int64_t per = int64_t(d.P) * d.plane_bytes + d.scale_bytes;
  const int chunks = int((per / 16 + 4 * 256 - 1) / (4 * 256));
  dim3 grid(unsigned(chunks < 8 ? chunks : 8), unsigned(E));
  k_cache_fetch<<<grid, 256, 0, st>>>(plan, d);
  return cudaGetLastError();
}

cudaError_t launch_cache_fetch(const moe_cache_plan_t& plan, int E, const moe_experts_t& host, const moe_experts_t& slots,
                               int H, int I, cudaStream_t st) {
  StoreDims d{};
  const bool bp = host.fmt == MOE_FMT_BITPLANE8, fp4 = host.fmt == MOE_FMT_NVFP4;
  d.P = bp ? 8 : 1;
  for (int m = 0; m < 2; ++m) {
    const int64_t N = m == 0 ? 2 * int64_t(I) : int64_t(H), K = m == 0 ? int64_t(H) : int64_t(I);
    d.plane_bytes = bp ? N * K / 8 : N * K / 2;
    d.scale_bytes = fp4 ? N * K / 16 : N * (K / 128) * 2;
    d.host_w = static_cast<const uint8_t*>(m == 0 ? host.w13 : host.w2);
    d.host_s = static_cast<const uint8_t*>(m == 0 ? host.w13_scale : host.w2_scale);
    d.slot_w = static_cast<uint8_t*>(const_cast<void*>(m == 0 ? slots.w13 : slots.w2));
    d.slot_s = static_cast<uint8_t*>(const_cast<void*>(m == 0 ? slots.w13_scale : slots.w2_scale));
    d.host_g = fp4 ? (m == 0 ? host.w13_gscale : host.w2_gscale) : nullptr;
    d.slot_g = fp4 ? const_cast<float*>(m == 0 ? slots.w13_gscale : slots.w2_gscale) : nullptr;
    const cudaError_t err = fetch_matrix(plan, E, d, st);
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace moe
