// Router: logits in one fixed fp32 order, top-k with softmax weights, and the
// stable permutation of (token, slot) pairs by expert.
//
// Logit order (pins the routing ids bit for bit): 32 partial sums; partial L
// accumulates h = 256 j + 8 L + i with j outer and i = 0..7 inner by fmaf from +0;
// partials are then added pairwise at lane distance 16, 8, 4, 2, 1; then + bias.
// One warp evaluates a 4-token x 8-expert tile: lane L holds partial L of all 32
// logits, and a recursive-halving exchange (which adds exactly the same pairs as
// the pairwise tree) leaves logit (t, e) = (L / 8, L % 8) in lane L.
#include <atomic>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kTileT = 4;  // tokens per warp tile
constexpr int kTileE = 8;  // experts per warp tile

template <int WT, int WE>
__global__ void __launch_bounds__(32 * WT * WE) k_router_logits(const uint16_t* __restrict__ x,
                                                                const uint16_t* __restrict__ wr,
                                                                const float* __restrict__ bias, int T, int H,
                                                                int E, float* __restrict__ logits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = (blockIdx.x * WT + warp % WT) * kTileT;
  const int e0 = (blockIdx.y * WE + warp / WT) * kTileE;
  const uint16_t* xr[kTileT];
  const uint16_t* wrow[kTileE];
#pragma unroll
  for (int t = 0; t < kTileT; ++t) xr[t] = (t0 + t < T) ? x + size_t(t0 + t) * H : nullptr;
#pragma unroll
  for (int e = 0; e < kTileE; ++e) wrow[e] = (e0 + e < E) ? wr + size_t(e0 + e) * H : nullptr;

  float acc[kTileT][kTileE];
#pragma unroll
  for (int t = 0; t < kTileT; ++t)
#pragma unroll
    for (int e = 0; e < kTileE; ++e) acc[t][e] = 0.f;

  const int J = H / 256;
  for (int j = 0; j < J; ++j) {
    const int h = 256 * j + 8 * lane;
    uint4 xv[kTileT], wv[kTileE];
#pragma unroll
    for (int t = 0; t < kTileT; ++t)
      xv[t] = xr[t] ? *reinterpret_cast<const uint4*>(xr[t] + h) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int e = 0; e < kTileE; ++e) wv[e] = wrow[e] ? ldg_nc_v4(wrow[e] + h) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float xf[kTileT], wf[kTileE];
#pragma unroll
      for (int t = 0; t < kTileT; ++t) {
        const uint32_t u = (i < 2) ? xv[t].x : (i < 4) ? xv[t].y : (i < 6) ? xv[t].z : xv[t].w;
        xf[t] = (i & 1) ? bf16_hi(u) : bf16_lo(u);
      }
#pragma unroll
      for (int e = 0; e < kTileE; ++e) {
        const uint32_t u = (i < 2) ? wv[e].x : (i < 4) ? wv[e].y : (i < 6) ? wv[e].z : wv[e].w;
        wf[e] = (i & 1) ? bf16_hi(u) : bf16_lo(u);
      }
#pragma unroll
      for (int t = 0; t < kTileT; ++t)
#pragma unroll
        for (int e = 0; e < kTileE; ++e) acc[t][e] = fmaf(xf[t], wf[e], acc[t][e]);
    }
  }

  // Recursive halving over the 32 outputs o = 8 t + e.
  float v[32];
#pragma unroll
  for (int o = 0; o < 32; ++o) v[o] = acc[o / kTileE][o % kTileE];
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) {
    const bool upper = (lane & d) != 0;
#pragma unroll
    for (int q = 0; q < d; ++q) {
      const float send = upper ? v[q] : v[q + d];
      const float keep = upper ? v[q + d] : v[q];
      v[q] = keep + __shfl_xor_sync(0xffffffffu, send, d);
    }
  }
  const int t = t0 + lane / kTileE, e = e0 + lane % kTileE;
  if (t < T && e < E) logits[size_t(t) * E + e] = bias ? v[0] + bias[e] : v[0];
}

// ---------------------------------------------------------------- top-k
// Order-preserving unsigned key of a logit: larger logit -> larger key.  NaN ranks
// with -inf; -0 is folded into +0 so that equal logits tie by expert id.  Key 0 is
// below every logit and marks "no candidate".
MOE_DEVICE uint32_t order_key(float f) {
  if (f != f) f = -INFINITY;
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
MOE_DEVICE float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// One warp selects token t's top-k from logits[t][0..E), E <= 32 * NV, and writes ids
// and softmax weights; also returns the ids to the caller's lanes (lane j holds slot
// j).  Lane L holds experts q*32 + L.  Each round takes the warp maximum of the lanes'
// best keys, then the lowest expert id among the lanes that hold that key.
template <int NV>
MOE_DEVICE int warp_topk_nv(const float* lg, int E, int k, int t, int32_t* __restrict__ ids,
                            float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NV];
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int e = q * 32 + lane;
    key[q] = (e < E) ? order_key(__ldcg(lg + e)) : 0u;
  }
  uint32_t my_key = 0;
  int my_id = -1;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0;
    int bq = 0;
#pragma unroll
    for (int q = 0; q < NV; ++q)
      if (key[q] > bk) {  // strict: the lowest expert id among this lane's equal keys
        bk = key[q];
        bq = q;
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t id = __reduce_min_sync(0xffffffffu, bk == m ? uint32_t(bq * 32 + lane) : 0xffffffffu);
    if (int(id & 31u) == lane) {
#pragma unroll
      for (int q = 0; q < NV; ++q)
        if (q == int(id >> 5)) key[q] = 0u;
    }
    if (lane == j) {
      my_key = m;
      my_id = int(id);
    }
  }
  // softmax over the k selected, relative to the largest (slot 0)
  const float mine = key_value(my_key);
  const float l0 = __shfl_sync(0xffffffffu, mine, 0);
  const float ex = (lane < k) ? expf(mine - l0) : 0.f;
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ex, j);
  if (lane < k) {
    ids[size_t(t) * k + lane] = my_id;
    w[size_t(t) * k + lane] = __fdiv_rn(ex, sum);
  }
  return my_id;
}

MOE_DEVICE int warp_topk(const float* lg, int E, int k, int t, int32_t* __restrict__ ids, float* __restrict__ w) {
  static_assert(MOE_MAX_EXPERTS <= 1024, "warp_topk holds at most 32 logits per lane");
  if (E <= 32) return warp_topk_nv<1>(lg, E, k, t, ids, w);
  if (E <= 64) return warp_topk_nv<2>(lg, E, k, t, ids, w);
  if (E <= 128) return warp_topk_nv<4>(lg, E, k, t, ids, w);
  if (E <= 256) return warp_topk_nv<8>(lg, E, k, t, ids, w);
  if (E <= 512) return warp_topk_nv<16>(lg, E, k, t, ids, w);
  return warp_topk_nv<32>(lg, E, k, t, ids, w);
}

__global__ void k_topk(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ ids,
                       float* __restrict__ w) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  warp_topk(logits + size_t(t) * E, E, k, t, ids, w);
}

// ---------------------------------------------------------------- permutation
// Stable counting sort of P = T*k pairs by expert, by one CTA of NW = blockDim.x/32
// warps.  Warp w owns pairs [w*P/NW, (w+1)*P/NW); `cnt` is [NW][E] ints and `tot` [E]
// ints of shared memory.  Writes expert_offsets, expert_list, sorted_pair, pair_to_row.
MOE_DEVICE void permute_block(const int32_t* ids, int P, int E, int* cnt, int* tot, const moe_routing_t& out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, NW = blockDim.x >> 5;
  for (int i = threadIdx.x; i < NW * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int beg = int((int64_t(warp) * P) / NW), end = int((int64_t(warp + 1) * P) / NW);
  for (int p = beg + lane; p < end; p += 32) atomicAdd(&cnt[warp * E + ids[p]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int t = 0;
    for (int w = 0; w < NW; ++w) t += cnt[w * E + e];
    tot[e] = t;
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive prefix over experts and the ordered list of active experts; lane L owns
    // the contiguous range [L*per, (L+1)*per)
    const int per = (E + 31) / 32;
    const int b = min(E, lane * per), en = min(E, b + per);
    int sum = 0, act = 0;
    for (int e = b; e < en; ++e) {
      sum += tot[e];
      act += tot[e] > 0;
    }
    int isum = sum, iact = act;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v1 = __shfl_up_sync(0xffffffffu, isum, off), v2 = __shfl_up_sync(0xffffffffu, iact, off);
      if (lane >= off) {
        isum += v1;
        iact += v2;
      }
    }
    int run = isum - sum, pos = iact - act;
    for (int e = b; e < en; ++e) {
      const int t = tot[e];
      out.expert_offsets[e] = run;
      if (t > 0) out.expert_list[1 + pos++] = e;
      tot[e] = run;
      run += t;
    }
    if (lane == 31) {
      out.expert_offsets[E] = P;
      out.expert_list[0] = iact;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = tot[e];
    for (int w = 0; w < NW; ++w) {
      const int c = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  // stable scatter: walk each warp's range in order, 32 pairs at a time
  for (int base = beg; base < end; base += 32) {
    const int p = base + lane;
    const bool ok = p < end;
    const int id = ok ? ids[p] : -1;
    const unsigned act = __ballot_sync(0xffffffffu, ok);
    const unsigned peers = __match_any_sync(0xffffffffu, id) & act;
    const unsigned lt = (1u << lane) - 1u;
    int pos = 0;
    if (ok) pos = cnt[warp * E + id] + __popc(peers & lt);
    __syncwarp();
    if (ok && (__ffs(peers) - 1) == lane) cnt[warp * E + id] += __popc(peers);
    __syncwarp();
    if (ok) {
      out.sorted_pair[pos] = p;
      out.pair_to_row[p] = pos;
    }
  }
}

__global__ void __launch_bounds__(1024) k_permute(const int32_t* __restrict__ ids, int P, int E,
                                                  moe_routing_t out) {
  extern __shared__ int smem_i[];
  permute_block(ids, P, E, smem_i, smem_i + 32 * E, out);
}

// ---------------------------------------------------------------- small batches, fused
// One launch for few tokens: CTA b computes the logits of experts 8b .. 8b+7 for every
// token (warp = expert; the tokens are staged once in shared memory; the router row's
// chunks are loaded before any FMA), in the same fixed order as k_router_logits.  The
// last CTA to finish (completion counter, reset to 0 by that CTA) reads all logits
// back, selects every token's top-k and builds the permutation.
constexpr int kFusedMaxT = 16;
constexpr int kFusedWarps = 8;

__global__ void __launch_bounds__(32 * kFusedWarps) k_route_fused(const uint16_t* __restrict__ x,
                                                                 const uint16_t* __restrict__ wr,
                                                                 const float* __restrict__ bias, int T, int H, int E,
                                                                 int k, float* logits, unsigned* ticket,
                                                                 moe_routing_t out) {
  extern __shared__ __align__(16) uint8_t smem_u8[];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kFusedWarps + warp;
  const uint16_t* wrow = wr + size_t(e < E ? e : 0) * H;
  const int J = H / 256;
  // the first eight 256-wide chunks of this warp's router row are requested before
  // the tokens are staged, so the two memory latencies overlap
  uint4 wv[8];
#pragma unroll
  for (int q = 0; q < 8; ++q)
    wv[q] = (e < E && q < J) ? ldg_nc_v4(wrow + 256 * q + 8 * lane) : make_uint4(0, 0, 0, 0);
  // stage the tokens, four 16-byte loads in flight per thread
  {
    const int n16 = T * H / 8;
    const uint4* xs = reinterpret_cast<const uint4*>(x);
    uint4* xd = reinterpret_cast<uint4*>(smem_u8);
    for (int i0 = threadIdx.x; i0 < n16; i0 += 4 * blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < n16) v[u] = xs[i];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < n16) xd[i] = v[u];
      }
    }
  }
  __syncthreads();
  if (e < E) {
    float acc[kFusedMaxT];
#pragma unroll
    for (int t = 0; t < kFusedMaxT; ++t) acc[t] = 0.f;
    for (int j0 = 0; j0 < J; j0 += 8) {
      if (j0 > 0) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          wv[q] = (j0 + q < J) ? ldg_nc_v4(wrow + 256 * (j0 + q) + 8 * lane) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (j0 + q >= J) break;
        const uint32_t wu[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
#pragma unroll
        for (int t = 0; t < kFusedMaxT; ++t) {
          if (t >= T) break;
          const uint4 xv = *reinterpret_cast<const uint4*>(smem_u8 + (size_t(t) * H + 256 * (j0 + q) + 8 * lane) * 2);
          const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float xf = (i & 1) ? bf16_hi(xu[i >> 1]) : bf16_lo(xu[i >> 1]);
            const float wf = (i & 1) ? bf16_hi(wu[i >> 1]) : bf16_lo(wu[i >> 1]);
            acc[t] = fmaf(xf, wf, acc[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kFusedMaxT; ++t) {
      if (t >= T) break;
      float v = acc[t];
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
      if (lane == 0) logits[size_t(t) * E + e] = bias ? v + bias[e] : v;
    }
  }
  // last CTA: top-k and permutation
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = (atomicAdd(ticket, 1u) == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  int* ids_s = reinterpret_cast<int*>(smem_u8);  // the staged tokens are no longer needed
  for (int t = warp; t < T; t += kFusedWarps) {
    const int id = warp_topk(logits + size_t(t) * E, E, k, t, out.topk_ids, out.topk_w);
    if (lane < k) ids_s[t * k + lane] = id;
  }
  __syncthreads();
  const int P = T * k;
  int* cnt = ids_s + ((P + 3) & ~3);
  permute_block(ids_s, P, E, cnt, cnt + kFusedWarps * E, out);
  if (threadIdx.x == 0) *ticket = 0u;
}

__global__ void k_select_bits(const float* __restrict__ w, int64_t n, float t0, float t1, float t2, uint8_t c0,
                              uint8_t c1, uint8_t c2, uint8_t c3, uint8_t* __restrict__ bits) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const float v = w[i];
  bits[i] = (v < t0) ? c0 : (v < t1) ? c1 : (v < t2) ? c2 : c3;
}

// ---------------------------------------------------------------- launchers
static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace: the 32-bit completion counter of k_route_fused in the first 256 bytes (it
// must start at 0; every fused launch leaves it at 0), then fp32 logits [T][E].  The
// counter's place does not depend on the shape, so one workspace serves calls of any
// smaller (T, E) after a larger one.
size_t route_workspace_bytes(int64_t T, int64_t E, int64_t /*k*/) { return kRouteCounterBytes + align256(size_t(T * E * 4)); }

static bool use_fused(int T, int H, int E, int k) {
  const size_t stage = size_t(T) * H * 2;
  const size_t perm = size_t(((T * k + 3) & ~3) + kFusedWarps * E + E) * 4;
  return T <= kFusedMaxT && stage <= 64 * 1024 && perm <= 64 * 1024;
}

// Largest dynamic shared memory the router kernels request: k_route_fused 64 KiB (the
// tokens, or the permutation's counters), k_permute 33 ints per expert.
constexpr int kFusedSmemMax = 64 * 1024;
constexpr int kPermuteSmemMax = 33 * MOE_MAX_EXPERTS * int(sizeof(int));

cudaError_t route_prepare_device() {
  // once per device: raise both kernels' dynamic shared-memory limit to the largest any
  // call requests, so no later call (e.g. one inside a stream capture) sets attributes
  static std::atomic<bool> done[128] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  err = cudaFuncSetAttribute(k_route_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmemMax);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, kPermuteSmemMax);
  if (err != cudaSuccess) return err;
  done[dev].store(true, std::memory_order_release);
  return cudaSuccess;
}

cudaError_t launch_route(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H, int E, int k,
                         const moe_routing_t& out, float* logits, unsigned* counter, cudaStream_t st) {
  cudaError_t err = route_prepare_device();
  if (err != cudaSuccess) return err;
  if (use_fused(T, H, E, k)) {
    const size_t stage = size_t(T) * H * 2;
    const size_t perm = size_t(((T * k + 3) & ~3) + kFusedWarps * E + E) * 4;
    const size_t smem = stage > perm ? stage : perm;
    k_route_fused<<<dim3(unsigned((E + kFusedWarps - 1) / kFusedWarps)), 32 * kFusedWarps, smem, st>>>(
        x, wr, bias, T, H, E, k, logits, counter, out);
    return cudaGetLastError();
  }
  if (T >= 256) {
    constexpr int WT = 4, WE = 4;
    dim3 grid((T + WT * kTileT - 1) / (WT * kTileT), (E + WE * kTileE - 1) / (WE * kTileE));
    k_router_logits<WT, WE><<<grid, 32 * WT * WE, 0, st>>>(x, wr, bias, T, H, E, logits);
  } else {
    dim3 grid((T + kTileT - 1) / kTileT, (E + kTileE - 1) / kTileE);
    k_router_logits<1, 1><<<grid, 32, 0, st>>>(x, wr, bias, T, H, E, logits);
  }
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int P = T * k;
  k_topk<<<(T + 7) / 8, 256, 0, st>>>(logits, T, E, k, out.topk_ids, out.topk_w);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  return launch_permute(out.topk_ids, P, E, out, st);
}

cudaError_t launch_route_ws(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H, int E, int k,
                            const moe_routing_t& out, void* ws, cudaStream_t st) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  return launch_route(x, wr, bias, T, H, E, k, out, reinterpret_cast<float*>(base + kRouteCounterBytes),
                      reinterpret_cast<unsigned*>(base), st);
}

cudaError_t launch_permute(const int32_t* ids, int P, int E, const moe_routing_t& out, cudaStream_t st) {
  const cudaError_t err = route_prepare_device();
  if (err != cudaSuccess) return err;
  const size_t smem = size_t(33 * E) * sizeof(int);
  k_permute<<<1, 1024, smem, st>>>(ids, P, E, out);
  return cudaGetLastError();
}

cudaError_t launch_select_bits(const float* w, int64_t n, const float thr[3], const uint8_t ch[4],
                               uint8_t* bits, cudaStream_t st) {
  const int threads = 256;
  k_select_bits<<<dim3(unsigned((n + threads - 1) / threads)), threads, 0, st>>>(
      w, n, thr[0], thr[1], thr[2], ch[0], ch[1], ch[2], ch[3], bits);
  return cudaGetLastError();
}

}  // namespace moe
