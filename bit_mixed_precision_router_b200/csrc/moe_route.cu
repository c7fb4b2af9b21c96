// Router: logits in one fixed fp32 order, top-k with softmax weights, and the
// stable permutation of (token, slot) pairs by expert.
//
// Logit order (pins the routing ids bit for bit): 32 partial sums; partial L
// accumulates h = 256 j + 8 L + i with j outer and i = 0..7 inner by fmaf from +0;
// partials are then added pairwise at lane distance 16, 8, 4, 2, 1; then + bias.
// One warp evaluates a 4-token x 8-expert tile: lane L holds partial L of all 32
// logits, and a recursive-halving exchange (which adds exactly the same pairs as
// the pairwise tree) leaves logit (t, e) = (L / 8, L % 8) in lane L.
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
struct Cand {
  float v;
  int i;
};
MOE_DEVICE bool better(Cand a, Cand b) { return a.v > b.v || (a.v == b.v && a.i < b.i); }

// One warp selects token t's top-k from logits[t][0..E) and writes ids and
// softmax weights; also returns the ids to the caller's lanes (lane j holds slot j).
MOE_DEVICE int warp_topk(const float* __restrict__ lg, int E, int k, int t, int32_t* __restrict__ ids,
                         float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  constexpr int kMaxPerLane = MOE_MAX_EXPERTS / 32;
  float val[kMaxPerLane];
  uint32_t taken = 0;
#pragma unroll
  for (int q = 0; q < kMaxPerLane; ++q) {
    const int e = q * 32 + lane;
    float f = (e < E) ? lg[e] : -INFINITY;
    if (f != f) f = -INFINITY;  // NaN ranks last
    val[q] = f;
  }
  Cand mine{-INFINITY, 0x7fffffff};
  int my_id = -1;
  for (int j = 0; j < k; ++j) {
    Cand best{-INFINITY, 0x7fffffff};
#pragma unroll
    for (int q = 0; q < kMaxPerLane; ++q) {
      const int e = q * 32 + lane;
      if (e < E && !((taken >> q) & 1u)) {
        const Cand c{val[q], e};
        if (better(c, best)) best = c;
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      Cand o{__shfl_xor_sync(0xffffffffu, best.v, off), __shfl_xor_sync(0xffffffffu, best.i, off)};
      if (better(o, best)) best = o;
    }
    if ((best.i & 31) == lane) taken |= 1u << (best.i >> 5);
    if (lane == j) {
      mine = best;
      my_id = best.i;
    }
  }
  // softmax over the k selected, relative to the largest (slot 0)
  const float l0 = __shfl_sync(0xffffffffu, mine.v, 0);
  const float ex = (lane < k) ? expf(mine.v - l0) : 0.f;
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ex, j);
  if (lane < k) {
    ids[size_t(t) * k + lane] = my_id;
    w[size_t(t) * k + lane] = __fdiv_rn(ex, sum);
  }
  return my_id;
}

__global__ void k_topk(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ ids,
                       float* __restrict__ w) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  warp_topk(logits + size_t(t) * E, E, k, t, ids, w);
}

// ---------------------------------------------------------------- permutation
// Block-wide exclusive scan of one value per thread (blockDim.x == 1024).
MOE_DEVICE int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += n;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sums[lane];
    int si = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, si, off);
      if (lane >= off) si += n;
    }
    warp_sums[lane] = si - s;  // exclusive prefix of warp totals
    if (lane == 31) *total = si;
  }
  __syncthreads();
  return warp_sums[warp] + inc - v;
}

// Stable counting sort of P = T*k pairs by expert.  One CTA of 1024 threads.
// Warp w owns pairs [w*P/32, (w+1)*P/32); cnt is [32][E] ints of shared memory.
MOE_DEVICE void permute_block(const int32_t* ids, int P, int E, int* cnt, int* scratch,
                              const moe_routing_t& out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 32 * E; i += 1024) cnt[i] = 0;
  __syncthreads();
  const int beg = int((int64_t(warp) * P) / 32), end = int((int64_t(warp + 1) * P) / 32);
  for (int p = beg + lane; p < end; p += 32) atomicAdd(&cnt[warp * E + ids[p]], 1);
  __syncthreads();
  // per expert: column prefix over warps, then the scan over experts
  int* warp_sums = scratch;   // [32]
  int* total_out = scratch + 32;
  int* n_active = scratch + 33;
  for (int eb = 0; eb < E; eb += 1024) {
    // E <= 1024, so this loop runs once; kept explicit for clarity
    const int e = eb + threadIdx.x;
    int tot = 0;
    if (e < E)
      for (int ww = 0; ww < 32; ++ww) tot += cnt[ww * E + e];
    const int off = block_exclusive_scan(tot, warp_sums, total_out);
    const int flag = (e < E && tot > 0) ? 1 : 0;
    const int pos = block_exclusive_scan(flag, warp_sums, n_active);
    if (e < E) {
      out.expert_offsets[e] = off;
      if (flag) out.expert_list[1 + pos] = e;
      int run = off;
      for (int ww = 0; ww < 32; ++ww) {
        const int c = cnt[ww * E + e];
        cnt[ww * E + e] = run;
        run += c;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    out.expert_offsets[E] = P;
    out.expert_list[0] = *n_active;
  }
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
  __shared__ int scratch[40];
  permute_block(ids, P, E, smem_i, scratch, out);
}

// Small batches: top-k of every token and the permutation in one CTA.
__global__ void __launch_bounds__(1024) k_topk_permute_small(const float* __restrict__ logits, int T, int E,
                                                             int k, moe_routing_t out) {
  extern __shared__ int smem_i[];
  __shared__ int scratch[40];
  int* ids_s = smem_i + 32 * E;  // [T*k]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < T; t += 32) {
    const int id = warp_topk(logits + size_t(t) * E, E, k, t, out.topk_ids, out.topk_w);
    if (lane < k) ids_s[t * k + lane] = id;
  }
  __syncthreads();
  permute_block(ids_s, T * k, E, smem_i, scratch, out);
}

__global__ void k_select_bits(const float* __restrict__ w, int64_t n, float t0, float t1, float t2, uint8_t c0,
                              uint8_t c1, uint8_t c2, uint8_t c3, uint8_t* __restrict__ bits) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const float v = w[i];
  bits[i] = (v < t0) ? c0 : (v < t1) ? c1 : (v < t2) ? c2 : c3;
}

// ---------------------------------------------------------------- launchers
constexpr int kSmallT = 64;

size_t route_workspace_bytes(int64_t T, int64_t E, int64_t /*k*/) {
  return size_t(((T * E * 4) + 255) / 256 * 256);
}

cudaError_t launch_route(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H, int E, int k,
                         const moe_routing_t& out, void* ws, cudaStream_t st) {
  float* logits = static_cast<float*>(ws);
  if (T >= 256) {
    constexpr int WT = 4, WE = 4;
    dim3 grid((T + WT * kTileT - 1) / (WT * kTileT), (E + WE * kTileE - 1) / (WE * kTileE));
    k_router_logits<WT, WE><<<grid, 32 * WT * WE, 0, st>>>(x, wr, bias, T, H, E, logits);
  } else {
    dim3 grid((T + kTileT - 1) / kTileT, (E + kTileE - 1) / kTileE);
    k_router_logits<1, 1><<<grid, 32, 0, st>>>(x, wr, bias, T, H, E, logits);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int P = T * k;
  if (T <= kSmallT) {
    const size_t smem = size_t(32 * E + P) * sizeof(int);
    if (smem > 48 * 1024) {
      err = cudaFuncSetAttribute(k_topk_permute_small, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      if (err != cudaSuccess) return err;
    }
    k_topk_permute_small<<<1, 1024, smem, st>>>(logits, T, E, k, out);
    return cudaGetLastError();
  }
  k_topk<<<(T + 7) / 8, 256, 0, st>>>(logits, T, E, k, out.topk_ids, out.topk_w);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const size_t smem = size_t(32 * E) * sizeof(int);
  if (smem > 48 * 1024) {
    err = cudaFuncSetAttribute(k_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
  }
  k_permute<<<1, 1024, smem, st>>>(out.topk_ids, P, E, out);
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
