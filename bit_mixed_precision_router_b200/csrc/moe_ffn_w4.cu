// Grouped expert FFN for INT4 group-128 experts on the weight-streaming path (decode-sized
// expert groups): "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference",
// abstract (symmetric group-128 four-bit routed experts, all selected experts executed by
// fused grouped kernels).
//
// Three launches per call:
//   k_w4_stage     x bf16 [T][H] -> xq fp16 [T][H]: x/16 in MMA-fragment order (below);
//   k_w4_gemv<0>   gate/up: h = silu(x W_gate^T) * (x W_up^T) -> hq fp16 [P][I], h/16 in the
//                  same fragment order (the down GEMV's B operand);
//   k_w4_gemv<1>   down: y_rows bf16 [P][H] = h W2^T.
//
// k_w4_gemv is persistent: the work list is every (active expert, 16-row unit) pair, W =
// A * U units (A active experts, U = rows per expert / 16), and CTA b takes the contiguous
// units [b W / G, (b+1) W / G) of it (G = grid size), so the CTAs' shares differ by at most
// one unit and a CTA changes expert at most a few times.  A unit's 16 rows are
//   gate/up: rows 0..7 = gate rows 8u..8u+7, rows 8..15 = the up rows I+8u..I+8u+7 (one m16
//            MMA fragment holds gate and up of 8 intermediate rows: SwiGLU in the epilogue);
//   down:    rows 16u..16u+15.
// One CTA = one producer warp + eight consumer warps.  The producer streams each unit's
// weights in stages of 16 rows x 1024 K (512 bytes of packed INT4 per row) with bulk copies
// on the TMA engine (one 16-lane instruction per stage) into a 4-deep ring of shared-memory
// slots guarded by mbarriers; the unit's bf16 scales travel with its first stage.  Consumer
// warp w computes K-group 8s + w of stage s: two shared loads of packed weights, nibbles ->
// exact fp16 codes q = u - 8 in registers, mma.sync m16n8k16 against the activations (B
// operand, read from the staged copy through L1), fp32 accumulation, the group scale applied
// per group.  At the end of a unit the eight partial sums meet in shared memory and the
// epilogue writes h or y.  The producer runs up to four stages ahead, across unit and expert
// boundaries, so the weight stream does not stop during a unit's reduction.
//
// Nibble -> fp16: for a packed word w (element j of the word in nibble j),
//   (w & 0x000F000F) | 0x64006400 = fp16 (1024 + u0, 1024 + u4)  -> minus 1032 = (q0, q4)
//   (w & 0x00F000F0) | 0x64006400 = fp16 (1024 + 16 u1, 1024 + 16 u5) -> *1/16 - 72 = (q1, q5)
// and the same on w >> 8 for (q2, q6), (q3, q7): every result is an exact small integer.
// The activations of the word's eight elements are therefore staged as the fp16 pairs
// (x0, x4), (x1, x5), (x2, x6), (x3, x7), each scaled by 1/16 (exact for |x| in fp16's
// normal range; the factor is applied back in the epilogue).  Fragment order of a staged
// row: element k = 128 G + 32 c + 8 m + j sits in the 16-byte chunk (G, m, c) at byte
// G*256 + m*64 + c*16, so lane (g, c) of a warp reads 64 consecutive bytes per (G, m) with
// its three neighbours.
#include <atomic>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kRowsW4 = 16;                       // weight rows per unit
constexpr int kConsumerWarps = 8;
constexpr int kThreadsW4 = 32 * (kConsumerWarps + 1);
constexpr int kStageGroups = 8;                   // K-groups of 128 per stage
constexpr int kStageRowBytes = kStageGroups * 64; // packed INT4 bytes of one row per stage
constexpr int kRowPitch = kStageRowBytes + 64;    // rows g, g+1 start 64 bytes apart modulo 128:
                                                  // a quarter warp's 16-byte loads hit 8 distinct bank quads
constexpr int kDepthW4 = 4;                       // stages in flight
constexpr int kMaxGroups = 64;                    // K <= 8192
constexpr int kUnitScaleBytes = kRowsW4 * kMaxGroups * 2;
constexpr int kSlotBytes = kRowsW4 * kRowPitch + kUnitScaleBytes;  // weights + the unit's scales
constexpr int kRedFloats = kConsumerWarps * 2 * 32 * 4;           // partial sums of one unit
constexpr int kWarpScaleBytes = kRowsW4 * kStageGroups * 2;        // a warp's scales of one unit
constexpr size_t kSmemW4 = size_t(kDepthW4) * kSlotBytes + 2 * kRedFloats * 4 +
                           size_t(kConsumerWarps) * kWarpScaleBytes + 2 * kDepthW4 * 8;

enum { kModeGateUp = 0, kModeDown = 1 };

struct W4Args {
  const uint8_t* act;      // B operand rows, fp16 fragment order: xq [T][K] (gate/up) or hq [P][K] (down)
  const int32_t* expert_list;
  const int32_t* offsets;
  const int32_t* sorted_pair;
  const uint8_t* w;        // packed INT4 [E][N][K/8] words
  const uint8_t* s;        // bf16 scales [E][N][K/128]
  void* out;               // gate/up: hq fp16 [P][I]; down: y bf16 [P][H]
  unsigned* err;
  int K, N, I, k;
  int units;               // U = units per expert
};

MOE_DEVICE uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
MOE_DEVICE uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
MOE_DEVICE void mbar_arrive_cta(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
MOE_DEVICE void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumerWarps) : "memory"); }
// 16-byte global load kept in L1 (the staged activations: every unit of an expert reads them)
MOE_DEVICE uint4 ldg_l1_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::evict_last.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Expert-matrix row of unit row r.
MOE_DEVICE int unit_row(int mode, int u, int r, int I) {
  if (mode == kModeGateUp) return r < 8 ? 8 * u + r : I + 8 * u + r - 8;
  return kRowsW4 * u + r;
}

// One K-group (16 rows x 128) of the thread's slice: wa / wb = its 16 bytes of rows g and
// g+8 (32 K-elements, 4 words), xv[nt][m] = the staged activations of word m for token
// column g of tile nt.  Adds sa * (row g partial), sb * (row g+8 partial) to acc.
template <bool TWO>
MOE_DEVICE void w4_group(uint4 wa, uint4 wb, const uint4 (&xv)[2][4], float sa, float sb, float (&acc)[2][4]) {
  const uint32_t wa_[4] = {wa.x, wa.y, wa.z, wa.w};
  const uint32_t wb_[4] = {wb.x, wb.y, wb.z, wb.w};
  constexpr uint32_t kMagic = 0x64006400u;  // fp16 (1024, 1024)
  constexpr uint32_t kOff = 0x64086408u;    // fp16 (1032, 1032)
  constexpr uint32_t kSixteenth = 0x2C002C00u;  // fp16 (1/16, 1/16)
  constexpr uint32_t kMinus72 = 0xD480D480u;    // fp16 (-72, -72)
  constexpr int NT = TWO ? 2 : 1;
  float t[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) t[nt][i] = 0.f;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t ah = wa_[m] >> 8, bh = wb_[m] >> 8;
    const uint32_t qa0 = hsub2((wa_[m] & 0x000F000Fu) | kMagic, kOff);
    const uint32_t qa1 = hfma2((wa_[m] & 0x00F000F0u) | kMagic, kSixteenth, kMinus72);
    const uint32_t qa2 = hsub2((ah & 0x000F000Fu) | kMagic, kOff);
    const uint32_t qa3 = hfma2((ah & 0x00F000F0u) | kMagic, kSixteenth, kMinus72);
    const uint32_t qb0 = hsub2((wb_[m] & 0x000F000Fu) | kMagic, kOff);
    const uint32_t qb1 = hfma2((wb_[m] & 0x00F000F0u) | kMagic, kSixteenth, kMinus72);
    const uint32_t qb2 = hsub2((bh & 0x000F000Fu) | kMagic, kOff);
    const uint32_t qb3 = hfma2((bh & 0x00F000F0u) | kMagic, kSixteenth, kMinus72);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      mma_f16(t[nt], qa0, qb0, qa1, qb1, xv[nt][m].x, xv[nt][m].y);
      mma_f16(t[nt], qa2, qb2, qa3, qb3, xv[nt][m].z, xv[nt][m].w);
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    acc[nt][0] = fmaf(sa, t[nt][0], acc[nt][0]);
    acc[nt][1] = fmaf(sa, t[nt][1], acc[nt][1]);
    acc[nt][2] = fmaf(sb, t[nt][2], acc[nt][2]);
    acc[nt][3] = fmaf(sb, t[nt][3], acc[nt][3]);
  }
}

// The work item (unit) the CTA handles at list position i.
struct Unit {
  int e, u, row0, n_e;
};
MOE_DEVICE Unit unit_at(const W4Args& a, int64_t i) {
  const int slot = int(i / a.units);
  Unit r;
  r.u = int(i - int64_t(slot) * a.units);
  r.e = a.expert_list[1 + slot];
  r.row0 = a.offsets[r.e];
  r.n_e = a.offsets[r.e + 1] - r.row0;
  return r;
}

template <int MODE>
__global__ void __launch_bounds__(kThreadsW4, 2) k_w4_gemv(W4Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* slots = smem;
  float* red = reinterpret_cast<float*>(smem + size_t(kDepthW4) * kSlotBytes);
  uint8_t* wscale = reinterpret_cast<uint8_t*>(red + 2 * kRedFloats);
  uint64_t* full = reinterpret_cast<uint64_t*>(wscale + kConsumerWarps * kWarpScaleBytes);
  uint64_t* empty = full + kDepthW4;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K, GK = K / 128, S = (GK + kStageGroups - 1) / kStageGroups;
  const int64_t W = int64_t(a.expert_list[0]) * a.units;
  const int64_t i0 = int64_t(blockIdx.x) * W / gridDim.x, i1 = int64_t(blockIdx.x + 1) * W / gridDim.x;
  const size_t row_bytes = size_t(K) / 2;
  const size_t scale_row_bytes = size_t(GK) * 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDepthW4; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer warp
    uint32_t it = 0;
    bool ok = true;
    for (int64_t i = i0; i < i1 && ok; ++i) {
      const Unit un = unit_at(a, i);
      const int nch = (un.n_e + 15) / 16;
      const uint8_t* wrow = a.w + (size_t(un.e) * a.N + unit_row(MODE, un.u, lane & 15, a.I)) * row_bytes;
      for (int ch = 0; ch < nch && ok; ++ch) {
        for (int s = 0; s < S; ++s, ++it) {
          const int slot = int(it % kDepthW4);
          if (it >= kDepthW4) {
            ok = mbar_wait(&empty[slot], (it / kDepthW4 - 1) & 1, a.err);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
          }
          const int ng = min(kStageGroups, GK - s * kStageGroups);
          const bool with_scales = (s == 0 && ch == 0);
          const uint32_t bytes = uint32_t(kRowsW4 * ng * 64) + (with_scales ? uint32_t(kRowsW4 * scale_row_bytes) : 0u);
          uint8_t* dst = slots + size_t(slot) * kSlotBytes;
          if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
          __syncwarp();
          if (lane < kRowsW4) {
            bulk_g2s(dst + lane * kRowPitch, wrow + size_t(s) * kStageRowBytes, uint32_t(ng * 64), &full[slot]);
          } else if (with_scales && lane < kRowsW4 + (MODE == kModeGateUp ? 2 : 1)) {
            // the unit's scales: rows of the unit in order (gate/up: two runs of 8 rows)
            const int half = lane - kRowsW4;
            const int nrows = MODE == kModeGateUp ? 8 : 16;
            const size_t src_row = size_t(un.e) * a.N + unit_row(MODE, un.u, 8 * half, a.I);
            bulk_g2s(dst + kRowsW4 * kRowPitch + size_t(8 * half) * scale_row_bytes, a.s + src_row * scale_row_bytes,
                     uint32_t(nrows * scale_row_bytes), &full[slot]);
          }
        }
      }
    }
    // drain: on a normal exit every issued stage was consumed; after a timeout, wait (bounded)
    // for the copies still in flight so none lands after the CTA exits
    if (!ok && lane == 0) {
      const uint32_t n = it < kDepthW4 ? it : kDepthW4;
      for (uint32_t j = 0; j < n; ++j) {
        const uint32_t st = it - 1 - j;
        mbar_wait(&full[st % kDepthW4], (st / kDepthW4) & 1, a.err);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumer warps
  const int g = lane >> 2, c = lane & 3;
  uint8_t* my_scales = wscale + warp * kWarpScaleBytes;  // [16 rows][stage s] bf16
  uint32_t it = 0;
  int buf = 0;
  bool ok = true;
  for (int64_t i = i0; i < i1; ++i) {
    const Unit un = unit_at(a, i);
    const int nch = (un.n_e + 15) / 16;
    for (int ch = 0; ch < nch; ++ch) {
      const int nvalid = min(16, un.n_e - 16 * ch);
      const bool two = nvalid > 8;
      // B rows of this chunk's token columns g and 8 + g (an absent column reads a valid
      // row: each output column depends only on its own B column)
      const uint8_t* brow[2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int r = un.row0 + 16 * ch + min(nt * 8 + g, nvalid - 1);
        const size_t arow = MODE == kModeGateUp ? size_t(a.sorted_pair[r] / a.k) : size_t(r);
        brow[nt] = a.act + arow * size_t(K) * 2 + c * 16;
      }
      float acc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[nt][q] = 0.f;
      for (int s = 0; s < S; ++s, ++it) {
        const int slot = int(it % kDepthW4);
        const uint8_t* src = slots + size_t(slot) * kSlotBytes;
        const int G = s * kStageGroups + warp;
        // activations of this warp's group, issued before the wait (they do not depend on it)
        uint4 xv[2][4];
        if (G < GK) {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            if (nt == 1 && !two) break;
#pragma unroll
            for (int m = 0; m < 4; ++m) xv[nt][m] = ldg_l1_v4(brow[nt] + G * 256 + m * 64);
          }
        }
        if (ok) {
          ok = mbar_wait(&full[slot], (it / kDepthW4) & 1, a.err);
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        if (s == 0 && ch == 0) {
          // this warp's scales of the unit: rows 0..15, groups warp, warp + 8, ... (<= 8)
          const uint16_t* us = reinterpret_cast<const uint16_t*>(src + kRowsW4 * kRowPitch);
          for (int q = lane; q < kRowsW4 * S; q += 32) {
            const int r = q / S, ss = q - r * S, GG = ss * kStageGroups + warp;
            reinterpret_cast<uint16_t*>(my_scales)[r * kStageGroups + ss] = GG < GK ? us[r * GK + GG] : 0;
          }
          __syncwarp();
        }
        if (G < GK) {
          const uint4 wa = *reinterpret_cast<const uint4*>(src + g * kRowPitch + warp * 64 + c * 16);
          const uint4 wb = *reinterpret_cast<const uint4*>(src + (g + 8) * kRowPitch + warp * 64 + c * 16);
          const uint16_t* ms = reinterpret_cast<const uint16_t*>(my_scales);
          const float sa = bf16_bits_to_float(ms[g * kStageGroups + s]);
          const float sb = bf16_bits_to_float(ms[(g + 8) * kStageGroups + s]);
          if (two)
            w4_group<true>(wa, wb, xv, sa, sb, acc);
          else
            w4_group<false>(wa, wb, xv, sa, sb, acc);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cta(&empty[slot]);
      }
      // ---- the eight warps' partial sums -> one unit result
      float4* rp = reinterpret_cast<float4*>(red + buf * kRedFloats) + warp * 64;
      rp[lane] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
      rp[32 + lane] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
      consumer_sync();
      const float* rb = red + buf * kRedFloats;
      const int tid = threadIdx.x;
      if (MODE == kModeGateUp) {
        if (tid < 128) {
          // (tile nt, lane l, column jj): gate = entry jj, up = entry 2 + jj
          const int nt = tid >> 6, l = (tid >> 1) & 31, jj = tid & 1;
          const int gg = l >> 2, cc = l & 3, n = nt * 8 + 2 * cc + jj;
          float gate = 0.f, up = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            gate += rb[(w * 64 + nt * 32 + l) * 4 + jj];
            up += rb[(w * 64 + nt * 32 + l) * 4 + 2 + jj];
          }
          if (n < nvalid) {
            const float h = silu(gate * 16.f) * (up * 16.f);
            // intermediate index 8u + gg: chunk (G, m, c) of the row, half 2 (gg % 4) + gg / 4
            const int uu = un.u, GG = uu >> 4, cq = (uu >> 2) & 3, mq = uu & 3;
            const size_t off = size_t(un.row0 + 16 * ch + n) * size_t(a.I) * 2 + GG * 256 + mq * 64 + cq * 16 +
                               (2 * (gg & 3) + (gg >> 2)) * 2;
            *reinterpret_cast<__half*>(static_cast<uint8_t*>(a.out) + off) = __float2half_rn(h * 0.0625f);
          }
        }
      } else {
        // (tile nt, lane l, entry q): row 16u + gg (+8 for q >= 2), column 2cc + (q & 1)
        const int nt = tid >> 7, l = (tid >> 2) & 31, q = tid & 3;
        const int gg = l >> 2, cc = l & 3, n = nt * 8 + 2 * cc + (q & 1);
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) v += rb[(w * 64 + nt * 32 + l) * 4 + q];
        if (n < nvalid) {
          const int col = kRowsW4 * un.u + gg + (q >= 2 ? 8 : 0);
          static_cast<uint16_t*>(a.out)[size_t(un.row0 + 16 * ch + n) * size_t(a.N) + col] =
              float_to_bf16_bits(v * 16.f);
        }
      }
      buf ^= 1;
    }
  }
}

// x bf16 [T][K] -> xq fp16 [T][K], x/16 in fragment order; one thread per 8 elements.
__global__ void k_w4_stage(const uint4* __restrict__ x, int64_t n8, int K8, uint4* __restrict__ xq) {
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= n8) return;
  const int64_t t = i / K8;
  const int q = int(i - t * K8);  // 8-element chunk of the row: G = q / 16, c = (q / 4) % 4, m = q % 4
  const uint4 v = x[i];
  const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                      bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const __half2 h = __floats2half2_rn(f[p] * 0.0625f, f[p + 4] * 0.0625f);
    o[p] = *reinterpret_cast<const uint32_t*>(&h);
  }
  const int G = q >> 4, cq = (q >> 2) & 3, mq = q & 3;
  xq[t * K8 + G * 16 + mq * 4 + cq] = make_uint4(o[0], o[1], o[2], o[3]);
}

int sm_count() {
  static std::atomic<int> cached[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int MODE>
cudaError_t launch_w4_mode(const W4Args& a, int max_units, cudaStream_t st) {
  static std::atomic<bool> raised[128] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!raised[dev].load(std::memory_order_relaxed)) {
    err = cudaFuncSetAttribute(k_w4_gemv<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemW4));
    if (err != cudaSuccess) return err;
    raised[dev].store(true, std::memory_order_relaxed);
  }
  int grid = 2 * sm_count();
  if (grid > max_units) grid = max_units;
  if (grid < 1) grid = 1;
  k_w4_gemv<MODE><<<grid, kThreadsW4, kSmemW4, st>>>(a);
  return cudaGetLastError();
}

size_t align256w(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

bool w4_gemv_shape_supported(int64_t H, int64_t I) {
  return H % 128 == 0 && I % 128 == 0 && H / 128 <= kMaxGroups && I / 128 <= kMaxGroups;
}

size_t w4_gemv_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t k) {
  return align256w(size_t(T) * H * 2) + align256w(size_t(T) * k * I * 2);
}

cudaError_t launch_w4_gemv(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex, int T, int H, int I,
                           int E, int k, uint16_t* y_rows, void* ws, cudaStream_t st) {
  unsigned* err = device_error_word();
  if (!err) return cudaErrorUnknown;
  uint8_t* xq = static_cast<uint8_t*>(ws);
  uint8_t* hq = xq + align256w(size_t(T) * H * 2);
  const int64_t n8 = int64_t(T) * H / 8;
  k_w4_stage<<<unsigned((n8 + 255) / 256), 256, 0, st>>>(reinterpret_cast<const uint4*>(x), n8, H / 8,
                                                         reinterpret_cast<uint4*>(xq));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int P = T * k;
  const int max_experts = P < E ? P : E;
  W4Args a{};
  a.expert_list = r.expert_list;
  a.offsets = r.expert_offsets;
  a.sorted_pair = r.sorted_pair;
  a.err = err;
  a.I = I;
  a.k = k;
  // gate/up
  a.act = xq;
  a.w = static_cast<const uint8_t*>(ex.w13);
  a.s = static_cast<const uint8_t*>(ex.w13_scale);
  a.out = hq;
  a.K = H;
  a.N = 2 * I;
  a.units = I / 8;
  e = launch_w4_mode<kModeGateUp>(a, max_experts * a.units, st);
  if (e != cudaSuccess) return e;
  // down
  a.act = hq;
  a.w = static_cast<const uint8_t*>(ex.w2);
  a.s = static_cast<const uint8_t*>(ex.w2_scale);
  a.out = y_rows;
  a.K = I;
  a.N = H;
  a.units = H / kRowsW4;
  return launch_w4_mode<kModeDown>(a, max_experts * a.units, st);
}

}  // namespace moe
