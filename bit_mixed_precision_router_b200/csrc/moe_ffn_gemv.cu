// Grouped expert FFN, weight-streaming path (decode-sized expert groups).
//
// One CTA = one routed expert x one tile of 16 weight rows, full K:
//   gate/up: smem rows 0..7 = gate rows 8t..8t+7, rows 8..15 = the matching up rows,
//            so one m16 MMA fragment yields gate and up of 8 intermediate rows and
//            SwiGLU is applied in the epilogue;
//   down:    smem rows 0..15 = down rows 16t..16t+15.
// Warp 0 issues one bulk copy (TMA engine) per weight row (per plane for the
// bitplane format) into padded shared memory, so the whole tile is in flight at
// once; the 4 warps split K, dequantise in registers and feed mma.sync with the
// expert's tokens on the MMA's N dimension (16 per pass); partial sums meet in
// shared memory in a fixed warp order.  Expert weights are read once per CTA no
// matter how many tokens the expert received.
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

enum { kGateUp = 0, kDown = 1 };
constexpr int kRows = 16;    // weight rows per CTA
constexpr int kWarps = 4;    // K split
constexpr int kChunk = 16;   // tokens per pass (two n8 tiles)

struct FfnArgs {
  const void* act;  // gate/up: x [T][K] (bf16, or fp16*2^-8 for NVFP4); down: h [P][K]
  int K;            // reduction length: H (gate/up) or I (down)
  int N;            // rows per expert matrix: 2I or H
  int I;
  int k;
  const int32_t* expert_list;
  const int32_t* offsets;
  const int32_t* sorted_pair;
  const uint8_t* bits;  // bitplane: per pair
  const void* w;
  const void* s;
  const float* gscale;  // NVFP4
  void* out;            // gate/up: h [P][I]; down: y [P][H]
  int out_ld;
  unsigned* err;
};

// Row stride (bytes) of a K-contiguous weight row of `row_bytes` in shared memory,
// padded so that the 16-byte (W4/NVFP4) or 4-byte (bitplane) loads of the 32 lanes
// hit distinct banks.
__host__ __device__ inline int smem_stride_16B(int row_bytes) {
  // row_bytes / 16 is a multiple of 4; make the stride / 16 an odd multiple of 4 (mod 8 == 4)
  return ((row_bytes / 16) % 8 == 4) ? row_bytes : row_bytes + 64;
}
__host__ __device__ inline int smem_stride_4B(int row_bytes) {
  // stride / 4 must be 4 * odd (mod 32 in {4, 12, 20, 28})
  return (((row_bytes / 16) & 1) == 1) ? row_bytes : row_bytes + 16;
}

template <int FMT>
__host__ __device__ inline int weight_row_bytes(int K) {
  return FMT == MOE_FMT_BITPLANE8 ? K / 8 : K / 2;
}
template <int FMT>
__host__ __device__ inline int weight_stride(int K) {
  return FMT == MOE_FMT_BITPLANE8 ? smem_stride_4B(K / 8) : smem_stride_16B(K / 2);
}
template <int FMT>
__host__ inline size_t ffn_smem_bytes(int K) {
  const int planes = FMT == MOE_FMT_BITPLANE8 ? 8 : 1;
  return size_t(planes) * kRows * weight_stride<FMT>(K);
}

// ---------------------------------------------------------------- group steps
// Every step handles one group of 128 K-elements for the thread's 32-element slice
// (lane = 4g + c owns K-elements 32c .. 32c+31 of the group) of smem rows g and
// g+8, for up to two n8 tiles of tokens whose activation slices are in xv[nt][0..3].

// INT4: word m of the slice holds elements 8m .. 8m+7.  Nibbles j and j+4 are
// lifted into one bf16x2 as 128 + u (exponent of 128, nibble in the low mantissa
// bits); the MMA therefore sums (q + 136) * x and a second MMA with A = 136
// removes the offset.  The activations are paired (j, j+4) to match.
MOE_DEVICE void w4_group(const uint8_t* rowA, const uint8_t* rowB, const uint4 (&xv)[2][4], bool two, float sa,
                         float sb, float (&acc)[2][4]) {
  const uint4 wa = *reinterpret_cast<const uint4*>(rowA);
  const uint4 wb = *reinterpret_cast<const uint4*>(rowB);
  const uint32_t wa_[4] = {wa.x, wa.y, wa.z, wa.w};
  const uint32_t wb_[4] = {wb.x, wb.y, wb.z, wb.w};
  constexpr uint32_t kMagic = 0x43004300u;  // bf16 (128, 128)
  constexpr uint32_t kOff = 0x43084308u;    // bf16 (136, 136)
  float tmp[2][4], corr[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) tmp[nt][i] = corr[nt][i] = 0.f;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    uint32_t pa[4], pb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      pa[j] = ((wa_[m] >> (4 * j)) & 0x000F000Fu) | kMagic;
      pb[j] = ((wb_[m] >> (4 * j)) & 0x000F000Fu) | kMagic;
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      if (nt == 1 && !two) break;
      const uint4 xx = xv[nt][m];
      const uint32_t b00 = __byte_perm(xx.x, xx.z, 0x5410), b01 = __byte_perm(xx.x, xx.z, 0x7632);
      const uint32_t b10 = __byte_perm(xx.y, xx.w, 0x5410), b11 = __byte_perm(xx.y, xx.w, 0x7632);
      mma_bf16(tmp[nt], pa[0], pb[0], pa[1], pb[1], b00, b01);
      mma_bf16(tmp[nt], pa[2], pb[2], pa[3], pb[3], b10, b11);
      mma_bf16(corr[nt], kOff, kOff, kOff, kOff, b00, b01);
      mma_bf16(corr[nt], kOff, kOff, kOff, kOff, b10, b11);
    }
  }
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    acc[nt][0] = fmaf(sa, tmp[nt][0] - corr[nt][0], acc[nt][0]);
    acc[nt][1] = fmaf(sa, tmp[nt][1] - corr[nt][1], acc[nt][1]);
    acc[nt][2] = fmaf(sb, tmp[nt][2] - corr[nt][2], acc[nt][2]);
    acc[nt][3] = fmaf(sb, tmp[nt][3] - corr[nt][3], acc[nt][3]);
  }
}

// Bitplanes: plane word bit j <-> element j of the 32-element slice.  Bits j and
// j+16 are moved to bit 7 / 23 of a bf16x2 whose other bits spell 0.5, giving
// A = 0.5 + 0.5 * bit; activations are paired (j, j+16).  For token t read at
// b_t planes the group contributes
//   sum_{p < b_t} 2^(8-p) * T_p + (c_b + 2^(8-b) - 384) * X,
// with T_p the plane-p MMA sum and X = sum of the activations over the slice
// (an MMA with A = 1), which equals sum_k (u'_k - 128) x_k.
MOE_DEVICE uint32_t bit_pair(uint32_t w, int j) {
  const uint32_t s = (j <= 7) ? (w << (7 - j)) : (w >> (j - 7));
  return (s & 0x00800080u) | 0x3F003F00u;
}
MOE_DEVICE float plane_coef_x(int b) {  // c_b + 2^(8-b) - 384
  return (b >= 8) ? -383.f : float(3 * (1 << (7 - b)) - 384);
}

MOE_DEVICE void bp_group(const uint8_t* base, int stride, int G, int g, int c, int nplanes,
                         const uint4 (&xv)[2][4], bool two, const int (&bt)[2][2], float sa, float sb,
                         float (&acc)[2][4]) {
  uint32_t R[2][16];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const uint32_t* q = reinterpret_cast<const uint32_t*>(&xv[nt][0]);
#pragma unroll
    for (int i = 0; i < 16; ++i) R[nt][i] = q[i];
  }
  constexpr uint32_t kOne = 0x3F803F80u;
  float X[2][4], grp[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) X[nt][i] = grp[nt][i] = 0.f;
  // X = sum of activations (plane independent)
#pragma unroll
  for (int s = 0; s < 8; ++s) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      if (nt == 1 && !two) break;
      const uint32_t b0 = __byte_perm(R[nt][s], R[nt][s + 8], 0x5410);
      const uint32_t b1 = __byte_perm(R[nt][s], R[nt][s + 8], 0x7632);
      mma_bf16(X[nt], kOne, kOne, kOne, kOne, b0, b1);
    }
  }
  for (int p = 0; p < nplanes; ++p) {
    const uint8_t* pr = base + (p * kRows + g) * stride + G * 16 + c * 4;
    const uint32_t wa = *reinterpret_cast<const uint32_t*>(pr);
    const uint32_t wb = *reinterpret_cast<const uint32_t*>(pr + 8 * stride);
    float tp[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) tp[nt][i] = 0.f;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t a0 = bit_pair(wa, 2 * s), a2 = bit_pair(wa, 2 * s + 1);
      const uint32_t a1 = bit_pair(wb, 2 * s), a3 = bit_pair(wb, 2 * s + 1);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        if (nt == 1 && !two) break;
        const uint32_t b0 = __byte_perm(R[nt][s], R[nt][s + 8], 0x5410);
        const uint32_t b1 = __byte_perm(R[nt][s], R[nt][s + 8], 0x7632);
        mma_bf16(tp[nt], a0, a1, a2, a3, b0, b1);
      }
    }
    const float f = float(1 << (8 - p));
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float f0 = (p < bt[nt][0]) ? f : 0.f, f1 = (p < bt[nt][1]) ? f : 0.f;
      grp[nt][0] = fmaf(f0, tp[nt][0], grp[nt][0]);
      grp[nt][1] = fmaf(f1, tp[nt][1], grp[nt][1]);
      grp[nt][2] = fmaf(f0, tp[nt][2], grp[nt][2]);
      grp[nt][3] = fmaf(f1, tp[nt][3], grp[nt][3]);
    }
  }
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const float x0 = plane_coef_x(bt[nt][0]), x1 = plane_coef_x(bt[nt][1]);
    acc[nt][0] = fmaf(sa, fmaf(x0, X[nt][0], grp[nt][0]), acc[nt][0]);
    acc[nt][1] = fmaf(sa, fmaf(x1, X[nt][1], grp[nt][1]), acc[nt][1]);
    acc[nt][2] = fmaf(sb, fmaf(x0, X[nt][2], grp[nt][2]), acc[nt][2]);
    acc[nt][3] = fmaf(sb, fmaf(x1, X[nt][3], grp[nt][3]), acc[nt][3]);
  }
}

// NVFP4: byte i of a word holds elements 2i (low nibble) and 2i+1; each byte is
// converted to an fp16 pair and multiplied by its E4M3 block scale (exact in fp16);
// activations are fp16 (pre-scaled by 2^-8) in natural pairs.
MOE_DEVICE uint32_t e2m1x2_to_h2(uint32_t byte) {
  const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
  return uint32_t(r.x) | (uint32_t(r.y) << 16);
}
MOE_DEVICE uint32_t e4m3_to_h2(uint32_t byte) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(byte), __NV_E4M3);
  return uint32_t(h.x) | (uint32_t(h.x) << 16);
}
MOE_DEVICE uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

MOE_DEVICE void fp4_group(const uint8_t* rowA, const uint8_t* rowB, uint32_t scA, uint32_t scB,
                          const uint4 (&xv)[2][4], bool two, float (&acc)[2][4]) {
  const uint4 wa = *reinterpret_cast<const uint4*>(rowA);
  const uint4 wb = *reinterpret_cast<const uint4*>(rowB);
  const uint32_t wa_[4] = {wa.x, wa.y, wa.z, wa.w};
  const uint32_t wb_[4] = {wb.x, wb.y, wb.z, wb.w};
  // block scales: words 0,1 -> block 2c (byte 0 of sc), words 2,3 -> block 2c+1 (byte 1)
  const uint32_t sA[2] = {e4m3_to_h2(scA & 0xFF), e4m3_to_h2((scA >> 8) & 0xFF)};
  const uint32_t sB[2] = {e4m3_to_h2(scB & 0xFF), e4m3_to_h2((scB >> 8) & 0xFF)};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    uint32_t ha[4], hb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ha[i] = hmul2(e2m1x2_to_h2((wa_[m] >> (8 * i)) & 0xFF), sA[m >> 1]);
      hb[i] = hmul2(e2m1x2_to_h2((wb_[m] >> (8 * i)) & 0xFF), sB[m >> 1]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      if (nt == 1 && !two) break;
      const uint4 xx = xv[nt][m];
      mma_f16(acc[nt], ha[0], hb[0], ha[1], hb[1], xx.x, xx.y);
      mma_f16(acc[nt], ha[2], hb[2], ha[3], hb[3], xx.z, xx.w);
    }
  }
}

// ---------------------------------------------------------------- kernel
template <int FMT, int MODE>
__global__ void __launch_bounds__(32 * kWarps) k_ffn_gemv(FfnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bar;
  __shared__ float red[kWarps][2][32][4];
  __shared__ int s_bmax;

  const int slot = blockIdx.y;
  if (slot >= a.expert_list[0]) return;
  const int e = a.expert_list[1 + slot];
  const int row0 = a.offsets[e];
  const int n_e = a.offsets[e + 1] - row0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int K = a.K;
  const int stride = weight_stride<FMT>(K);
  const int row_bytes = weight_row_bytes<FMT>(K);

  // expert-matrix row of smem row i
  auto wrow = [&](int i) -> int {
    if (MODE == kGateUp) return (i < 8) ? (8 * blockIdx.x + i) : (a.I + 8 * blockIdx.x + i - 8);
    return kRows * blockIdx.x + i;
  };

  int nplanes = 1;
  if (FMT == MOE_FMT_BITPLANE8) {
    int bm = 1;
    for (int n = threadIdx.x; n < n_e; n += blockDim.x) bm = max(bm, int(a.bits[a.sorted_pair[row0 + n]]));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) bm = max(bm, __shfl_xor_sync(0xffffffffu, bm, off));
    if (threadIdx.x == 0) s_bmax = 1;
    __syncthreads();
    if (lane == 0) atomicMax(&s_bmax, bm);
    __syncthreads();
    nplanes = min(8, s_bmax);
  }

  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(&bar, uint32_t(nplanes * kRows * row_bytes));
    __syncwarp();
    for (int q = lane; q < nplanes * kRows; q += 32) {
      const int i = q % kRows, pl = q / kRows;
      const uint8_t* src;
      if (FMT == MOE_FMT_BITPLANE8)
        src = static_cast<const uint8_t*>(a.w) + ((size_t(e) * 8 + pl) * a.N + wrow(i)) * size_t(row_bytes);
      else
        src = static_cast<const uint8_t*>(a.w) + (size_t(e) * a.N + wrow(i)) * size_t(row_bytes);
      bulk_g2s(smem + (pl * kRows + i) * stride, src, uint32_t(row_bytes), &bar);
    }
  }

  const int Gtot = K / 128;
  const int gpw = (Gtot + kWarps - 1) / kWarps;
  const int gb = min(Gtot, warp * gpw), ge = min(Gtot, gb + gpw);
  const int rA = wrow(g), rB = wrow(g + 8);

  const bool ok = mbar_wait(&bar, 0, a.err);
  if (!__syncthreads_and(ok)) return;

  for (int n0 = 0; n0 < n_e; n0 += kChunk) {
    const bool two = (n_e - n0) > 8;
    // B operand rows: token column g of each n8 tile
    const uint8_t* arow[2];
    int bt[2][2] = {{8, 8}, {8, 8}};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int n = n0 + nt * 8 + g;
      arow[nt] = nullptr;
      if (n < n_e) {
        const int r = row0 + n;
        const int arow_idx = (MODE == kGateUp) ? a.sorted_pair[r] / a.k : r;
        arow[nt] = static_cast<const uint8_t*>(a.act) + size_t(arow_idx) * K * 2;
      }
      if (FMT == MOE_FMT_BITPLANE8) {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int nn = n0 + nt * 8 + 2 * c + jj;
          bt[nt][jj] = (nn < n_e) ? int(a.bits[a.sorted_pair[row0 + nn]]) : 8;
        }
      }
    }
    auto load_x = [&](uint4 (&xv)[2][4], int G) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int m = 0; m < 4; ++m)
          xv[nt][m] = arow[nt] ? *reinterpret_cast<const uint4*>(arow[nt] + (size_t(G) * 128 + c * 32 + m * 8) * 2)
                               : make_uint4(0, 0, 0, 0);
    };

    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

    uint4 xc[2][4], xn[2][4];
    if (gb < ge) load_x(xc, gb);
    for (int G = gb; G < ge; ++G) {
      if (G + 1 < ge) load_x(xn, G + 1);
      if (FMT == MOE_FMT_W4G128) {
        const uint16_t* s = static_cast<const uint16_t*>(a.s);
        const float sa = bf16_bits_to_float(s[(size_t(e) * a.N + rA) * Gtot + G]);
        const float sb = bf16_bits_to_float(s[(size_t(e) * a.N + rB) * Gtot + G]);
        const uint8_t* rowA = smem + g * stride + G * 64 + c * 16;
        w4_group(rowA, rowA + 8 * stride, xc, two, sa, sb, acc);
      } else if (FMT == MOE_FMT_BITPLANE8) {
        const uint16_t* s = static_cast<const uint16_t*>(a.s);
        const float sa = bf16_bits_to_float(s[(size_t(e) * a.N + rA) * Gtot + G]);
        const float sb = bf16_bits_to_float(s[(size_t(e) * a.N + rB) * Gtot + G]);
        bp_group(smem, stride, G, g, c, nplanes, xc, two, bt, sa, sb, acc);
      } else {
        const uint8_t* s = static_cast<const uint8_t*>(a.s);
        const size_t spr = size_t(K / 16);
        const uint32_t scA = *reinterpret_cast<const uint16_t*>(s + (size_t(e) * a.N + rA) * spr + G * 8 + 2 * c);
        const uint32_t scB = *reinterpret_cast<const uint16_t*>(s + (size_t(e) * a.N + rB) * spr + G * 8 + 2 * c);
        const uint8_t* rowA = smem + g * stride + G * 64 + c * 16;
        fp4_group(rowA, rowA + 8 * stride, scA, scB, xc, two, acc);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int m = 0; m < 4; ++m) xc[nt][m] = xn[nt][m];
    }

#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][nt][lane][i] = acc[nt][i];
    __syncthreads();
    if (warp == 0) {
      float post = 1.f;
      if (FMT == MOE_FMT_NVFP4) post = a.gscale[e] * 256.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float sacc = red[0][nt][lane][i];
#pragma unroll
          for (int ww = 1; ww < kWarps; ++ww) sacc += red[ww][nt][lane][i];
          v[i] = sacc * post;
        }
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int n = n0 + nt * 8 + 2 * c + jj;
          if (n >= n_e) continue;
          const size_t orow = size_t(row0 + n) * a.out_ld;
          if (MODE == kGateUp) {
            const float h = silu(v[jj]) * v[2 + jj];
            const int col = 8 * blockIdx.x + g;
            if (FMT == MOE_FMT_NVFP4)
              static_cast<__half*>(a.out)[orow + col] = __float2half_rn(h * (1.0f / 256.f));
            else
              static_cast<uint16_t*>(a.out)[orow + col] = float_to_bf16_bits(h);
          } else {
            uint16_t* y = static_cast<uint16_t*>(a.out);
            y[orow + kRows * blockIdx.x + g] = float_to_bf16_bits(v[jj]);
            y[orow + kRows * blockIdx.x + g + 8] = float_to_bf16_bits(v[2 + jj]);
          }
        }
      }
    }
    __syncthreads();
  }
}

// x (bf16) -> fp16 * 2^-8 for the NVFP4 path (exact for |x| in [2^-6, 1.6e7]).
__global__ void k_to_f16_scaled(const uint16_t* __restrict__ x, int64_t n, __half* __restrict__ y) {
  const int64_t i = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) * 2;
  if (i >= n) return;
  const uint32_t v = *reinterpret_cast<const uint32_t*>(x + i);
  *reinterpret_cast<__half2*>(y + i) = __floats2half2_rn(bf16_lo(v) * (1.0f / 256.f), bf16_hi(v) * (1.0f / 256.f));
}

// ---------------------------------------------------------------- launchers
static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

size_t ffn_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t /*E*/, int64_t k, moe_format_t fmt) {
  size_t b = align256(size_t(T * k * I * 2));  // h
  if (fmt == MOE_FMT_NVFP4) b += align256(size_t(T * H * 2));  // x as fp16
  return b;
}

template <int FMT, int MODE>
static cudaError_t launch_one(const FfnArgs& a, int tiles, int slots, cudaStream_t st) {
  const size_t smem = ffn_smem_bytes<FMT>(a.K);
  if (smem > 48 * 1024) {
    cudaError_t err =
        cudaFuncSetAttribute(k_ffn_gemv<FMT, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
  }
  k_ffn_gemv<FMT, MODE><<<dim3(unsigned(tiles), unsigned(slots)), 32 * kWarps, smem, st>>>(a);
  return cudaGetLastError();
}

template <int FMT>
static cudaError_t launch_fmt(const void* act_x, const moe_routing_t& r, const moe_experts_t& ex,
                              const uint8_t* bits, int T, int H, int I, int E, int k, uint16_t* y_rows,
                              void* hbuf, cudaStream_t st) {
  const int P = T * k;
  const int slots = P < E ? P : E;
  FfnArgs a{};
  a.k = k;
  a.I = I;
  a.expert_list = r.expert_list;
  a.offsets = r.expert_offsets;
  a.sorted_pair = r.sorted_pair;
  a.bits = bits;
  a.err = device_error_word();
  // gate/up
  a.act = act_x;
  a.K = H;
  a.N = 2 * I;
  a.w = ex.w13;
  a.s = ex.w13_scale;
  a.gscale = ex.w13_gscale;
  a.out = hbuf;
  a.out_ld = I;
  cudaError_t err = launch_one<FMT, kGateUp>(a, I / 8, slots, st);
  if (err != cudaSuccess) return err;
  // down
  a.act = hbuf;
  a.K = I;
  a.N = H;
  a.w = ex.w2;
  a.s = ex.w2_scale;
  a.gscale = ex.w2_gscale;
  a.out = y_rows;
  a.out_ld = H;
  return launch_one<FMT, kDown>(a, H / kRows, slots, st);
}

cudaError_t launch_grouped_ffn(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex,
                               const uint8_t* bits, int T, int H, int I, int E, int k, uint16_t* y_rows,
                               void* ws, cudaStream_t st) {
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  void* hbuf = w8;
  switch (ex.fmt) {
    case MOE_FMT_W4G128:
      return launch_fmt<MOE_FMT_W4G128>(x, r, ex, bits, T, H, I, E, k, y_rows, hbuf, st);
    case MOE_FMT_BITPLANE8:
      return launch_fmt<MOE_FMT_BITPLANE8>(x, r, ex, bits, T, H, I, E, k, y_rows, hbuf, st);
    case MOE_FMT_NVFP4: {
      __half* x16 = reinterpret_cast<__half*>(w8 + align256(size_t(T) * k * I * 2));
      const int64_t n = int64_t(T) * H;
      k_to_f16_scaled<<<dim3(unsigned((n / 2 + 255) / 256)), 256, 0, st>>>(x, n, x16);
      cudaError_t err = cudaGetLastError();
      if (err != cudaSuccess) return err;
      return launch_fmt<MOE_FMT_NVFP4>(x16, r, ex, bits, T, H, I, E, k, y_rows, hbuf, st);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
