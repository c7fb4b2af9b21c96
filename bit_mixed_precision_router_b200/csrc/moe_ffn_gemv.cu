// Grouped expert FFN, weight-streaming path (decode-sized expert groups).
//
// Work: every routed expert's weight matrix is cut into units of 16 rows x full K
//   gate/up: rows 0..7 = gate rows 8t..8t+7, rows 8..15 = the matching up rows (one m16
//            MMA fragment gives gate and up of 8 intermediate rows, so SwiGLU runs in
//            the epilogue);
//   down:    rows 0..15 = down rows 16t..16t+15.
// One CTA = one routed expert x 4 warps, each warp owning one 16-row unit; four CTAs per
// SM (small CTAs start at different times, so one CTA staging its tokens overlaps the
// other CTAs' weight streams).  Wide rows (K = 7168: one staged token row fits a 4-warp
// CTA's budget) take one CTA of 16 warps per SM instead, whose stage holds several rows;
// bitplanes use 8-warp CTAs, two per SM.  The expert's
// activations for a chunk of up to `nx` tokens are staged once per CTA in shared memory,
// already paired the way the dequantised weights pair them and with their per-group sums.
// Each warp then streams its own units group by group (16 rows x 128 K-elements per group)
// through a private ring of shared-memory slots with 16-byte cp.async copies kept several
// groups ahead (commit/wait groups, no cross-warp handshake), and per group: shared loads,
// nibble / bit / FP4 -> fp16 or bf16 in registers, mma.sync m16n8k16 with the tokens on N.
// W4 takes two groups per wait and converts nibbles to fp16 against activations staged
// in fp16 (see w4h_group); its group loop is unrolled over one turn of the ring, so slot
// offsets are constants.  Expert weights are read from HBM once per token chunk.  In a
// tensor-core GEMM batch the same kernel runs over the experts with at most 16 rows only.
#include <atomic>
#include <climits>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

enum { kGateUp = 0, kDown = 1 };
constexpr int kRows = 16;     // weight rows per unit
constexpr int kWarps = 4;     // warps per CTA (W4, NVFP4), each owning whole units
constexpr int kWarpsBP = 8;   // bitplanes: eight warps share one activation stage
constexpr int kDepth = 6;     // group steps in flight per warp (NVFP4)
constexpr int kDepthW4 = 6;   // W4: groups in flight per warp, consumed and refilled two at a time
constexpr int kMaxTok = 16;   // tokens per activation stage (two n8 tiles)
constexpr size_t kSmemTarget = 55 * 1024;  // four CTAs per SM
constexpr int kWarpsWide = 16;                 // wide rows: one 16-warp CTA per SM
constexpr size_t kSmemTargetWide = 219 * 1024;
// Bitplanes: a group step holds only the planes the chunk reads (b x 16 rows x 16 bytes),
// so a fixed per-warp ring of 16 plane slots is min(8, 16 / b) steps deep (8 at b <= 2, 5
// at b = 3, 4, 3, then 2 at b >= 6); two 8-warp CTAs per SM still stage 16 tokens at
// K = 2048 (16 warps per SM).
constexpr int kRingBP = 16 * kRows * 16;
constexpr size_t kSmemTargetBP = 112 * 1024;
__host__ __device__ constexpr int bp_depth(int nplanes) { return (16 / nplanes) < 8 ? 16 / nplanes : 8; }
template <int FMT>
__host__ __device__ constexpr int warps_of() {
  return FMT == MOE_FMT_BITPLANE8 ? kWarpsBP : kWarps;
}

struct FfnArgs {
  const void* act;  // gate/up: x bf16 [T][K]; down: h [P][K] (bf16, or fp16*2^-8 for NVFP4)
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
  int max_rows;  // experts with more routed rows are left to the tensor-core GEMM
  // shared-memory plan (bytes), filled by the launcher
  int nx, x_stride, slot_bytes, warp_bytes, off_x, off_xsum, off_bits;
};

template <int FMT>
__host__ __device__ constexpr int depth_of() {
  return FMT == MOE_FMT_W4G128 ? kDepthW4 : kDepth;
}
template <int FMT>
__host__ __device__ inline int slot_bytes_of() {  // one group step of one unit (bitplanes: all 8 planes)
  return FMT == MOE_FMT_BITPLANE8 ? 8 * kRows * 16 : (FMT == MOE_FMT_NVFP4 ? kRows * 64 + kRows * 8 : kRows * 64);
}
template <int FMT>
__host__ __device__ inline int ring_bytes_of() {  // one warp's ring of group slots
  return FMT == MOE_FMT_BITPLANE8 ? kRingBP : depth_of<FMT>() * slot_bytes_of<FMT>();
}
// x rows: stride/16 = 4 (mod 8) keeps the 8 lanes of a quarter warp on distinct banks
__host__ __device__ inline int stride_16B(int row_bytes) {
  return ((row_bytes / 16) % 8 == 4) ? row_bytes : row_bytes + ((4 - (row_bytes / 16) % 8) + 8) % 8 * 16;
}

// ---------------------------------------------------------------- async copies
MOE_DEVICE void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
MOE_DEVICE void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
MOE_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
MOE_DEVICE void cp_async_wait_n() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
MOE_DEVICE void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------- group steps
// One group of 128 K-elements for the thread's slice (lane = 4g + c owns elements
// 32c .. 32c+31 of the group) of unit rows g and g+8, for one or two n8 token tiles.
// xv[nt][m] holds the pre-paired activations of word m of the slice for token column g
// of tile nt; X[nt][j] the group sum of the activations of token 2c+j of tile nt.

// INT4, fp16 route.  For a word w (element j of the word at nibble j)
//   (w & 0x000F000F) | 0x64006400 = fp16 (1024 + u0, 1024 + u4)
//   (w & 0x00F000F0) | 0x64006400 = fp16 (1024 + 16 u1, 1024 + 16 u5)
// and the same on w >> 8 for (u2, u6) and (16 u3, 16 u7): one shift and four LOP3 per
// eight weights.  The activations were staged as fp16 x/16 opposite the first kind and
// x/256 opposite the second, so each product is (1032 + q) x/16 or (72 + q) x/16 (q = u - 8);
// the accumulator starts at the staged seed -(1032 sum x/16 + 1152 sum x/256) of the
// group and ends at sum q x/16, scaled by s into the row's sum (the factor 16 is applied
// once, in the epilogue).
template <bool TWO>
MOE_DEVICE void w4h_group(uint4 wa, uint4 wb, const uint4 (&xv)[2][4], float sa, float sb,
                          const float (&S)[2][2], float (&acc)[2][4]) {
  const uint32_t wa_[4] = {wa.x, wa.y, wa.z, wa.w};
  const uint32_t wb_[4] = {wb.x, wb.y, wb.z, wb.w};
  constexpr uint32_t kM = 0x64006400u;  // fp16 (1024, 1024)
  constexpr int NT = TWO ? 2 : 1;
  float t[2][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    t[nt][0] = t[nt][2] = S[nt][0];
    t[nt][1] = t[nt][3] = S[nt][1];
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t ah = wa_[m] >> 8, bh = wb_[m] >> 8;
    const uint32_t pa0 = (wa_[m] & 0x000F000Fu) | kM, pa1 = (wa_[m] & 0x00F000F0u) | kM;
    const uint32_t pa2 = (ah & 0x000F000Fu) | kM, pa3 = (ah & 0x00F000F0u) | kM;
    const uint32_t pb0 = (wb_[m] & 0x000F000Fu) | kM, pb1 = (wb_[m] & 0x00F000F0u) | kM;
    const uint32_t pb2 = (bh & 0x000F000Fu) | kM, pb3 = (bh & 0x00F000F0u) | kM;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint4 xx = xv[nt][m];
      mma_f16(t[nt], pa0, pb0, pa1, pb1, xx.x, xx.y);
      mma_f16(t[nt], pa2, pb2, pa3, pb3, xx.z, xx.w);
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

// Bitplanes: plane-word bit j <-> element j of the lane's 32-element slice; MMA step s
// pairs bits (j, j+16) for j = 2s, 2s+1 into one bf16x2 A register (the activations were
// staged in the same pairing).  Plane p's register is bf16(2^(7-p)) in both halves with
// the plane bit OR-ed into a mantissa or the sign bit, so A = 2^(7-p) (1 + g_j bit):
//   j = 0..6   the bit stays in place (mantissa bit j):       g_j = 2^(j-7)
//   j = 7..13  mantissa bit j-7 of w >> 7 (one shift per word): g_j = 2^(j-14)
//   j = 14     the bit moves to mantissa bit 6 (one shift):    g_j = 1/2
//   j = 15     the bit stays in place (the sign):              g_j = -2
// With the activations staged as x'_k = x_k / g_j(k) (exact: powers of two), one
// accumulator collects every plane:  T = sum_{p<b} 2^(7-p) (X' + sum_k bit_pk x_k),
// X' = sum_k x'_k, so that, with X = sum_k x_k and u' the b-bit floor-and-compensation
// code (floor = sum_{p<b} 2^(7-p) bit_p, compensation c_b = 2^(7-b) for b < 8, 0 for 8),
//   sum_k (u'_k - 128) x_k = T - (256 - 2^(8-b)) X' + (c_b - 128) X.
// w7 = w >> 7 (once per plane word): bits 7..13 sit in mantissa bits 0..6 of w7
template <int J>
MOE_DEVICE uint32_t bp_a(uint32_t w, uint32_t w7, uint32_t base) {
  if constexpr (J <= 6) return (w & (0x00010001u << J)) | base;
  else if constexpr (J <= 13) return (w7 & (0x00010001u << (J - 7))) | base;
  else if constexpr (J == 15) return (w & 0x80008000u) | base;
  else return ((w >> (J - 6)) & 0x00400040u) | base;
}
// activation scale 1 / g_j of pair j
MOE_DEVICE float bp_xscale(int j) {
  return j <= 6 ? float(1 << (7 - j)) : j <= 13 ? float(1 << (14 - j)) : (j == 15 ? -0.5f : 2.f);
}

// Widths of the chunk's tokens as one lane sees them: the C columns 2c, 2c+1 (+8) for
// the epilogue, the B column g (+8) for the tail planes, and the chunk's min / max.
struct BpChunk {
  int nplanes, pmin;
  float k1[2][2], k2[2][2];  // per C column: 256 - 2^(8-b) and c_b - 128 of its width b
  int bB[2];
};

// one plane of one group: 8 MMA steps per n8 tile; MASK zeroes the B columns of tokens
// narrower than this plane
template <bool TWO, bool MASK>
MOE_DEVICE void bp_plane(uint32_t wa, uint32_t wb, int p, const uint4 (&xv)[2][4], const BpChunk& bc,
                         float (&t0)[2][4], float (&t1)[2][4]) {
  const uint32_t e = uint32_t(134 - p) << 7;  // bf16 2^(7-p)
  const uint32_t base = e | (e << 16);
  bool keep[2] = {true, true};
  if (MASK) {
    keep[0] = p < bc.bB[0];
    keep[1] = p < bc.bB[1];
  }
  const uint32_t wa7 = wa >> 7, wb7 = wb >> 7;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    uint32_t a0, a1, a2, a3;
#define MOE_BP_STEP(S)                                                      \
  case S:                                                                   \
    a0 = bp_a<2 * S>(wa, wa7, base), a2 = bp_a<2 * S + 1>(wa, wa7, base); \
    a1 = bp_a<2 * S>(wb, wb7, base), a3 = bp_a<2 * S + 1>(wb, wb7, base); \
    break;
    switch (s) {
      MOE_BP_STEP(0)
      MOE_BP_STEP(1)
      MOE_BP_STEP(2)
      MOE_BP_STEP(3)
      MOE_BP_STEP(4)
      MOE_BP_STEP(5)
      MOE_BP_STEP(6)
      default:
        a0 = bp_a<14>(wa, wa7, base), a2 = bp_a<15>(wa, wa7, base);
        a1 = bp_a<14>(wb, wb7, base), a3 = bp_a<15>(wb, wb7, base);
        break;
    }
#undef MOE_BP_STEP
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      if (nt == 1 && !TWO) break;
      const uint4 xx = xv[nt][s >> 1];
      uint32_t b0 = (s & 1) ? xx.z : xx.x, b1 = (s & 1) ? xx.w : xx.y;
      if (MASK && !keep[nt]) b0 = b1 = 0u;
      float(&t)[4] = (s & 1) ? t1[nt] : t0[nt];
      mma_bf16(t, a0, a1, a2, a3, b0, b1);
    }
  }
}

// pl: the lane's word of plane 0, row g; planes are 16 rows x 16 bytes apart.  X / X2:
// the group sums X and X' of the lane's C columns.
template <bool TWO>
MOE_DEVICE void bp_group(const uint8_t* pl, const BpChunk& bc, const uint4 (&xv)[2][4], float sa, float sb,
                         const float (&X)[2][2], const float (&X2)[2][2], float (&acc)[2][4]) {
  float t0[2][4], t1[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) t0[nt][i] = t1[nt][i] = 0.f;
  int p = 0;
  for (; p < bc.pmin; ++p)  // planes every token of the chunk reads
    bp_plane<TWO, false>(*reinterpret_cast<const uint32_t*>(pl + p * kRows * 16),
                         *reinterpret_cast<const uint32_t*>(pl + p * kRows * 16 + 8 * 16), p, xv, bc, t0, t1);
  for (; p < bc.nplanes; ++p)  // planes only the wider tokens read
    bp_plane<TWO, true>(*reinterpret_cast<const uint32_t*>(pl + p * kRows * 16),
                        *reinterpret_cast<const uint32_t*>(pl + p * kRows * 16 + 8 * 16), p, xv, bc, t0, t1);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    if (nt == 1 && !TWO) break;
    float corr[2];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) corr[jj] = fmaf(bc.k2[nt][jj], X[nt][jj], -bc.k1[nt][jj] * X2[nt][jj]);
    acc[nt][0] = fmaf(sa, (t0[nt][0] + t1[nt][0]) + corr[0], acc[nt][0]);
    acc[nt][1] = fmaf(sa, (t0[nt][1] + t1[nt][1]) + corr[1], acc[nt][1]);
    acc[nt][2] = fmaf(sb, (t0[nt][2] + t1[nt][2]) + corr[0], acc[nt][2]);
    acc[nt][3] = fmaf(sb, (t0[nt][3] + t1[nt][3]) + corr[1], acc[nt][3]);
  }
}

// NVFP4: byte i of a word holds elements 2i (low nibble) and 2i+1; the hardware converts
// the pair to fp16 and the E4M3 block scale multiplies it in fp16 (exact); activations
// are fp16 * 2^-8 in natural pairs.
template <bool TWO>
MOE_DEVICE void fp4_group(uint4 wa, uint4 wb, uint32_t scA, uint32_t scB, const uint4 (&xv)[2][4],
                          float (&acc)[2][4]) {
  constexpr bool two = TWO;
  const uint32_t wa_[4] = {wa.x, wa.y, wa.z, wa.w};
  const uint32_t wb_[4] = {wb.x, wb.y, wb.z, wb.w};
  // words 0,1 -> block 2c (byte 0 of sc), words 2,3 -> block 2c+1 (byte 1)
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

// ---------------------------------------------------------------- one W4 unit
// Streams the warp's W4 unit two groups per step: waits for groups G, G+1, computes them,
// and refills their slots with groups G + kDepthW4, G + kDepthW4 + 1 (one commit group per
// step).  Per-lane addresses are formed once; the steps are unrolled over one turn of the
// ring, so every slot offset is a constant.
template <bool TWO, class Issue>
MOE_DEVICE void stream_w4(const FfnArgs& a, const uint8_t* wsm, const uint16_t* wscale, const uint8_t* xbuf,
                          const float* xsum, int GK, int g, int c, int nvalid, Issue&& issue, float (&acc)[2][4]) {
  constexpr int NT = TWO ? 2 : 1;
  constexpr int D = kDepthW4;
  // B column of an absent token: any staged row will do (each output column depends only
  // on its own B column, and absent columns are never stored)
  const uint8_t* xr[2] = {xbuf + size_t(min(g, nvalid - 1)) * a.x_stride + c * 16,
                          xbuf + size_t(min(8 + g, nvalid - 1)) * a.x_stride + c * 16};
  const float* sr = xsum + 2 * c;  // seeds [G][kMaxTok]: columns 2c, 2c+1 (+8 for the second tile)
  const uint16_t* wsa = wscale + g * GK;
  const uint16_t* wsb = wscale + (g + 8) * GK;
  const uint8_t* wl = wsm + g * 64 + c * 16;
  // the ring is walked D groups at a time, so every slot offset is a constant
  for (int G0 = 0; G0 < GK; G0 += D) {
#pragma unroll
    for (int hp = 0; hp < D; hp += 2) {
      const int G = G0 + hp;
      if (G >= GK) break;
      cp_async_wait_n<D / 2 - 1>();
      __syncwarp();  // every lane's copies of groups G, G+1 have landed
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int GG = G + h;
        if (GG < GK) {
          uint4 xv[2][4];
          float S[2][2];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int m = 0; m < 4; ++m) xv[nt][m] = *reinterpret_cast<const uint4*>(xr[nt] + GG * 256 + m * 64);
            const float2 s2 = *reinterpret_cast<const float2*>(sr + GG * kMaxTok + 8 * nt);
            S[nt][0] = s2.x;
            S[nt][1] = s2.y;
          }
          const uint8_t* wr = wl + (hp + h) * 1024;
          w4h_group<TWO>(*reinterpret_cast<const uint4*>(wr), *reinterpret_cast<const uint4*>(wr + 8 * 64), xv,
                         bf16_bits_to_float(wsa[GG]), bf16_bits_to_float(wsb[GG]), S, acc);
        }
      }
      __syncwarp();  // every lane is done with these slots before they are refilled
      if (G + D < GK) issue(G + D, hp);
      if (G + D + 1 < GK) issue(G + D + 1, hp + 1);
      cp_async_commit();
    }
  }
}

// ---------------------------------------------------------------- one unit (bitplane, NVFP4)
// Streams the warp's unit through a ring of D slots of `slot` bytes: for G = 0 .. GK-1,
// waits for group G's slot, computes it against the staged activations of one (TWO =
// false) or two n8 token tiles, and refills the slot with group G + D.
template <int FMT, bool TWO, int D, class Issue>
MOE_DEVICE void stream_unit(const FfnArgs& a, const uint8_t* wsm, int slot, const uint16_t* wscale,
                            const uint8_t* xbuf, const float* xsum, int GK, int g, int c, int nvalid,
                            const BpChunk& bc, Issue&& issue, float (&acc)[2][4]) {
  constexpr int NT = TWO ? 2 : 1;
  // B column of an absent token: any staged row will do (each output column depends only on
  // its own B column, and absent columns are never stored)
  const uint8_t* xb[2] = {xbuf + size_t(min(g, nvalid - 1)) * a.x_stride + c * 16,
                          xbuf + size_t(min(8 + g, nvalid - 1)) * a.x_stride + c * 16};
  auto step = [&](int G, int ring) {  // group G in ring slot `ring`, then its refill
    cp_async_wait_n<D - 1>();
    __syncwarp();  // every lane's copies of group G have landed
    const uint8_t* sl = wsm + ring * slot;
    uint4 xv[2][4];
    float X[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, X2[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint8_t* xr = xb[nt] + G * 256;
#pragma unroll
      for (int m = 0; m < 4; ++m) xv[nt][m] = *reinterpret_cast<const uint4*>(xr + m * 64);
      if (FMT == MOE_FMT_BITPLANE8) {  // group sums X, X' of C columns 2c, 2c+1 ([G][kMaxTok] each)
        const float2 x1 = *reinterpret_cast<const float2*>(xsum + G * kMaxTok + nt * 8 + 2 * c);
        const float2 x2 = *reinterpret_cast<const float2*>(xsum + (GK + G) * kMaxTok + nt * 8 + 2 * c);
        X[nt][0] = x1.x;
        X[nt][1] = x1.y;
        X2[nt][0] = x2.x;
        X2[nt][1] = x2.y;
      }
    }
    if (FMT == MOE_FMT_BITPLANE8) {
      bp_group<TWO>(sl + g * 16 + c * 4, bc, xv, bf16_bits_to_float(wscale[g * GK + G]),
                    bf16_bits_to_float(wscale[(g + 8) * GK + G]), X, X2, acc);
    } else {
      const uint8_t* wr = sl + g * 64 + c * 16;
      const uint8_t* sc = sl + kRows * 64;  // [16 rows][8 block scales]
      const uint32_t scA = *reinterpret_cast<const uint16_t*>(sc + g * 8 + 2 * c);
      const uint32_t scB = *reinterpret_cast<const uint16_t*>(sc + (g + 8) * 8 + 2 * c);
      fp4_group<TWO>(*reinterpret_cast<const uint4*>(wr), *reinterpret_cast<const uint4*>(wr + 8 * 64), scA, scB,
                     xv, acc);
    }
    __syncwarp();  // every lane is done with this slot before it is refilled
    if (G + D < GK) issue(G + D, ring);
    cp_async_commit();
  };
  if constexpr (FMT == MOE_FMT_NVFP4) {  // one turn of the ring at a time: constant slot offsets
    for (int G0 = 0; G0 < GK; G0 += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        if (G0 + d >= GK) break;
        step(G0 + d, d);
      }
    }
  } else {  // bitplanes: D depends on the chunk's widths; the slot is kept as a counter
    int ring = 0;  // G % D
    for (int G = 0; G < GK; ++G) {
      step(G, ring);
      ring = (ring == D - 1) ? 0 : ring + 1;
    }
  }
}

// bitplanes: the ring depth for the chunk's prefix length, as a compile-time constant
template <bool TWO, class Issue>
MOE_DEVICE void stream_unit_bp(const FfnArgs& a, const uint8_t* wsm, const uint16_t* wscale, const uint8_t* xbuf,
                               const float* xsum, int GK, int g, int c, int nvalid, const BpChunk& bc,
                               Issue&& issue, float (&acc)[2][4]) {
  const int slot = bc.nplanes * kRows * 16;
  switch (bp_depth(bc.nplanes)) {
    case 8:
      stream_unit<MOE_FMT_BITPLANE8, TWO, 8>(a, wsm, slot, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue, acc);
      break;
    case 5:
      stream_unit<MOE_FMT_BITPLANE8, TWO, 5>(a, wsm, slot, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue, acc);
      break;
    case 4:
      stream_unit<MOE_FMT_BITPLANE8, TWO, 4>(a, wsm, slot, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue, acc);
      break;
    case 3:
      stream_unit<MOE_FMT_BITPLANE8, TWO, 3>(a, wsm, slot, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue, acc);
      break;
    default:
      stream_unit<MOE_FMT_BITPLANE8, TWO, 2>(a, wsm, slot, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue, acc);
      break;
  }
}

// ---------------------------------------------------------------- kernel
template <int FMT, int MODE, int WARPS>
__global__ void __launch_bounds__(32 * WARPS, 16 / WARPS) k_ffn_gemv(FfnArgs a) {
  constexpr int THREADS = 32 * WARPS;
  extern __shared__ __align__(128) uint8_t smem[];

  const int slot = blockIdx.y;
  if (slot >= a.expert_list[0]) return;
  const int e = a.expert_list[1 + slot];
  const int row0 = a.offsets[e];
  const int n_e = a.offsets[e + 1] - row0;
  if (n_e > a.max_rows) return;  // this expert's rows go through the tensor-core GEMM
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int K = a.K, GK = K / 128;
  const int TPE = (MODE == kGateUp) ? a.I / 8 : a.N / kRows;
  const int rt = blockIdx.x * WARPS + warp;  // this warp's unit
  const bool has_unit = rt < TPE;

  uint8_t* xbuf = smem + a.off_x;
  float* xsum = reinterpret_cast<float*>(smem + a.off_xsum);
  int* sbits = reinterpret_cast<int*>(smem + a.off_bits);
  uint8_t* wsm = smem + size_t(warp) * a.warp_bytes;  // this warp's ring (+ scales)
  uint16_t* wscale = reinterpret_cast<uint16_t*>(wsm + ring_bytes_of<FMT>());

  auto wrow = [&](int i) -> int {  // expert-matrix row of unit row i
    if (MODE == kGateUp) return (i < 8) ? (8 * rt + i) : (a.I + 8 * rt + i - 8);
    return kRows * rt + i;
  };

  // ---- per-lane copy plan of this warp's unit
  // W4 / NVFP4: per step the lane copies 16 bytes of rows r = lane/4 and r + 8 (chunk lane%4),
  //             plus (NVFP4, lane < 16) the 8 block scales of row lane.
  // Bitplanes:  per step the lane copies the 16-byte group word of row lane%16 for planes
  //             lane/16, lane/16 + 2, ... below the chunk's prefix length.
  const uint8_t* wbase = static_cast<const uint8_t*>(a.w);
  const size_t rbK = size_t(FMT == MOE_FMT_BITPLANE8 ? K / 8 : K / 2);  // bytes per weight row (per plane)
  const size_t pstride = size_t(a.N) * rbK;
  const uint8_t* srcA = wbase;
  const uint8_t* srcB = wbase;
  const uint8_t* sbA = wbase;
  if (has_unit) {
    if (FMT == MOE_FMT_BITPLANE8) {
      srcA = wbase + (size_t(e) * 8 + (lane >> 4)) * pstride + size_t(wrow(lane & 15)) * rbK;
    } else {
      const int r = lane >> 2;
      srcA = wbase + (size_t(e) * a.N + wrow(r)) * rbK + (lane & 3) * 16;
      srcB = wbase + (size_t(e) * a.N + wrow(r + 8)) * rbK + (lane & 3) * 16;
      if (FMT == MOE_FMT_NVFP4)
        sbA = static_cast<const uint8_t*>(a.s) + (size_t(e) * a.N + wrow(lane & 15)) * size_t(K / 16);
    }
  }

  for (int tok0 = 0; tok0 < n_e; tok0 += a.nx) {
    const int nvalid = min(a.nx, n_e - tok0);
    const bool two = nvalid > 8;
    if (tok0 > 0) __syncthreads();  // the previous chunk's activations are no longer read

    // bitplanes: prefix length of this chunk (known before any weight is requested): lane n
    // reads token n's width (nvalid <= 16), one warp max-reduction
    int nplanes = 1, pmin = 1;
    if (FMT == MOE_FMT_BITPLANE8) {
      const int v = (lane < nvalid) ? min(8, max(1, int(a.bits[a.sorted_pair[row0 + tok0 + lane]]))) : 0;
      nplanes = max(1, __reduce_max_sync(0xffffffffu, v));
      pmin = __reduce_min_sync(0xffffffffu, lane < nvalid ? v : 8);
    }
    // ring geometry of this chunk: bitplane slots hold the chunk's nplanes planes only
    const int ring_slot = (FMT == MOE_FMT_BITPLANE8) ? nplanes * kRows * 16 : a.slot_bytes;
    const int ring_depth = (FMT == MOE_FMT_BITPLANE8) ? bp_depth(nplanes) : depth_of<FMT>();
    auto issue = [&](int G, int slot) {  // copy group G of the unit into ring slot `slot` (= G % ring_depth)
      uint8_t* dst = wsm + slot * ring_slot;
      if (FMT == MOE_FMT_BITPLANE8) {
        const int i = lane & 15;
        for (int p = lane >> 4; p < nplanes; p += 2)
          cp_async16(dst + (p * kRows + i) * 16, srcA + size_t(p - (lane >> 4)) * pstride + G * 16);
      } else {
        const int r = lane >> 2;
        cp_async16(dst + r * 64 + (lane & 3) * 16, srcA + G * 64);
        cp_async16(dst + (r + 8) * 64 + (lane & 3) * 16, srcB + G * 64);
        if (FMT == MOE_FMT_NVFP4 && lane < 16) cp_async8(dst + kRows * 64 + lane * 8, sbA + G * 8);
      }
    };
    // start this warp's weight stream before staging activations (the two overlap); the
    // unit's 16 rows x GK scales travel in the first commit group
    if (has_unit) {
      if (FMT != MOE_FMT_NVFP4) {
        const uint16_t* sb = static_cast<const uint16_t*>(a.s);
        if ((GK & 7) == 0) {  // whole 16-byte chunks per row
          const int cpr = GK / 8;
          for (int idx = lane; idx < kRows * cpr; idx += 32) {
            const int i = idx / cpr, ch = idx - i * cpr;
            cp_async16(wscale + i * GK + ch * 8, sb + (size_t(e) * a.N + wrow(i)) * GK + ch * 8);
          }
        } else {  // batched loads: eight in flight per lane
          const int n = kRows * GK;
          for (int base = 0; base < n; base += 32 * 8) {
            uint16_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int idx = base + u * 32 + lane;
              if (idx < n) {
                const int i = idx / GK, gg = idx - i * GK;
                v[u] = sb[(size_t(e) * a.N + wrow(i)) * GK + gg];
              }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int idx = base + u * 32 + lane;
              if (idx < n) wscale[idx] = v[u];
            }
          }
        }
      }
      if (FMT == MOE_FMT_W4G128) {  // two groups per commit group
        for (int G = 0; G < kDepthW4; G += 2) {
          if (G < GK) issue(G, G);
          if (G + 1 < GK) issue(G + 1, G + 1);
          cp_async_commit();
        }
      } else {
        for (int G = 0; G < ring_depth; ++G) {
          if (G < GK) issue(G, G);
          cp_async_commit();
        }
      }
    }

    // ---- stage activations: slice q = (token n, 32-element slice sl), pre-paired per format
    const int slices = K / 32;
    const int nslices = nvalid * slices;
    for (int q0 = 0; q0 < nslices; q0 += THREADS) {
      const int q = q0 + threadIdx.x;
      const bool ok = q < nslices;
      float ssum = 0.f, ssum2 = 0.f;
      int n = 0, sl = 0;
      if (ok) {
        n = q / slices;
        sl = q - n * slices;
        const int r = row0 + tok0 + n;
        const size_t arow = (MODE == kGateUp) ? size_t(a.sorted_pair[r] / a.k) : size_t(r);
        const uint4* src =
            reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.act) + (arow * K + size_t(sl) * 32) * 2);
        uint32_t R[16];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint4 v = src[m];
          R[4 * m] = v.x;
          R[4 * m + 1] = v.y;
          R[4 * m + 2] = v.z;
          R[4 * m + 3] = v.w;
        }
        uint32_t O[16];
        if (FMT == MOE_FMT_W4G128) {
          // word m: fp16 (x0, x4)/16, (x1, x5)/256, (x2, x6)/16, (x3, x7)/256, and the seed
          // -(1032 * sum of the /16 values + 1152 * sum of the /256 values)
          float lo = 0.f, hi = 0.f;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t r0 = R[4 * m], r1 = R[4 * m + 1], r2 = R[4 * m + 2], r3 = R[4 * m + 3];
            const __half2 h0 = __floats2half2_rn(bf16_lo(r0) * 0.0625f, bf16_lo(r2) * 0.0625f);
            const __half2 h1 = __floats2half2_rn(bf16_hi(r0) * 0.00390625f, bf16_hi(r2) * 0.00390625f);
            const __half2 h2 = __floats2half2_rn(bf16_lo(r1) * 0.0625f, bf16_lo(r3) * 0.0625f);
            const __half2 h3 = __floats2half2_rn(bf16_hi(r1) * 0.00390625f, bf16_hi(r3) * 0.00390625f);
            O[4 * m] = *reinterpret_cast<const uint32_t*>(&h0);
            O[4 * m + 1] = *reinterpret_cast<const uint32_t*>(&h1);
            O[4 * m + 2] = *reinterpret_cast<const uint32_t*>(&h2);
            O[4 * m + 3] = *reinterpret_cast<const uint32_t*>(&h3);
            const float2 f0 = __half22float2(h0), f1 = __half22float2(h1), f2 = __half22float2(h2),
                         f3 = __half22float2(h3);
            lo += (f0.x + f0.y) + (f2.x + f2.y);
            hi += (f1.x + f1.y) + (f3.x + f3.y);
          }
          ssum = -1032.f * lo - 1152.f * hi;
        } else if (FMT == MOE_FMT_BITPLANE8) {
          // step s: (x_2s, x_2s+16), (x_2s+1, x_2s+17), each pair j scaled by 1 / g_j (exact)
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const float f0 = bp_xscale(2 * s), f1 = bp_xscale(2 * s + 1);
            const float lo0 = bf16_lo(R[s]) * f0, hi0 = bf16_lo(R[s + 8]) * f0;
            const float lo1 = bf16_hi(R[s]) * f1, hi1 = bf16_hi(R[s + 8]) * f1;
            O[2 * s] = uint32_t(float_to_bf16_bits(lo0)) | (uint32_t(float_to_bf16_bits(hi0)) << 16);
            O[2 * s + 1] = uint32_t(float_to_bf16_bits(lo1)) | (uint32_t(float_to_bf16_bits(hi1)) << 16);
            ssum2 += (lo0 + hi0) + (lo1 + hi1);
          }
        } else {
          if (MODE == kGateUp) {  // bf16 -> fp16 * 2^-8, natural pairs
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const __half2 h = __floats2half2_rn(bf16_lo(R[i]) * (1.0f / 256.f), bf16_hi(R[i]) * (1.0f / 256.f));
              O[i] = *reinterpret_cast<const uint32_t*>(&h);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) O[i] = R[i];
          }
        }
        if (FMT == MOE_FMT_BITPLANE8) {
#pragma unroll
          for (int i = 0; i < 16; ++i) ssum += bf16_lo(R[i]) + bf16_hi(R[i]);
        }
        // slice sl = group G, lane slice cc; word m of the slice goes to 16-byte chunk 4m + cc
        const int G = sl >> 2, cc = sl & 3;
        uint8_t* dst = xbuf + size_t(n) * a.x_stride + G * 256;
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(dst + (4 * m + cc) * 16) =
              make_uint4(O[4 * m], O[4 * m + 1], O[4 * m + 2], O[4 * m + 3]);
      }
      if (FMT != MOE_FMT_NVFP4) {  // group sums: the 4 slices of a group are 4 consecutive lanes
        ssum += __shfl_xor_sync(0xffffffffu, ssum, 1);
        ssum += __shfl_xor_sync(0xffffffffu, ssum, 2);
        if (ok && (sl & 3) == 0) xsum[(sl >> 2) * kMaxTok + n] = ssum;
      }
      if (FMT == MOE_FMT_BITPLANE8) {  // and X' ([GK + G][kMaxTok])
        ssum2 += __shfl_xor_sync(0xffffffffu, ssum2, 1);
        ssum2 += __shfl_xor_sync(0xffffffffu, ssum2, 2);
        if (ok && (sl & 3) == 0) xsum[(slices / 4 + (sl >> 2)) * kMaxTok + n] = ssum2;
      }
    }
    if (FMT == MOE_FMT_BITPLANE8)
      for (int n = threadIdx.x; n < kMaxTok; n += THREADS)
        sbits[n] = (n < nvalid) ? min(8, max(1, int(a.bits[a.sorted_pair[row0 + tok0 + n]]))) : 8;
    __syncthreads();
    if (!has_unit) continue;

    BpChunk bc{nplanes, pmin, {{0.f, 0.f}, {0.f, 0.f}}, {{0.f, 0.f}, {0.f, 0.f}}, {8, 8}};
    if (FMT == MOE_FMT_BITPLANE8) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int b = sbits[nt * 8 + 2 * c + jj];
          bc.k1[nt][jj] = float(256 - (1 << (8 - b)));
          bc.k2[nt][jj] = float((b < 8 ? (1 << (7 - b)) : 0) - 128);
        }
        bc.bB[nt] = sbits[nt * 8 + g];
      }
    }

    // ---- stream the unit: group G is computed while groups G+1 .. G+kDepth-1 are in flight
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    if constexpr (FMT == MOE_FMT_W4G128) {
      if (two)
        stream_w4<true>(a, wsm, wscale, xbuf, xsum, GK, g, c, nvalid, issue, acc);
      else
        stream_w4<false>(a, wsm, wscale, xbuf, xsum, GK, g, c, nvalid, issue, acc);
    } else if constexpr (FMT == MOE_FMT_BITPLANE8) {
      if (two)
        stream_unit_bp<true>(a, wsm, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue, acc);
      else
        stream_unit_bp<false>(a, wsm, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue, acc);
    } else {
      if (two)
        stream_unit<FMT, true, kDepth>(a, wsm, a.slot_bytes, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue,
                                       acc);
      else
        stream_unit<FMT, false, kDepth>(a, wsm, a.slot_bytes, wscale, xbuf, xsum, GK, g, c, nvalid, bc, issue,
                                        acc);
    }
    cp_async_wait_all();

    // ---- epilogue: C fragment = rows g / g+8, tokens 2c, 2c+1 of each n8 tile
    float post = 1.f;
    if (FMT == MOE_FMT_NVFP4) post = a.gscale[e] * 256.f;
    if (FMT == MOE_FMT_W4G128) post = 16.f;  // the activations were staged as x/16
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int n = nt * 8 + 2 * c + jj;
        if (n >= nvalid) continue;
        const size_t orow = size_t(row0 + tok0 + n) * a.out_ld;
        const float v0 = acc[nt][jj] * post, v1 = acc[nt][2 + jj] * post;
        if (MODE == kGateUp) {
          const float h = silu(v0) * v1;
          const int col = 8 * rt + g;
          if (FMT == MOE_FMT_NVFP4)
            static_cast<__half*>(a.out)[orow + col] = __float2half_rn(h * (1.0f / 256.f));
          else
            static_cast<uint16_t*>(a.out)[orow + col] = float_to_bf16_bits(h);
        } else {
          uint16_t* y = static_cast<uint16_t*>(a.out);
          y[orow + kRows * rt + g] = float_to_bf16_bits(v0);
          y[orow + kRows * rt + g + 8] = float_to_bf16_bits(v1);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- launch planning
static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

size_t ffn_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, moe_format_t fmt) {
  if (use_umma_path(T, E, k, fmt)) return umma_workspace_bytes(T, H, I, k);
  return align256(size_t(T * k * I * 2));  // h
}

// Shared-memory plan of a CTA of `warps` warps within `target` bytes: the warps' rings and
// scales, then as many staged token rows (nx, at most 16) as fit.
template <int FMT>
static bool plan(FfnArgs& a, int warps = warps_of<FMT>(), size_t target = 0) {
  const int K = a.K, GK = K / 128;
  a.slot_bytes = slot_bytes_of<FMT>();
  const int scale_bytes = (FMT == MOE_FMT_NVFP4) ? 0 : int(align256(size_t(kRows) * GK * 2));
  a.warp_bytes = int(align256(size_t(ring_bytes_of<FMT>()) + scale_bytes));
  a.x_stride = stride_16B(K * 2);
  const int nsum = (FMT == MOE_FMT_BITPLANE8) ? 2 : 1;  // bitplanes: X and X'
  const size_t fixed = size_t(warps) * a.warp_bytes + align256(size_t(nsum) * kMaxTok * GK * 4) + 256;
  if (!target) target = (FMT == MOE_FMT_BITPLANE8) ? kSmemTargetBP : kSmemTarget;
  const size_t room = fixed < target ? target - fixed : 0;
  int nx = int(room / size_t(a.x_stride));
  nx = nx < 1 ? 1 : nx;  // wide rows: at least one token row (then one CTA per SM)
  a.nx = nx > kMaxTok ? kMaxTok : nx;
  size_t off = size_t(warps) * a.warp_bytes;
  a.off_x = int(off);
  off += align256(size_t(a.nx) * a.x_stride);
  a.off_xsum = int(off);
  off += align256(size_t(nsum) * kMaxTok * GK * 4);
  a.off_bits = int(off);
  off += 256;
  return off <= 220 * 1024;
}

template <int FMT, int MODE, int WARPS>
static cudaError_t launch_plan(const FfnArgs& a, int slots, cudaStream_t st) {
  const size_t smem = size_t(a.off_bits) + 256;
  // raise the kernel's dynamic shared-memory limit once per device (kept out of later
  // calls, which may be inside a graph capture)
  static std::atomic<bool> raised[128] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!raised[dev].load(std::memory_order_relaxed)) {
    cudaError_t err =
        cudaFuncSetAttribute(k_ffn_gemv<FMT, MODE, WARPS>, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
    if (err != cudaSuccess) return err;
    raised[dev].store(true, std::memory_order_relaxed);
  }
  const int TPE = (MODE == kGateUp) ? a.I / 8 : a.N / kRows;
  k_ffn_gemv<FMT, MODE, WARPS><<<dim3(unsigned((TPE + WARPS - 1) / WARPS), unsigned(slots)), 32 * WARPS, smem, st>>>(a);
  return cudaGetLastError();
}

// need: tokens an expert may bring (at most T).  Four small CTAs per SM stage up to 16
// token rows each; when wide rows (large K) leave room for fewer than min(need, 4), an
// expert's weights would stream once per staged token, so W4 / NVFP4 switch to one CTA of
// 16 warps per SM, whose single activation stage holds several rows for all 16 warps.
template <int FMT, int MODE>
static cudaError_t launch_one(FfnArgs a, int slots, int need, cudaStream_t st) {
  if (!plan<FMT>(a)) return cudaErrorInvalidValue;
  if constexpr (FMT != MOE_FMT_BITPLANE8) {
    if (a.nx < (need < 4 ? need : 4)) {
      FfnArgs b = a;
      if (plan<FMT>(b, kWarpsWide, kSmemTargetWide) && b.nx > a.nx)
        return launch_plan<FMT, MODE, kWarpsWide>(b, slots, st);
    }
  }
  return launch_plan<FMT, MODE, warps_of<FMT>()>(a, slots, st);
}

template <int FMT>
static cudaError_t launch_fmt(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex,
                              const uint8_t* bits, int T, int H, int I, int E, int k, uint16_t* y_rows, void* hbuf,
                              cudaStream_t st) {
  const int P = T * k;
  const int slots = P < E ? P : E;
  FfnArgs a{};
  a.k = k;
  a.I = I;
  a.expert_list = r.expert_list;
  a.offsets = r.expert_offsets;
  a.sorted_pair = r.sorted_pair;
  a.bits = bits;
  a.max_rows = INT_MAX;
  // gate/up
  a.act = x;
  a.K = H;
  a.N = 2 * I;
  a.w = ex.w13;
  a.s = ex.w13_scale;
  a.gscale = ex.w13_gscale;
  a.out = hbuf;
  a.out_ld = I;
  cudaError_t err = launch_one<FMT, kGateUp>(a, slots, T, st);
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
  return launch_one<FMT, kDown>(a, slots, T, st);
}

// One pass (gate/up or down) of the weight-streaming path over the experts with at most
// max_rows routed rows: the small experts of a batch that otherwise takes the GEMM.  h rows
// of those experts are written and read in this path's own format (disjoint from the GEMM's).
template <int FMT>
static cudaError_t launch_small_fmt(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex, int T,
                                    int H, int I, int E, int k, void* hbuf, uint16_t* y_rows, bool down,
                                    int max_rows, cudaStream_t st) {
  const int P = T * k;
  FfnArgs a{};
  a.k = k;
  a.I = I;
  a.expert_list = r.expert_list;
  a.offsets = r.expert_offsets;
  a.sorted_pair = r.sorted_pair;
  a.max_rows = max_rows;
  if (!down) {
    a.act = x;
    a.K = H;
    a.N = 2 * I;
    a.w = ex.w13;
    a.s = ex.w13_scale;
    a.gscale = ex.w13_gscale;
    a.out = hbuf;
    a.out_ld = I;
    return launch_one<FMT, kGateUp>(a, P < E ? P : E, T < max_rows ? T : max_rows, st);
  }
  a.act = hbuf;
  a.K = I;
  a.N = H;
  a.w = ex.w2;
  a.s = ex.w2_scale;
  a.gscale = ex.w2_gscale;
  a.out = y_rows;
  a.out_ld = H;
  return launch_one<FMT, kDown>(a, P < E ? P : E, T < max_rows ? T : max_rows, st);
}

cudaError_t launch_gemv_small(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex, int T, int H, int I,
                              int E, int k, void* hbuf, uint16_t* y_rows, bool down, int max_rows, cudaStream_t st) {
  if (ex.fmt == MOE_FMT_W4G128)
    return launch_small_fmt<MOE_FMT_W4G128>(x, r, ex, T, H, I, E, k, hbuf, y_rows, down, max_rows, st);
  if (ex.fmt == MOE_FMT_NVFP4)
    return launch_small_fmt<MOE_FMT_NVFP4>(x, r, ex, T, H, I, E, k, hbuf, y_rows, down, max_rows, st);
  return cudaErrorInvalidValue;
}

bool ffn_shape_supported(int64_t H, int64_t I, moe_format_t fmt) {
  FfnArgs a{};
  bool ok = true;
  for (int64_t K : {H, I}) {
    a.K = int(K);
    ok = ok && (fmt == MOE_FMT_BITPLANE8 ? plan<MOE_FMT_BITPLANE8>(a)
                : fmt == MOE_FMT_NVFP4   ? plan<MOE_FMT_NVFP4>(a)
                                         : plan<MOE_FMT_W4G128>(a));
  }
  return ok;
}

cudaError_t launch_grouped_ffn(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex,
                               const uint8_t* bits, int T, int H, int I, int E, int k, uint16_t* y_rows, void* ws,
                               cudaStream_t st) {
  if (use_umma_path(T, E, k, ex.fmt)) return launch_grouped_ffn_umma(x, r, ex, T, H, I, E, k, y_rows, ws, st);
  switch (ex.fmt) {
    case MOE_FMT_W4G128:
      return launch_fmt<MOE_FMT_W4G128>(x, r, ex, bits, T, H, I, E, k, y_rows, ws, st);
    case MOE_FMT_BITPLANE8:
      return launch_fmt<MOE_FMT_BITPLANE8>(x, r, ex, bits, T, H, I, E, k, y_rows, ws, st);
    case MOE_FMT_NVFP4:
      return launch_fmt<MOE_FMT_NVFP4>(x, r, ex, bits, T, H, I, E, k, y_rows, ws, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
