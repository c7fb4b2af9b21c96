// Grouped FFN for prefill-sized batches on the fifth-generation tensor cores
// (tcgen05, accumulators in tensor memory).
//
// Per expert e, the routed rows r in [off_e, off_{e+1}) (sorted order) are
//   gate/up:  g, u = x[token(r)] . deq(W13_e)^T,  h[r] = silu(g) * u   (fp16, scaled)
//   down:     y[r] = h[r] . deq(W2_e)^T                                 (bf16)
// i.e. the same contraction as the weight-streaming GEMV, organised as a GEMM
// when each expert sees enough rows for the weights to be worth reusing.
//
// Tile = 128 weight rows (the tensor-memory lanes, MMA M) x up to 192 routed rows
// (MMA N) x the whole K.  For gate/up, the 128 weight rows are 64 gate rows and
// the 64 matching up rows, arranged so that each warp quarter of the lanes holds
// 16 gate rows and their 16 up rows: the SwiGLU product is formed in the epilogue
// with one lane exchange.
// Roles inside one persistent CTA (one per SM, 512 threads):
//   warp  0     TMA producer: per 128-wide K stage (one scale group), the packed
//               weight tile (8 KiB) into a 4-stage ring and the routed rows (fp16,
//               128-byte swizzled K-major, two 2-D boxes of 64 K) into a 3-stage ring.
//               For gate/up the rows are the tokens gathered into routed order by
//               k_gather_rows first (one bandwidth-bound pass; gathering 4 rows per TMA
//               instruction inside the GEMM could not feed the tensor cores);
//   warp  1     allocates tensor memory; one thread issues tcgen05.mma (kind::f16,
//               fp16 in, fp32 accumulate), eight per stage, A from tensor memory, B
//               from shared memory; tcgen05.commit releases the stages;
//   warps 4-11  dequantise the weights from shared memory straight into tensor
//               memory (tcgen05.st, 2 stages of 64 columns): warp 4 + 4 s + q handles
//               rows 32 q .. 32 q + 31 of the stages n with n % 2 == s, so two warps
//               per sub-partition overlap each other's waits; the fp16 weight operand
//               never exists in shared memory;
//   warps 12-15 drain one of the two accumulators (tcgen05.ld) while the other is
//               being accumulated, apply SwiGLU, and store h (fp16, scaled) or y (bf16).
// The work list (expert, row tile, weight tile) is built by every CTA from the
// routing offsets and walked round-robin across CTAs; experts with at most 16 routed
// rows get no tiles and are left to a pass of the weight-streaming GEMV.
//
// The same file holds the W4A4 path (k_ffn_fp4 and its helpers, further down): NVFP4
// weights and activations, both fed as E2M1 codes with E4M3 block scales to the
// block-scaled FP4 MMA (kind::mxf4nvf4).
//
// Dequantisation (W4 group-128): (u - 8) * s with u the stored nibble and s the
// group's bf16 scale, formed as fp16 (1024 + u) by byte permutes, then an fp16 add of
// -1032 (exact) and an fp16 multiply by s.  q has 4 significant bits and s 8, so the
// product needs at most 12: rounded to fp16's 11 it is off by at most 2^-12 relative
// (exact in most cases), the only difference from the dequantisation of the definition
// for scales in fp16's normal range (s >= 2^-14).  The activations are the fp16 operand
// x/16 (h/16 for the down GEMM); the factor 16 is applied in the epilogue.
//
// Every wait is bounded (mbar_wait): a wait that runs out sets the device error
// word and the role stops; the CTA still frees its tensor memory.
#include <atomic>
#include <cuda.h>  // CUtensorMap and its enums; the encoder is reached through the runtime

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kTM = 128;        // weight rows per tile (tensor-memory lanes)
constexpr int kTN = 192;        // routed rows per tile (MMA N at most)
constexpr int kKB = 128;        // K elements per stage = one scale group: two 128-byte swizzle atoms of bf16
constexpr int kAtomK = 64;      // K elements of one 128-byte swizzle atom
constexpr int kBStages = 3;     // routed-row stages in shared memory
constexpr int kWStages = 4;     // packed-weight stages in shared memory
constexpr int kAStages = 2;     // dequantised weight stages in tensor memory (64 columns each)
constexpr int kDeqSets = 2;     // dequantising warp sets, alternating K blocks
constexpr int kThreadsU = 32 * (4 + 4 * kDeqSets + 4);
constexpr int kTmemCols = 512;  // accumulators at columns 0 and 192, A stages at 384 + 64 a
constexpr int kACol0 = 2 * kTN;
constexpr int kAtomBytes = kTN * 128;   // one swizzle atom of routed rows
constexpr int kBStageBytes = 2 * kAtomBytes;
constexpr int kWStageBytes = kTM * 64;  // 128 rows x 128 nibbles
constexpr int kACols = kKB / 2;         // tensor-memory columns of one A stage
constexpr int kScaleAhead = 4;          // scale groups (stages) requested ahead by the dequantisers

constexpr int kProdWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kDeqWarp0 = 4;
constexpr int kEpiWarp0 = kDeqWarp0 + 4 * kDeqSets;

// shared memory plan (offsets from a 1024-byte aligned base)
constexpr int kOffB = 0;
constexpr int kOffW = kOffB + kBStages * kBStageBytes;
constexpr int kOffPre = kOffW + kWStages * kWStageBytes;  // tile prefix over experts
constexpr int kOffOffs = kOffPre + ((MOE_MAX_EXPERTS + 1) * 4 + 255) / 256 * 256;  // routing offsets
constexpr int kOffBar = kOffOffs + ((MOE_MAX_EXPERTS + 1) * 4 + 255) / 256 * 256;
constexpr int kNumBars = 2 * kBStages + 2 * kWStages + 2 * kAStages + 4;
constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr int kSmemUsed = kOffTmemSlot + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;  // + alignment slack; > half an SM: one CTA per SM
static_assert(kSmemBytes > 114 * 1024 && kSmemBytes <= 227 * 1024, "shared-memory plan");
static_assert(kACol0 + kAStages * kACols <= kTmemCols, "tensor-memory plan");

constexpr int kGateUp = 0, kDown = 1;
// Experts with at most this many routed rows stream through the GEMV even in a GEMM batch:
// a GEMM tile costs its K/16 MMAs whatever its row count, a GEMV pass reads the weights once
// for up to 16 tokens.
constexpr int kSmallRows = 16;

struct UmmaArgs {
  int K, I, E, k;
  int wtiles;                // weight tiles per expert
  int n_rows;                // rows of one expert's weight matrix (2I or H)
  const int32_t* offsets;    // [E+1]
  const int32_t* sorted_pair;
  const uint16_t* s;         // W4: bf16 scales [E][n_rows][K/128]
  const uint8_t* bs;         // NVFP4: E4M3 block scales [E][n_rows][K/16]
  const float* gs;           // NVFP4: per-expert fp32 scale of this matrix [E]
  uint16_t* out;             // gate/up: h [P][I] (fp16 h/16 for W4, h/256 for NVFP4); down: y [P][H] bf16
  int out_ld;
  int min_rows;              // experts with fewer routed rows are left to the weight-streaming GEMV
  unsigned* err;
};

// ---------------------------------------------------------------- PTX wrappers
MOE_DEVICE void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
               "r"(ncols)
               : "memory");
}
MOE_DEVICE void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
MOE_DEVICE void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
MOE_DEVICE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEVICE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
MOE_DEVICE void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, M = 128, N from idesc, K = 16.
MOE_DEVICE void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}
MOE_DEVICE void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
MOE_DEVICE void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 consecutive 32-bit columns of this thread's lane <- v[0..31]
MOE_DEVICE void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
// v[0..31] <- 32 consecutive 32-bit columns of this thread's lane
MOE_DEVICE void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
        "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
        "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

MOE_DEVICE void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// 2-D tiled tensor load (box of the map) at element coordinates (c0 inner, c1 outer).
MOE_DEVICE void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}
MOE_DEVICE uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// mbar_wait taken by a whole warp: the result is the same in every lane, so the
// warp stays converged for the .sync.aligned tensor-memory instructions.
MOE_DEVICE bool warp_wait(uint64_t* bar, uint32_t parity, unsigned* err) {
  const bool ok = mbar_wait(bar, parity, err);
  return __all_sync(0xffffffffu, ok);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 bytes,
// 8-row groups 1024 bytes apart (base 1024-aligned; the start may advance by 32
// bytes per K=16 step inside the 128-byte row).
MOE_DEVICE uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t(1) << 16;             // leading byte offset (unused with this swizzle)
  d |= uint64_t(1024 >> 4) << 32;     // stride byte offset: next 8-row group
  d |= uint64_t(1) << 46;             // descriptor version
  d |= uint64_t(2) << 61;             // 128-byte swizzle
  return d;
}
// Instruction descriptor: fp32 accumulate, A and B both fp16 (both formats), both
// K-major, M = 128.
template <int FMT>
MOE_DEVICE uint32_t idesc_mma(int n) {
  constexpr uint32_t ab = 0u;  // 0 = f16 (1 would be bf16)
  return (1u << 4) | (ab << 7) | (ab << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kTM >> 4) << 24);
}
// The activation operand's scale: W4 stages x/16 and h/16, NVFP4 x/256 and h/256.
template <int FMT>
__host__ __device__ constexpr float act_scale() {
  return FMT == MOE_FMT_NVFP4 ? 1.f / 256.f : 1.f / 16.f;
}

// ---------------------------------------------------------------- W4 dequant
// w holds elements 8i..8i+7 of one row (element j at bits 4j); p[0..3] receive
// the pairs (0,1), (2,3), (4,5), (6,7) as fp16x2 (1024 + u_lo, 1024 + u_hi).
MOE_DEVICE void w4_word_pairs(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu;         // n0 n2 n4 n6
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // n1 n3 n5 n7
  const uint32_t u01 = __byte_perm(lo, hi, 0x5140);  // n0 n1 n2 n3
  const uint32_t u23 = __byte_perm(lo, hi, 0x7362);  // n4 n5 n6 n7
  const uint32_t k64 = 0x64646464u;  // high byte of fp16 1024
  p[0] = __byte_perm(u01, k64, 0x4140);
  p[1] = __byte_perm(u01, k64, 0x4342);
  p[2] = __byte_perm(u23, k64, 0x4140);
  p[3] = __byte_perm(u23, k64, 0x4342);
}
MOE_DEVICE uint32_t hadd2u(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ---------------------------------------------------------------- work list
struct Tile {
  int e, r0, nrows, wt;
};

// `offsets` is the CTA's shared-memory copy of the routing offsets.
MOE_DEVICE Tile tile_of(int item, const int* pre, int E, int wtiles, const int* offsets) {
  const int t = item / wtiles;
  Tile tl;
  tl.wt = item - t * wtiles;
  int lo = 0, hi = E;  // largest e with pre[e] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pre[mid] <= t) lo = mid;
    else hi = mid;
  }
  tl.e = lo;
  const int beg = offsets[lo], end = offsets[lo + 1];
  tl.r0 = beg + (t - pre[lo]) * kTN;
  tl.nrows = min(kTN, end - tl.r0);
  return tl;
}

template <int FMT, int MODE>
__global__ void __launch_bounds__(kThreadsU, 1)
    k_ffn_umma(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_w, UmmaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  int* pre = reinterpret_cast<int*>(smem + kOffPre);
  int* offs = reinterpret_cast<int*>(smem + kOffOffs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* fullB = bars;
  uint64_t* emptyB = fullB + kBStages;
  uint64_t* fullW = emptyB + kBStages;
  uint64_t* emptyW = fullW + kWStages;
  uint64_t* fullA = emptyW + kWStages;
  uint64_t* emptyA = fullA + kAStages;
  uint64_t* accFull = emptyA + kAStages;
  uint64_t* accEmpty = accFull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;

  // ---- the routing offsets into shared memory (every role reads them per tile)
  for (int i = tid; i <= E; i += blockDim.x) offs[i] = a.offsets[i];
  __syncthreads();
  // ---- tiles per expert and their prefix (warp 0), barriers (warp 2), tensor memory (warp 1)
  if (warp == 0) {
    const int per = (E + 31) / 32;
    const int b = min(E, lane * per), en = min(E, b + per);
    int sum = 0;
    // row tiles of expert e (none for an expert below min_rows: the GEMV takes it)
    auto tiles = [&](int e) {
      const int n = offs[e + 1] - offs[e];
      return n < a.min_rows ? 0 : (n + kTN - 1) / kTN;
    };
    for (int e = b; e < en; ++e) sum += tiles(e);
    int inc = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += v;
    }
    int run = inc - sum;
    for (int e = b; e < en; ++e) {
      pre[e] = run;
      run += tiles(e);
    }
    if (lane == 31) pre[E] = inc;
  } else if (tid == 64) {
    for (int i = 0; i < kBStages; ++i) {
      mbar_init(&fullB[i], 1);
      mbar_init(&emptyB[i], 1);
    }
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&fullW[i], 1);
      mbar_init(&emptyW[i], 4);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&fullA[i], 4);  // the four warps of the set that wrote the stage
      mbar_init(&emptyA[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accFull[i], 1);
      mbar_init(&accEmpty[i], 4);
    }
    fence_mbar_init();
  } else if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = pre[E] * a.wtiles;
  const int KB = a.K / kKB;

  if (warp == kProdWarp) {
    // ------------------------------------------------ TMA producer
    int n = 0;  // k-blocks issued
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const Tile tl = tile_of(item, pre, E, a.wtiles, offs);
      int wr0, wr1;  // weight box rows
      if (MODE == kGateUp) {
        wr0 = tl.e * a.n_rows + tl.wt * 64;
        wr1 = wr0 + a.I;
      } else {
        wr0 = tl.e * a.n_rows + tl.wt * kTM;
        wr1 = 0;
      }
      for (int kb = 0; kb < KB; ++kb, ++n) {
        const int sw = n % kWStages, sb = n % kBStages;
        if (!warp_wait(&emptyW[sw], ((n / kWStages) & 1) ^ 1, a.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&fullW[sw], uint32_t(kWStageBytes));
          const uint32_t wdst = sbase + kOffW + sw * kWStageBytes;
          if (MODE == kGateUp) {
            tma_load_2d(wdst, &tm_w, kb * 64, wr0, &fullW[sw]);
            tma_load_2d(wdst + kWStageBytes / 2, &tm_w, kb * 64, wr1, &fullW[sw]);
          } else {
            tma_load_2d(wdst, &tm_w, kb * 64, wr0, &fullW[sw]);
          }
        }
        if (!warp_wait(&emptyB[sb], ((n / kBStages) & 1) ^ 1, a.err)) {
          ok = false;
          break;
        }
        const uint32_t bdst = sbase + kOffB + sb * kBStageBytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&fullB[sb], uint32_t(kBStageBytes));
          tma_load_2d(bdst, &tm_b, kb * kKB, tl.r0, &fullB[sb]);
          tma_load_2d(bdst + kAtomBytes, &tm_b, kb * kKB + kAtomK, tl.r0, &fullB[sb]);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      int n = 0, it = 0;
      bool ok = true;
      const uint64_t bdesc0 = sw128_desc(sbase + kOffB);
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
        const Tile tl = tile_of(item, pre, E, a.wtiles, offs);
        const int ab = it & 1;
        if (!mbar_wait(&accEmpty[ab], ((it >> 1) & 1) ^ 1, a.err)) break;
        tc_fence_after();
        const uint32_t idesc = idesc_mma<FMT>((tl.nrows + 15) & ~15);
        const uint32_t d_tmem = tmem + uint32_t(ab * kTN);
        for (int kb = 0; kb < KB; ++kb, ++n) {
          const int sb = n % kBStages, sa = n % kAStages;
          if (!mbar_wait(&fullA[sa], (n / kAStages) & 1, a.err) || !mbar_wait(&fullB[sb], (n / kBStages) & 1, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = bdesc0 + uint64_t((sb * kBStageBytes) >> 4);
          const uint32_t a_tmem = tmem + uint32_t(kACol0 + sa * kACols);
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk)  // atom kk / 4, 32 bytes per K=16 step inside it
            tc_mma_ts(d_tmem, a_tmem + kk * 8, bdesc + uint64_t((kk >> 2) * (kAtomBytes >> 4) + 2 * (kk & 3)),
                      idesc, (kb | kk) != 0);
          tc_commit(&emptyB[sb]);
          tc_commit(&emptyA[sa]);
        }
        if (ok) tc_commit(&accFull[ab]);
      }
      // the last accumulation must be complete before the tensor memory is freed
      if (it > 0 && ok) mbar_wait(&accFull[(it - 1) & 1], ((it - 1) >> 1) & 1, a.err);
    }
    __syncwarp();
  } else if (warp >= kDeqWarp0 && warp < kEpiWarp0) {
    // ------------------------------------------------ dequantise W into tensor memory
    const int quarter = (warp - kDeqWarp0) & 3, set = (warp - kDeqWarp0) >> 2;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const int KG = a.K / 128;
    // row of this lane inside the weight box(es); for gate/up, lanes 0-15 of each
    // quarter hold gate rows and lanes 16-31 the up rows of the same 16 columns
    const int srow = (MODE == kGateUp) ? ((lane < 16) ? quarter * 16 + lane : 64 + quarter * 16 + (lane - 16))
                                       : quarter * 32 + lane;
    const int my_items = blockIdx.x < n_items ? (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
    const int total = my_items * KB;
    // scales: one bf16 per stage (128 K), requested kScaleAhead of this set's stages ahead;
    // set s converts stages n = 2 m + s (m = 0, 1, ...)
    const int my_stages = (total - set + 1) / 2;
    // W4: the stage's bf16 group scale; NVFP4: the stage's eight E4M3 block scales
    int s_li = -1;
    size_t s_row = 0;  // index of this lane's weight row in [E * n_rows]
    auto scale_at = [&](int m) -> uint2 {
      const int n = 2 * m + set;
      const int li = n / KB, grp = n - li * KB;
      if (li != s_li) {
        s_li = li;
        const Tile tl = tile_of(int(blockIdx.x) + li * int(gridDim.x), pre, E, a.wtiles, offs);
        int r;
        if (MODE == kGateUp) r = (srow < 64) ? tl.wt * 64 + srow : a.I + tl.wt * 64 + (srow - 64);
        else r = tl.wt * kTM + srow;
        s_row = size_t(tl.e) * a.n_rows + r;
      }
      if (FMT == MOE_FMT_NVFP4) return *reinterpret_cast<const uint2*>(a.bs + s_row * size_t(KG * 8) + grp * 8);
      return make_uint2(a.s[s_row * KG + grp], 0u);
    };
    uint2 sring[kScaleAhead];
#pragma unroll
    for (int q = 0; q < kScaleAhead; ++q) sring[q] = (q < my_stages) ? scale_at(q) : make_uint2(0u, 0u);
    bool ok = true;
    for (int m0 = 0; m0 < my_stages && ok; m0 += kScaleAhead) {
#pragma unroll
      for (int q = 0; q < kScaleAhead; ++q) {
        const int m = m0 + q;
        if (m >= my_stages) break;
        const uint2 sv = sring[q];
        if (m + kScaleAhead < my_stages) sring[q] = scale_at(m + kScaleAhead);
        const int n = 2 * m + set;
        const int sw = n % kWStages, sa = n % kAStages;
        if (!warp_wait(&fullW[sw], (n / kWStages) & 1, a.err)) {
          ok = false;
          break;
        }
        const uint32_t wrow = sbase + kOffW + sw * kWStageBytes + srow * 64;
        uint4 wq[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) wq[h] = lds128(wrow + 16 * h);
        __syncwarp();
        if (lane == 0) mbar_arrive(&emptyW[sw]);
        uint32_t v[2][32];
        if (FMT == MOE_FMT_NVFP4) {
          // byte c of the row's 64 = elements 2c, 2c+1 (column c); 16 elements per block scale,
          // e2m1 * e4m3 is exact in fp16
          uint32_t sb2[8];
#pragma unroll
          for (int b = 0; b < 8; ++b) sb2[b] = e4m3_to_h2(((b < 4 ? sv.x : sv.y) >> (8 * (b & 3))) & 0xFFu);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t words[8] = {wq[2 * h].x,     wq[2 * h].y,     wq[2 * h].z,     wq[2 * h].w,
                                       wq[2 * h + 1].x, wq[2 * h + 1].y, wq[2 * h + 1].z, wq[2 * h + 1].w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
              for (int j = 0; j < 4; ++j)
                v[h][4 * i + j] = hmul2(e2m1x2_to_h2((words[i] >> (8 * j)) & 0xFFu), sb2[4 * h + (i >> 1)]);
          }
        } else {
          const __half sh = __float2half_rn(bf16_bits_to_float(uint16_t(sv.x)));  // exact in fp16's normal range
          const uint32_t s2 = uint32_t(__half_as_ushort(sh)) * 0x10001u;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t words[8] = {wq[2 * h].x,     wq[2 * h].y,     wq[2 * h].z,     wq[2 * h].w,
                                       wq[2 * h + 1].x, wq[2 * h + 1].y, wq[2 * h + 1].z, wq[2 * h + 1].w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              uint32_t p[4];
              w4_word_pairs(words[i], p);
#pragma unroll
              for (int j = 0; j < 4; ++j) v[h][4 * i + j] = hmul2(hadd2u(p[j], 0xE408E408u), s2);  // (u-8)*s
            }
          }
        }
        if (!warp_wait(&emptyA[sa], ((n / kAStages) & 1) ^ 1, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32(tmem + lane_base + uint32_t(kACol0 + sa * kACols), v[0]);
        tmem_st32(tmem + lane_base + uint32_t(kACol0 + sa * kACols + 32), v[1]);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&fullA[sa]);
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------ epilogue
    const int quarter = warp - kEpiWarp0;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
      const Tile tl = tile_of(item, pre, E, a.wtiles, offs);
      const int ab = it & 1;
      if (!warp_wait(&accFull[ab], (it >> 1) & 1, a.err)) break;
      tc_fence_after();
      // the accumulator holds sum w' * x * act_scale (NVFP4: w' = e2m1 * e4m3, the
      // per-tensor scale still to apply)
      const float post = (FMT == MOE_FMT_NVFP4) ? 256.f * a.gs[tl.e] : 16.f;
      for (int c0 = 0; c0 < tl.nrows; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + uint32_t(ab * kTN + c0), v);
        tc_wait_ld();
        const int nc = min(32, tl.nrows - c0);
        if (MODE == kDown) {
          uint16_t* o = a.out + size_t(tl.r0 + c0) * a.out_ld + tl.wt * kTM + quarter * 32 + lane;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c < nc) o[size_t(c) * a.out_ld] = float_to_bf16_bits(__uint_as_float(v[c]) * post);
        } else {
          // lane l < 16 holds gate column i, lane l + 16 the up value of the same i
          uint16_t* o = a.out + size_t(tl.r0 + c0) * a.out_ld + tl.wt * 64 + quarter * 16 + (lane & 15);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float mine = __uint_as_float(v[c]) * post;
            const float up = __shfl_xor_sync(0xffffffffu, mine, 16);
            if (lane < 16 && c < nc) {
              const float hv = silu(mine) * up;
              o[size_t(c) * a.out_ld] = __half_as_ushort(__float2half_rn(hv * act_scale<FMT>()));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accEmpty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// xs[r] = x[sorted_pair[r] / k]: the token rows in routed order, written as the GEMM's
// fp16 B operand x * act_scale (x/16 for W4, x/256 for NVFP4); one warp per row, 16
// bytes per lane per step, four steps in flight.
template <int FMT>
__global__ void __launch_bounds__(256) k_gather_rows(const uint4* __restrict__ x, const int32_t* __restrict__ sorted_pair,
                                                     int P, int k, int row16, uint4* __restrict__ xs) {
  const int lane = threadIdx.x & 31;
  const int nwarps = int(gridDim.x) * (blockDim.x >> 5);
  for (int r = int(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < P; r += nwarps) {
    const uint4* src = x + int64_t(__ldg(sorted_pair + r) / k) * row16;
    uint4* dst = xs + int64_t(r) * row16;
    for (int c0 = 0; c0 < row16; c0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u + lane;
        if (c < row16) v[u] = __ldg(src + c);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u + lane;
        if (c < row16) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __half2 hh =
                __floats2half2_rn(bf16_lo(w[i]) * act_scale<FMT>(), bf16_hi(w[i]) * act_scale<FMT>());
            o[i] = *reinterpret_cast<const uint32_t*>(&hh);
          }
          dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map over a row-major [rows][cols] array with `row_bytes` between rows.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
                 uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static std::atomic<int> cached[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (!n) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int FMT, int MODE>
cudaError_t launch_umma_one(const CUtensorMap& tb, const CUtensorMap& tw, const UmmaArgs& a, cudaStream_t st) {
  static std::atomic<bool> raised[128] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!raised[dev].load(std::memory_order_relaxed)) {
    const cudaError_t err =
        cudaFuncSetAttribute(k_ffn_umma<FMT, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    raised[dev].store(true, std::memory_order_relaxed);
  }
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  k_ffn_umma<FMT, MODE><<<nsm, kThreadsU, kSmemBytes, st>>>(tb, tw, a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- W4A4 on the FP4 tensor cores
// tcgen05.mma kind::mxf4nvf4 with block16 scales: A = 128 weight rows of E2M1 codes, B = 128
// routed rows of E2M1 codes, both from shared memory (K-major, 128-byte swizzle; 256 codes
// = 128 bytes per row per stage), their E4M3 block scales in tensor memory.  Per 64-element
// K block (one MMA) a scale block of 512 bytes holds, for tile row m = m0 + 32 m1 and its
// four 16-element sub-blocks kk, the byte 16 m0 + 4 m1 + kk; tcgen05.cp (32x128b, warpx4)
// puts it into four tensor-memory columns of every lane quarter: lane 32 r + m0, column m1,
// byte kk.  The weight scales are laid out that way once per set of experts from the
// row-major scales (k_sf_tiles_w, moe_w4a4_prepare); the activation scales in every call by
// the routed-row scatter (k_route_fp4_rows).
constexpr int kF4TM = 128, kF4TN = 128;
constexpr int kF4Stages = 3;                        // K stages of 256 elements (128 bytes per row)
// Two CTAs per SM, each with one accumulator buffer: one CTA's epilogue overlaps the other's
// main loop (measured faster than one CTA with six stages and two accumulator buffers).
constexpr int kF4AccBufs = 1;
constexpr int kF4TmemCols = 256;                    // per CTA: two CTAs share the SM's 512 columns
constexpr int kF4ABytes = kF4TM * 128, kF4BBytes = kF4TN * 128, kF4SfBytes = 4 * 512;
constexpr int kF4StageBytes = kF4ABytes + kF4BBytes + 2 * kF4SfBytes;  // 36 KiB
constexpr int kF4OffPre = kF4Stages * kF4StageBytes;
constexpr int kF4NumBars = 2 * kF4Stages + 4;
// shared memory after the stages: the row-tile prefix and the routing offsets ([E+1] each),
// the barriers, the tensor-memory slot; + 1024 bytes of alignment slack.  E <= 256 keeps
// two CTAs per SM (~112 KiB each); larger E runs one.
__host__ __device__ constexpr int f4_offs_bytes(int E) { return ((E + 1) * 4 + 255) / 256 * 256; }
__host__ __device__ constexpr int f4_smem_bytes(int E) {
  return kF4OffPre + 2 * f4_offs_bytes(E) + kF4NumBars * 8 + 16 + 1024;
}
constexpr int kF4SmemMax = f4_smem_bytes(MOE_MAX_EXPERTS);
constexpr int kF4Threads = 256;                     // producer, MMA, 2 idle, 4 epilogue warps
// tensor-memory columns: the accumulator at 0, the scales of stage s at 128 + 32 s (A) and
// 144 + 32 s (B), 4 columns per 64-element K block
constexpr uint32_t kF4SfaCol = kF4AccBufs * kF4TN, kF4SfbCol = kF4AccBufs * kF4TN + 16, kF4SfStageCols = 32;
static_assert(kF4SfaCol + kF4Stages * kF4SfStageCols <= kF4TmemCols, "tensor-memory plan");
static_assert(kF4SmemMax <= 227 * 1024, "shared-memory plan");
static_assert(2 * f4_smem_bytes(256) + 2048 <= 228 * 1024, "two CTAs per SM at E <= 256");
static_assert(kF4StageBytes % 1024 == 0, "stage alignment for the 128-byte swizzle");

struct F4Args {
  int K, I, E, wtiles, n_rows;
  const int32_t* offsets;
  const uint8_t* sfa;       // weight scales, tiled: [E][wtiles][K/64][512]
  const uint8_t* sfb;       // activation scales, tiled: [row tiles][K/64][512]
  const float* gs;          // per-expert weight scale of this matrix [E]
  const float* act_amax;    // amax of the activation tensor (scale amax / 2688)
  uint16_t* out;            // down: y bf16 [P][H]
  int out_ld;
  float* out_f32;           // gate/up: h fp32 [P][I]
  float* out_amax;          // gate/up: amax of h
  unsigned* err;
};

// Shared-memory descriptor of a 512-byte scale block for tcgen05.cp: K-major, no swizzle,
// 16-byte rows, 8-row core matrices 128 bytes apart.
MOE_DEVICE uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t(1) << 16;          // leading byte offset (one core matrix along K)
  d |= uint64_t(128 >> 4) << 32;   // stride byte offset: next 8 rows
  d |= uint64_t(1) << 46;          // descriptor version
  return d;                        // layout type 0: no swizzle
}
MOE_DEVICE void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T with E4M3 block-16 scales from tensor memory; M = 128, K = 64.
MOE_DEVICE void tc_mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t sfa,
                           uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}
// Instruction descriptor (block-scaled): A and B E2M1 (format 1), K-major, E4M3 scales,
// N = 128, M = 128, scale ids 0.
constexpr uint32_t kF4Idesc = (1u << 7) | (1u << 10) | (uint32_t(kF4TN >> 3) << 17) | (uint32_t(kF4TM >> 4) << 24);

MOE_DEVICE Tile tile_of_n(int item, const int* pre, int E, int wtiles, const int* offsets, int tn, int* rtile) {
  const int t = item / wtiles;
  Tile tl;
  tl.wt = item - t * wtiles;
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pre[mid] <= t) lo = mid;
    else hi = mid;
  }
  tl.e = lo;
  const int beg = offsets[lo], end = offsets[lo + 1];
  tl.r0 = beg + (t - pre[lo]) * tn;
  tl.nrows = min(tn, end - tl.r0);
  *rtile = t;
  return tl;
}

template <int MODE>
__global__ void __launch_bounds__(kF4Threads, 2)
    k_ffn_fp4(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_w, F4Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  const int E = a.E;
  int* pre = reinterpret_cast<int*>(smem + kF4OffPre);
  int* offs = reinterpret_cast<int*>(smem + kF4OffPre + f4_offs_bytes(E));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kF4OffPre + 2 * f4_offs_bytes(E));
  uint64_t* full = bars;
  uint64_t* empty = full + kF4Stages;
  uint64_t* accFull = empty + kF4Stages;
  uint64_t* accEmpty = accFull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kF4NumBars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int i = tid; i <= E; i += blockDim.x) offs[i] = a.offsets[i];
  __syncthreads();
  if (warp == 0) {  // row tiles of kF4TN per expert, and their prefix
    const int per = (E + 31) / 32;
    const int b = min(E, lane * per), en = min(E, b + per);
    int sum = 0;
    for (int e = b; e < en; ++e) sum += (offs[e + 1] - offs[e] + kF4TN - 1) / kF4TN;
    int inc = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += v;
    }
    int run = inc - sum;
    for (int e = b; e < en; ++e) {
      pre[e] = run;
      run += (offs[e + 1] - offs[e] + kF4TN - 1) / kF4TN;
    }
    if (lane == 31) pre[E] = inc;
  } else if (tid == 64) {
    for (int i = 0; i < kF4Stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accFull[i], 1);
      mbar_init(&accEmpty[i], 4);
    }
    fence_mbar_init();
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kF4TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = pre[E] * a.wtiles;
  const int KB64 = a.K / 64, KS = (KB64 + 3) / 4;  // the last stage may hold 2 of its 4 K blocks

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    int n = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      int rt = 0;
      const Tile tl = tile_of_n(item, pre, E, a.wtiles, offs, kF4TN, &rt);
      for (int ks = 0; ks < KS; ++ks, ++n) {
        const int s = n % kF4Stages;
        if (!warp_wait(&empty[s], ((n / kF4Stages) & 1) ^ 1, a.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const uint32_t st = sbase + s * kF4StageBytes;
          const uint32_t sf_bytes = uint32_t(min(4, KB64 - 4 * ks)) * 512u;
          mbar_arrive_expect_tx(&full[s], uint32_t(kF4ABytes + kF4BBytes) + 2 * sf_bytes);
          if (MODE == kGateUp) {  // rows 32q..32q+15: gate rows 16q.., 32q+16..: the matching up rows
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int g0 = tl.e * a.n_rows + tl.wt * 64 + 16 * q;
              tma_load_2d(st + (32 * q) * 128, &tm_w, ks * 128, g0, &full[s]);
              tma_load_2d(st + (32 * q + 16) * 128, &tm_w, ks * 128, g0 + a.I, &full[s]);
            }
          } else {
            tma_load_2d(st, &tm_w, ks * 128, tl.e * a.n_rows + tl.wt * kF4TM, &full[s]);
          }
          tma_load_2d(st + kF4ABytes, &tm_b, ks * 128, tl.r0, &full[s]);
          bulk_g2s(smem + s * kF4StageBytes + kF4ABytes + kF4BBytes,
                   a.sfa + (size_t(tl.e * a.wtiles + tl.wt) * KB64 + 4 * ks) * 512, sf_bytes, &full[s]);
          bulk_g2s(smem + s * kF4StageBytes + kF4ABytes + kF4BBytes + kF4SfBytes,
                   a.sfb + (size_t(rt) * KB64 + 4 * ks) * 512, sf_bytes, &full[s]);
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (one thread)
    if (lane == 0) {
      int n = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
        const int ab = it % kF4AccBufs;
        if (!mbar_wait(&accEmpty[ab], ((it / kF4AccBufs) & 1) ^ 1, a.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + uint32_t(ab * kF4TN);
        for (int ks = 0; ks < KS; ++ks, ++n) {
          const int s = n % kF4Stages;
          if (!mbar_wait(&full[s], (n / kF4Stages) & 1, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * kF4StageBytes;
          const uint32_t sfa = tmem + kF4SfaCol + kF4SfStageCols * s, sfb = tmem + kF4SfbCol + kF4SfStageCols * s;
          const int nkb = min(4, KB64 - 4 * ks);
          const uint64_t adesc = sw128_desc(st), bdesc = sw128_desc(st + kF4ABytes);
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            if (kb < nkb) {
              tc_cp_sf(sfa + 4 * kb, sf_desc(st + kF4ABytes + kF4BBytes + 512 * kb));
              tc_cp_sf(sfb + 4 * kb, sf_desc(st + kF4ABytes + kF4BBytes + kF4SfBytes + 512 * kb));
            }
          }
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)  // 32 bytes (64 codes) per MMA inside the 128-byte row
            if (kb < nkb)
              tc_mma_fp4(d_tmem, adesc + uint64_t(2 * kb), bdesc + uint64_t(2 * kb), kF4Idesc, sfa + 4 * kb,
                         sfb + 4 * kb, (ks | kb) != 0);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&accFull[ab]);
      }
      if (it > 0 && ok) mbar_wait(&accFull[(it - 1) % kF4AccBufs], ((it - 1) / kF4AccBufs) & 1, a.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue
    const int quarter = warp - 4;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
      int rt = 0;
      const Tile tl = tile_of_n(item, pre, E, a.wtiles, offs, kF4TN, &rt);
      const int ab = it % kF4AccBufs;
      if (!warp_wait(&accFull[ab], (it / kF4AccBufs) & 1, a.err)) break;
      tc_fence_after();
      const float post = a.gs[tl.e] * __fdiv_rn(*a.act_amax, 2688.0f);
      float amax = 0.f;
      for (int c0 = 0; c0 < tl.nrows; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + uint32_t(ab * kF4TN + c0), v);
        tc_wait_ld();
        const int nc = min(32, tl.nrows - c0);
        if (MODE == kDown) {
          uint16_t* o = a.out + size_t(tl.r0 + c0) * a.out_ld + tl.wt * kF4TM + quarter * 32 + lane;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c < nc) o[size_t(c) * a.out_ld] = float_to_bf16_bits(__uint_as_float(v[c]) * post);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float mine = __uint_as_float(v[c]) * post;
            const float up = __shfl_xor_sync(0xffffffffu, mine, 16);
            if (lane < 16 && c < nc) {
              const float hv = silu(mine) * up;
              a.out_f32[size_t(tl.r0 + c0 + c) * a.out_ld + tl.wt * 64 + quarter * 16 + lane] = hv;
              amax = fmaxf(amax, fabsf(hv));
            }
          }
        }
      }
      if (MODE == kGateUp) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) atomicMax(reinterpret_cast<unsigned*>(a.out_amax), __float_as_uint(amax));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accEmpty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kF4TmemCols);
  }
}

// Weight scales, row-major E4M3 [E][N][K/16] -> tiled [E][wtiles][K/64][512]: tile wt, K block
// kb, tile row m = m0 + 32 m1 (gate/up: m1 = q, m0 < 16 the gate row 64 wt + 16 q + m0, else
// the up row I + 64 wt + 16 q + m0 - 16; down: row 128 wt + m), byte 16 m0 + 4 m1 + kk.
// One thread per (E, wtile, kb, m0): 16 bytes.
__global__ void k_sf_tiles_w(const uint8_t* __restrict__ sb, int E, int N, int K, int I, int gate_up,
                             uint8_t* __restrict__ out) {
  const int KB = K / 64, wtiles = gate_up ? I / 64 : N / 128;
  const int64_t total = int64_t(E) * wtiles * KB * 32;
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= total) return;
  const int m0 = int(i % 32);
  int64_t r = i / 32;
  const int kb = int(r % KB);
  r /= KB;
  const int wt = int(r % wtiles);
  const int e = int(r / wtiles);
  uint32_t w[4];
#pragma unroll
  for (int m1 = 0; m1 < 4; ++m1) {
    int row;
    if (gate_up) row = (m0 < 16) ? 64 * wt + 16 * m1 + m0 : I + 64 * wt + 16 * m1 + (m0 - 16);
    else row = 128 * wt + 32 * m1 + m0;
    w[m1] = *reinterpret_cast<const uint32_t*>(sb + (size_t(e) * N + row) * (K / 16) + 4 * kb);
  }
  *reinterpret_cast<uint4*>(out + ((size_t(e) * wtiles + wt) * KB + kb) * 512 + 16 * m0) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Row tiles of kF4TN routed rows per expert: pre[e] for e <= E (one CTA).
__global__ void __launch_bounds__(1024) k_row_tile_prefix(const int32_t* __restrict__ offsets, int E,
                                                          int32_t* __restrict__ pre) {
  __shared__ int part[1024];
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int b = min(E, int(threadIdx.x) * per), en = min(E, b + per);
  int sum = 0;
  for (int e = b; e < en; ++e) sum += (offsets[e + 1] - offsets[e] + kF4TN - 1) / kF4TN;
  part[threadIdx.x] = sum;
  __syncthreads();
  for (int d = 1; d < int(blockDim.x); d <<= 1) {
    const int v = int(threadIdx.x) >= d ? part[threadIdx.x - d] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int run = part[threadIdx.x] - sum;
  for (int e = b; e < en; ++e) {
    pre[e] = run;
    run += (offsets[e + 1] - offsets[e] + kF4TN - 1) / kF4TN;
  }
  if (threadIdx.x == blockDim.x - 1) pre[E] = part[threadIdx.x];
}

// B operand rows in routed order and their tiled scales: routed row r of expert e (tile
// pre[e] + (r - off_e) / 128, tile row n = (r - off_e) % 128) takes the codes of source row
// src(r) (gate/up: its token; down: r) and scatters its E4M3 scales to byte 16 (n % 32) +
// 4 (n / 32) + kk of K block kb.  One thread per (row, K block of 64): 32 code bytes, 4 scales.
__global__ void k_route_fp4_rows(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sb,
                                 const int32_t* __restrict__ sorted_pair, int k, const int32_t* __restrict__ offsets,
                                 int E, const int32_t* __restrict__ pre, int P, int K, uint8_t* __restrict__ codes_out,
                                 uint8_t* __restrict__ sf_out) {
  const int KB = K / 64;
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i >= int64_t(P) * KB) return;
  const int r = int(i / KB), kb = int(i - int64_t(r) * KB);
  int lo = 0, hi = E;  // expert of row r: largest e with offsets[e] <= r
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= r) lo = mid;
    else hi = mid;
  }
  const int nrow = r - offsets[lo];
  const int tile = pre[lo] + nrow / kF4TN, n = nrow % kF4TN;
  const int64_t src = sorted_pair ? int64_t(sorted_pair[r] / k) : int64_t(r);
  if (codes_out) {
    const uint4* cs = reinterpret_cast<const uint4*>(codes + src * (K / 2) + kb * 32);
    uint4* cd = reinterpret_cast<uint4*>(codes_out + int64_t(r) * (K / 2) + kb * 32);
    cd[0] = cs[0];
    cd[1] = cs[1];
  }
  const uint32_t s4 = *reinterpret_cast<const uint32_t*>(sb + src * (K / 16) + 4 * kb);
  *reinterpret_cast<uint32_t*>(sf_out + (size_t(tile) * KB + kb) * 512 + 16 * (n % 32) + 4 * (n / 32)) = s4;
}

template <int MODE>
cudaError_t launch_fp4_one(const CUtensorMap& tb, const CUtensorMap& tw, const F4Args& a, cudaStream_t st) {
  static std::atomic<bool> raised[128] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!raised[dev].load(std::memory_order_relaxed)) {
    const cudaError_t err = cudaFuncSetAttribute(k_ffn_fp4<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kF4SmemMax);
    if (err != cudaSuccess) return err;
    raised[dev].store(true, std::memory_order_relaxed);
  }
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  k_ffn_fp4<MODE><<<2 * nsm, kF4Threads, f4_smem_bytes(a.E), st>>>(tb, tw, a);
  return cudaGetLastError();
}

}  // namespace

// At 32 or more rows per expert on average, the tensor-core GEMM (weights
// dequantised once per 192 rows) beats streaming the weights once per 16 rows.
bool use_umma_path(int64_t T, int64_t E, int64_t k, moe_format_t fmt) {
  return (fmt == MOE_FMT_W4G128 || fmt == MOE_FMT_NVFP4) && T * k >= 32 * E;
}

static size_t align256u(size_t b) { return (b + 255) / 256 * 256; }
size_t umma_h_bytes(int64_t T, int64_t I, int64_t k) { return align256u(size_t(T * k * I * 2)); }
// h [P][I], then the routed token rows [P][H] (fp16: x/16 for W4, x/256 for NVFP4)
size_t umma_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t k) {
  return umma_h_bytes(T, I, k) + align256u(size_t(T * k * H * 2));
}

template <int FMT>
static cudaError_t launch_umma_fmt(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex, int T, int H,
                                   int I, int E, int k, uint16_t* y_rows, void* hbuf, cudaStream_t st) {
  const int P = T * k;
  UmmaArgs a{};
  a.E = E;
  a.k = k;
  a.I = I;
  a.offsets = r.expert_offsets;
  a.sorted_pair = r.sorted_pair;
  a.min_rows = kSmallRows + 1;
  a.err = device_error_word();
  if (!a.err) return cudaErrorInvalidDevice;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const CUtensorMapDataType act_type = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  // the token rows in routed order, after h in the workspace
  uint16_t* xs = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(hbuf) + umma_h_bytes(T, I, k));
  k_gather_rows<FMT><<<4 * nsm, 256, 0, st>>>(reinterpret_cast<const uint4*>(x), r.sorted_pair, P, k, H / 8,
                                              reinterpret_cast<uint4*>(xs));
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  CUtensorMap tb, tw;
  // gate/up: routed token rows, two 64-K boxes per stage; weight boxes of 64 gate and 64 up
  // rows (packed W4 words and E2M1 codes both take K/2 bytes per row)
  if (!make_map_2d(&tb, act_type, xs, uint64_t(H), uint64_t(P), uint64_t(H) * 2, kAtomK, kTN,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, ex.w13, uint64_t(H) / 2, uint64_t(E) * 2 * I,
                   uint64_t(H) / 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  a.K = H;
  a.n_rows = 2 * I;
  a.wtiles = I / 64;
  a.s = static_cast<const uint16_t*>(ex.w13_scale);
  a.bs = static_cast<const uint8_t*>(ex.w13_scale);
  a.gs = ex.w13_gscale;
  a.out = static_cast<uint16_t*>(hbuf);
  a.out_ld = I;
  err = launch_umma_one<FMT, kGateUp>(tb, tw, a, st);
  if (err != cudaSuccess) return err;
  err = launch_gemv_small(x, r, ex, T, H, I, E, k, hbuf, y_rows, false, kSmallRows, st);
  if (err != cudaSuccess) return err;
  // down: h rows, two 64-K boxes per stage; weight boxes of 128 rows
  if (!make_map_2d(&tb, act_type, hbuf, uint64_t(I), uint64_t(P), uint64_t(I) * 2, kAtomK, kTN,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, ex.w2, uint64_t(I) / 2, uint64_t(E) * H, uint64_t(I) / 2, 64,
                   kTM, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  a.K = I;
  a.n_rows = H;
  a.wtiles = H / kTM;
  a.s = static_cast<const uint16_t*>(ex.w2_scale);
  a.bs = static_cast<const uint8_t*>(ex.w2_scale);
  a.gs = ex.w2_gscale;
  a.out = y_rows;
  a.out_ld = H;
  err = launch_umma_one<FMT, kDown>(tb, tw, a, st);
  if (err != cudaSuccess) return err;
  return launch_gemv_small(x, r, ex, T, H, I, E, k, hbuf, y_rows, true, kSmallRows, st);
}

cudaError_t launch_grouped_ffn_umma(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex, int T,
                                    int H, int I, int E, int k, uint16_t* y_rows, void* hbuf, cudaStream_t st) {
  if (ex.fmt == MOE_FMT_W4G128)
    return launch_umma_fmt<MOE_FMT_W4G128>(x, r, ex, T, H, I, E, k, y_rows, hbuf, st);
  if (ex.fmt == MOE_FMT_NVFP4) return launch_umma_fmt<MOE_FMT_NVFP4>(x, r, ex, T, H, I, E, k, y_rows, hbuf, st);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------- W4A4 (NVFP4 activations)
// Weight scales in the tensor-memory copy order, written once per set of experts: w13's
// [E][I/64][H/64][512] (gate/up tiles interleave 16 gate and 16 up rows), then w2's
// [E][H/128][I/64][512].
size_t w4a4_scale_tiles_bytes(int64_t H, int64_t I, int64_t E) {
  return align256u(size_t(E * 2 * I * H / 16)) + align256u(size_t(E * H * I / 16));
}

cudaError_t launch_w4a4_prepare(const moe_experts_t& ex, int H, int I, int E, uint8_t* tiles, cudaStream_t st) {
  const int64_t n13 = int64_t(E) * (I / 64) * (H / 64) * 32, n2 = int64_t(E) * (H / 128) * (I / 64) * 32;
  k_sf_tiles_w<<<unsigned((n13 + 255) / 256), 256, 0, st>>>(static_cast<const uint8_t*>(ex.w13_scale), E, 2 * I, H, I,
                                                            1, tiles);
  k_sf_tiles_w<<<unsigned((n2 + 255) / 256), 256, 0, st>>>(static_cast<const uint8_t*>(ex.w2_scale), E, H, I, I, 0,
                                                           tiles + align256u(size_t(int64_t(E) * 2 * I * H / 16)));
  return cudaGetLastError();
}

// Workspace: two amax words, the row-tile prefix, x codes [T][H/2] and scales [T][H/16], the
// routed x codes [P][H/2] and their tiled scales, h fp32 [P][I], h codes [P][I/2] and scales
// [P][I/16], and h's tiled scales.
struct W4a4Plan {
  size_t amax, pre, xc, xsb, bxc, sfbx, hf, hc, hsb, sfbh, total;
};
static W4a4Plan w4a4_plan(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
  const int64_t P = T * k, tiles = P / kF4TN + E;  // row tiles: sum over experts of ceil(n_e / 128)
  W4a4Plan p{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += align256u(bytes);
    return at;
  };
  p.amax = take(256);
  p.pre = take(size_t(E + 1) * 4);
  p.xc = take(size_t(T * H / 2));
  p.xsb = take(size_t(T * H / 16));
  p.bxc = take(size_t(P * H / 2));
  p.sfbx = take(size_t(tiles * (H / 64) * 512));
  p.hf = take(size_t(P * I * 4));
  p.hc = take(size_t(P * I / 2));
  p.hsb = take(size_t(P * I / 16));
  p.sfbh = take(size_t(tiles * (I / 64) * 512));
  p.total = o;
  return p;
}

size_t w4a4_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
  return w4a4_plan(T, H, I, E, k).total;
}

cudaError_t launch_grouped_ffn_w4a4(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex,
                                    const uint8_t* tiles, int T, int H, int I, int E, int k, uint16_t* y_rows,
                                    void* ws, cudaStream_t st) {
  const int P = T * k;
  const W4a4Plan pl = w4a4_plan(T, H, I, E, k);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* amax_x = reinterpret_cast<float*>(base + pl.amax);
  float* amax_h = amax_x + 1;
  int32_t* pre = reinterpret_cast<int32_t*>(base + pl.pre);
  cudaError_t err;
  k_row_tile_prefix<<<1, 1024, 0, st>>>(r.expert_offsets, E, pre);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  // x -> NVFP4 (one tensor), then its codes in routed-row order and its scales tiled
  err = launch_act_nvfp4<uint16_t>(x, int64_t(T) * H, base + pl.xc, base + pl.xsb, amax_x, st);
  if (err != cudaSuccess) return err;
  int64_t nb = int64_t(P) * (H / 64);
  k_route_fp4_rows<<<unsigned((nb + 255) / 256), 256, 0, st>>>(base + pl.xc, base + pl.xsb, r.sorted_pair, k,
                                                               r.expert_offsets, E, pre, P, H, base + pl.bxc,
                                                               base + pl.sfbx);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if ((err = cudaMemsetAsync(amax_h, 0, sizeof(float), st)) != cudaSuccess) return err;
  F4Args a{};
  a.E = E;
  a.I = I;
  a.offsets = r.expert_offsets;
  a.err = device_error_word();
  if (!a.err) return cudaErrorInvalidDevice;
  CUtensorMap tb, tw;
  // gate/up: weight boxes of 16 rows (gate and up interleaved per 16), B boxes of 128 rows
  if (!make_map_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, base + pl.bxc, uint64_t(H) / 2, uint64_t(P), uint64_t(H) / 2,
                   128, kF4TN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, ex.w13, uint64_t(H) / 2, uint64_t(E) * 2 * I,
                   uint64_t(H) / 2, 128, 16, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  a.K = H;
  a.n_rows = 2 * I;
  a.wtiles = I / 64;
  a.sfa = tiles;
  a.sfb = base + pl.sfbx;
  a.gs = ex.w13_gscale;
  a.act_amax = amax_x;
  a.out = nullptr;
  a.out_ld = I;
  a.out_f32 = reinterpret_cast<float*>(base + pl.hf);
  a.out_amax = amax_h;
  err = launch_fp4_one<kGateUp>(tb, tw, a, st);
  if (err != cudaSuccess) return err;
  // h (fp32, its amax taken by the epilogue) -> NVFP4 codes in routed order; scales tiled
  err = launch_act_nvfp4_codes<float>(reinterpret_cast<const float*>(base + pl.hf), int64_t(P) * I, base + pl.hc,
                                      base + pl.hsb, amax_h, st);
  if (err != cudaSuccess) return err;
  nb = int64_t(P) * (I / 64);
  k_route_fp4_rows<<<unsigned((nb + 255) / 256), 256, 0, st>>>(nullptr, base + pl.hsb, nullptr, 1, r.expert_offsets,
                                                               E, pre, P, I, nullptr, base + pl.sfbh);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if (!make_map_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, base + pl.hc, uint64_t(I) / 2, uint64_t(P), uint64_t(I) / 2,
                   128, kF4TN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, ex.w2, uint64_t(I) / 2, uint64_t(E) * H, uint64_t(I) / 2, 128,
                   kF4TM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  a.K = I;
  a.n_rows = H;
  a.wtiles = H / kF4TM;
  a.sfa = tiles + align256u(size_t(int64_t(E) * 2 * I * H / 16));
  a.sfb = base + pl.sfbh;
  a.gs = ex.w2_gscale;
  a.act_amax = amax_h;
  a.out = y_rows;
  a.out_ld = H;
  a.out_f32 = nullptr;
  a.out_amax = nullptr;
  return launch_fp4_one<kDown>(tb, tw, a, st);
}

}  // namespace moe
