// Grouped FFN for prefill-sized batches on the fifth-generation tensor cores
// (tcgen05, accumulators in tensor memory).
//
// Per expert e, the routed rows r in [off_e, off_{e+1}) (sorted order) are
//   gate/up:  g, u = x[token(r)] . deq(W13_e)^T,  h[r] = silu(g) * u   (bf16)
//   down:     y[r] = h[r] . deq(W2_e)^T                                 (bf16)
// i.e. the same contraction as the weight-streaming GEMV, organised as a GEMM
// when each expert sees enough rows for the weights to be worth reusing.
//
// Tile = 128 weight rows (the tensor-memory lanes, MMA M) x up to 128 rows of the
// expert (MMA N) x the whole K.  For gate/up, the 128 weight rows are 64 gate rows
// and the 64 matching up rows, arranged so that each warp quarter of the lanes
// holds 16 gate rows and their 16 up rows: the SwiGLU product is formed in the
// epilogue with one lane exchange.
// Roles inside one persistent CTA (one per SM, 384 threads):
//   warps 0-1   copy the B operand (token rows, bf16) with cp.async into a 6-stage
//               ring of 128-byte-swizzled K-major tiles in shared memory;
//   warp  2     allocates tensor memory and issues tcgen05.mma (kind::f16, bf16 in,
//               fp32 accumulate) from one thread, A from tensor memory, B from
//               shared memory; tcgen05.commit releases the stages;
//   warps 4-7   dequantise the packed weights of their 32 rows each straight into
//               tensor memory (tcgen05.st, 4 stages of 64 K-elements): the weight
//               operand never passes through shared memory;
//   warps 8-11  drain one of the two accumulators (tcgen05.ld) while the other is
//               being accumulated, apply SwiGLU, and store bf16 rows.
// The work list (expert, row tile, weight tile) is built by every CTA from the
// routing offsets and walked round-robin across CTAs.
//
// Dequantisation (W4 group-128): (u - 8) * s with u the stored nibble and s the
// group's bf16 scale, formed as bf16 (128 + u) by bit operations, then
// bf16 adds -136 exactly and multiplies by s with one rounding to bf16.  This is
// the only rounding that differs from the fp32 dequantisation of the definition
// (relative 2^-9 per weight, inside the FFN tolerance).
//
// Every wait is bounded (mbar_wait): a wait that runs out sets the device error
// word and the role stops; the CTA still frees its tensor memory.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kTM = 128;        // weight rows per tile (tensor-memory lanes)
constexpr int kTN = 128;        // rows of the expert per tile (MMA N at most)
constexpr int kKB = 64;         // K elements per block: one 128-byte swizzle row of bf16
constexpr int kBStages = 6;     // token-tile stages in shared memory
constexpr int kAStages = 4;     // dequantised weight stages in tensor memory
constexpr int kLag = 3;         // cp.async groups kept in flight before a stage is published
constexpr int kThreadsU = 384;
constexpr int kTmemCols = 512;  // accumulators at columns 0 and 128, A stages at 256 + 32 a
constexpr int kACol0 = 256;
constexpr int kBStageBytes = kTN * 128;
constexpr int kPrefetch = 4;    // k-blocks of packed weights held in registers ahead

constexpr int kProdThreads = 64;
constexpr int kMmaWarp = 2;
constexpr int kDeqWarp0 = 4;
constexpr int kEpiWarp0 = 8;

// shared memory plan (offsets from a 1024-byte aligned base)
constexpr int kOffB = 0;
constexpr int kOffPre = kOffB + kBStages * kBStageBytes;  // tile prefix over experts
constexpr int kOffBar = kOffPre + ((MOE_MAX_EXPERTS + 1) * 4 + 255) / 256 * 256;
constexpr int kNumBars = 2 * kBStages + 2 * kAStages + 4;
constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr int kSmemUsed = kOffTmemSlot + 16;
// + alignment slack; at least 120 KiB so that one CTA occupies an SM (and its
// tensor memory) alone
constexpr int kSmemBytes = (kSmemUsed + 1024) > 120 * 1024 ? (kSmemUsed + 1024) : 120 * 1024;

constexpr int kGateUp = 0, kDown = 1;

struct UmmaArgs {
  const uint16_t* act;       // gate/up: x [T][K]; down: h [P][K]
  int K, I, E, k;
  int wtiles;                // weight tiles per expert
  int n_rows;                // rows of one expert's weight matrix (2I or H)
  const int32_t* offsets;    // [E+1]
  const int32_t* sorted_pair;
  const uint32_t* w;         // packed W4 [E][n_rows][K/8]
  const uint16_t* s;         // bf16 scales [E][n_rows][K/128]
  uint16_t* out;             // gate/up: h [P][I]; down: y [P][H]
  int out_ld;
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

MOE_DEVICE void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
MOE_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
MOE_DEVICE void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
MOE_DEVICE void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
MOE_DEVICE void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
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
// Instruction descriptor: fp32 accumulate, bf16 A and B, both K-major, M = 128.
MOE_DEVICE uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kTM >> 4) << 24);
}

// ---------------------------------------------------------------- W4 dequant
// Two nibbles a (low half) and b (high half) as bf16x2 (128 + a, 128 + b).
// w holds elements 8i..8i+7 of one row (element j at bits 4j); the result pairs
// (0,1), (2,3), (4,5), (6,7) in p[0..3].
MOE_DEVICE void w4_word_pairs(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu;         // n0 n2 n4 n6
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // n1 n3 n5 n7
  const uint32_t u01 = __byte_perm(lo, hi, 0x5140);  // n0 n1 n2 n3
  const uint32_t u23 = __byte_perm(lo, hi, 0x7362);  // n4 n5 n6 n7
  const uint32_t k43 = 0x43434343u;
  p[0] = __byte_perm(u01, k43, 0x4140);
  p[1] = __byte_perm(u01, k43, 0x4342);
  p[2] = __byte_perm(u23, k43, 0x4140);
  p[3] = __byte_perm(u23, k43, 0x4342);
}

MOE_DEVICE uint32_t bf16x2_add(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hadd2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
MOE_DEVICE uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// ---------------------------------------------------------------- work list
struct Tile {
  int e, r0, nrows, wt;
};

MOE_DEVICE Tile tile_of(int item, const int* pre, int E, int wtiles, const int32_t* offsets) {
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

template <int MODE>
__global__ void __launch_bounds__(kThreadsU, 1) k_ffn_umma(UmmaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  int* pre = reinterpret_cast<int*>(smem + kOffPre);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* fullB = bars;
  uint64_t* emptyB = bars + kBStages;
  uint64_t* fullA = bars + 2 * kBStages;
  uint64_t* emptyA = fullA + kAStages;
  uint64_t* accFull = emptyA + kAStages;
  uint64_t* accEmpty = accFull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;

  // ---- tiles per expert and their prefix (warp 0), barriers (thread 32), tensor memory (warp 2)
  if (warp == 0) {
    const int per = (E + 31) / 32;
    const int b = min(E, lane * per), en = min(E, b + per);
    int sum = 0;
    for (int e = b; e < en; ++e) sum += (a.offsets[e + 1] - a.offsets[e] + kTN - 1) / kTN;
    int inc = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += v;
    }
    int run = inc - sum;
    for (int e = b; e < en; ++e) {
      pre[e] = run;
      run += (a.offsets[e + 1] - a.offsets[e] + kTN - 1) / kTN;
    }
    if (lane == 31) pre[E] = inc;
  } else if (tid == 32) {
    for (int i = 0; i < kBStages; ++i) {
      mbar_init(&fullB[i], kProdThreads);
      mbar_init(&emptyB[i], 1);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&fullA[i], 4);
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

  if (tid < kProdThreads) {
    // ------------------------------------------------ B producer (token rows)
    // thread: chunk c = tid % 8 of rows rr = tid / 8 + 8 i (i < 16); the chunk lands
    // at c ^ (row % 8) = c ^ (tid / 8) inside its 128-byte row
    const int c = tid & 7, rsub = tid >> 3;
    const uint32_t dst_off = uint32_t(rsub * 128 + ((c ^ rsub) << 4));
    int n = 0;  // stages issued
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const Tile tl = tile_of(item, pre, E, a.wtiles, a.offsets);
      // gate/up: the token of each row; down: rows r0 + rr of h, 8 rows apart
      const uint16_t* src[MODE == kGateUp ? 16 : 1];
      if (MODE == kGateUp) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int rr = rsub + 8 * i;
          const int r = tl.r0 + (rr < tl.nrows ? rr : 0);
          src[i] = a.act + size_t(a.sorted_pair[r] / a.k) * a.K + c * 8;
        }
      } else {
        src[0] = a.act + size_t(tl.r0 + rsub) * a.K + c * 8;
      }
      for (int kb = 0; kb < KB; ++kb, ++n) {
        const int st = n % kBStages;
        if (!mbar_wait(&emptyB[st], ((n / kBStages) & 1) ^ 1, a.err)) {
          ok = false;
          break;
        }
        const uint32_t dst = sbase + kOffB + st * kBStageBytes + dst_off;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (rsub + 8 * i < tl.nrows)
            cp_async16(dst + i * 1024, (MODE == kGateUp ? src[i] : src[0] + size_t(8 * i) * a.K) + kb * kKB);
        cp_async_commit();
        if (n >= kLag) {
          cp_async_wait<kLag>();
          fence_async_smem();
          mbar_arrive(&fullB[(n - kLag) % kBStages]);
        }
      }
    }
    // publish the stages still in flight
    cp_async_wait<0>();
    fence_async_smem();
    for (int m = (n > kLag ? n - kLag : 0); m < n; ++m) mbar_arrive(&fullB[m % kBStages]);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer
    int nb = 0, na = 0, it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
      const Tile tl = tile_of(item, pre, E, a.wtiles, a.offsets);
      const int ab = it & 1;
      if (!warp_wait(&accEmpty[ab], ((it >> 1) & 1) ^ 1, a.err)) break;
      tc_fence_after();
      const int nmma = (tl.nrows + 15) & ~15;
      const uint32_t idesc = idesc_bf16(nmma);
      const uint32_t d_tmem = tmem + uint32_t(ab * kTN);
      for (int kb = 0; kb < KB; ++kb, ++nb, ++na) {
        const int sb = nb % kBStages, sa = na % kAStages;
        if (!warp_wait(&fullB[sb], (nb / kBStages) & 1, a.err) || !warp_wait(&fullA[sa], (na / kAStages) & 1, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t b_addr = sbase + kOffB + sb * kBStageBytes;
          const uint32_t a_tmem = tmem + uint32_t(kACol0 + sa * 32);
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk)
            tc_mma_ts(d_tmem, a_tmem + kk * 8, sw128_desc(b_addr + kk * 32), idesc, (kb | kk) != 0);
          tc_commit(&emptyB[sb]);
          tc_commit(&emptyA[sa]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) tc_commit(&accFull[ab]);
      __syncwarp();
    }
    // the last accumulation must be complete before the tensor memory is freed
    if (it > 0 && ok) mbar_wait(&accFull[(it - 1) & 1], (((it - 1) >> 1) & 1), a.err);
  } else if (warp >= kDeqWarp0 && warp < kDeqWarp0 + 4) {
    // ------------------------------------------------ dequantise W into tensor memory
    // This CTA's k-blocks form one stream (its items in order, K blocks each); the
    // packed words and scale of block g + kPrefetch are requested while block g is
    // converted, across item boundaries too.
    const int quarter = warp - kDeqWarp0;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const int KW = a.K / 8, KG = a.K / 128;
    const int my_items = blockIdx.x < n_items ? (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
    const int total = my_items * KB;
    // weight row of this lane in tile column wt: for gate/up, lanes 0-15 of each
    // quarter hold gate rows and lanes 16-31 the up rows of the same 16 columns
    auto row_of = [&](int item) -> size_t {
      const Tile tl = tile_of(item, pre, E, a.wtiles, a.offsets);
      int n;
      if (MODE == kGateUp) {
        const int i = tl.wt * 64 + quarter * 16 + (lane & 15);
        n = (lane < 16) ? i : a.I + i;
      } else {
        n = tl.wt * kTM + quarter * 32 + lane;
      }
      return size_t(tl.e) * a.n_rows + n;
    };
    int p_idx = -1;  // local item index whose row pointers are cached
    const uint4* p_wp = nullptr;
    const uint16_t* p_sp = nullptr;
    auto fetch = [&](int g, uint4& w0, uint4& w1, uint16_t& sv) {
      const int li = g / KB, kb = g - li * KB;
      if (li != p_idx) {
        p_idx = li;
        const size_t row = row_of(int(blockIdx.x) + li * int(gridDim.x));
        p_wp = reinterpret_cast<const uint4*>(a.w + row * KW);
        p_sp = a.s + row * KG;
      }
      w0 = ldg_nc_v4(p_wp + 2 * kb);
      w1 = ldg_nc_v4(p_wp + 2 * kb + 1);
      sv = p_sp[kb >> 1];
    };
    uint4 ring0[kPrefetch], ring1[kPrefetch];
    uint16_t rings[kPrefetch];
#pragma unroll
    for (int q = 0; q < kPrefetch; ++q)
      if (q < total) fetch(q, ring0[q], ring1[q], rings[q]);
    bool ok = true;
    for (int g0 = 0; g0 < total && ok; g0 += kPrefetch) {
#pragma unroll
      for (int q = 0; q < kPrefetch; ++q) {
        const int g = g0 + q;
        if (g >= total) break;
        const uint4 w0 = ring0[q], w1 = ring1[q];
        const uint32_t sv = rings[q];
        if (g + kPrefetch < total) fetch(g + kPrefetch, ring0[q], ring1[q], rings[q]);
        const uint32_t s2 = sv | (sv << 16);
        const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t p[4];
          w4_word_pairs(words[i], p);
#pragma unroll
          for (int j = 0; j < 4; ++j) v[4 * i + j] = bf16x2_mul(bf16x2_add(p[j], 0xC308C308u), s2);  // (u-8)*s
        }
        const int sa = g % kAStages;
        if (!warp_wait(&emptyA[sa], ((g / kAStages) & 1) ^ 1, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32(tmem + lane_base + uint32_t(kACol0 + sa * 32), v);
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
      const Tile tl = tile_of(item, pre, E, a.wtiles, a.offsets);
      const int ab = it & 1;
      if (!warp_wait(&accFull[ab], (it >> 1) & 1, a.err)) break;
      tc_fence_after();
      for (int c0 = 0; c0 < tl.nrows; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + uint32_t(ab * kTN + c0), v);
        tc_wait_ld();
        const int nc = min(32, tl.nrows - c0);
        if (MODE == kDown) {
          uint16_t* o = a.out + size_t(tl.r0 + c0) * a.out_ld + tl.wt * kTM + quarter * 32 + lane;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c < nc) o[size_t(c) * a.out_ld] = float_to_bf16_bits(__uint_as_float(v[c]));
        } else {
          // lane l < 16 holds gate column i, lane l + 16 the up value of the same i
          uint16_t* o = a.out + size_t(tl.r0 + c0) * a.out_ld + tl.wt * 64 + quarter * 16 + (lane & 15);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float mine = __uint_as_float(v[c]);
            const float up = __shfl_xor_sync(0xffffffffu, mine, 16);
            if (lane < 16 && c < nc) o[size_t(c) * a.out_ld] = float_to_bf16_bits(silu(mine) * up);
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

int sm_count() {
  static int cached[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 0;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int MODE>
cudaError_t launch_umma_one(const UmmaArgs& a, cudaStream_t st) {
  static bool raised[128] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  if (!raised[dev]) {
    const cudaError_t err = cudaFuncSetAttribute(k_ffn_umma<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    raised[dev] = true;
  }
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  k_ffn_umma<MODE><<<nsm, kThreadsU, kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

// At 32 or more rows per expert on average, the tensor-core GEMM (weights
// dequantised once per 128 rows) beats streaming the weights once per 16 rows.
bool use_umma_path(int64_t T, int64_t E, int64_t k, moe_format_t fmt) {
  return fmt == MOE_FMT_W4G128 && T * k >= 32 * E;
}

cudaError_t launch_grouped_ffn_umma(const uint16_t* x, const moe_routing_t& r, const moe_experts_t& ex, int T,
                                    int H, int I, int E, int k, uint16_t* y_rows, void* hbuf, cudaStream_t st) {
  (void)T;
  if (ex.fmt != MOE_FMT_W4G128) return cudaErrorInvalidValue;
  UmmaArgs a{};
  a.E = E;
  a.k = k;
  a.I = I;
  a.offsets = r.expert_offsets;
  a.sorted_pair = r.sorted_pair;
  a.err = device_error_word();
  if (!a.err) return cudaErrorInvalidDevice;
  // gate/up: weight tiles of 64 gate + 64 up rows
  a.act = x;
  a.K = H;
  a.n_rows = 2 * I;
  a.wtiles = I / 64;
  a.w = static_cast<const uint32_t*>(ex.w13);
  a.s = static_cast<const uint16_t*>(ex.w13_scale);
  a.out = static_cast<uint16_t*>(hbuf);
  a.out_ld = I;
  cudaError_t err = launch_umma_one<kGateUp>(a, st);
  if (err != cudaSuccess) return err;
  // down
  a.act = static_cast<const uint16_t*>(hbuf);
  a.K = I;
  a.n_rows = H;
  a.wtiles = H / kTM;
  a.w = static_cast<const uint32_t*>(ex.w2);
  a.s = static_cast<const uint16_t*>(ex.w2_scale);
  a.out = y_rows;
  a.out_ld = H;
  return launch_umma_one<kDown>(a, st);
}

}  // namespace moe
