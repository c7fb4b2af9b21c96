/*
 * moe.h -- C ABI of the low-bit routed-expert MoE FFN layer for NVIDIA B200 (sm_100a).
 *
 * One Mixture-of-Experts feed-forward layer whose routed experts hold low-bit
 * weights, run as: router logits -> top-k with softmax weights -> permutation of
 * the (token, slot) pairs by expert -> grouped SwiGLU expert GEMV/GEMM that
 * dequantises the weights in-kernel -> routing-weighted combine.
 *
 * Sources (web pages; cited by title and section):
 *   [ExactMoE]  "Every Expert Counts: ExactMoE for Memory-Efficient W4A16
 *               Inference", abstract: symmetric group-128 four-bit weights on the
 *               routed experts only, router kept in BF16, top-k unchanged, all
 *               selected experts executed by fused grouped kernels.
 *   [PagedMoE]  "PagedMoE: Cross-Precision Expert Caching for Token-Level Dynamic
 *               Precision in SSD-Resident MoE Inference", abstract: one stored
 *               expert state in a bitplane layout, lower precisions being
 *               prefixes of higher ones; prefix length chosen per token from the
 *               routing weights; prefixes executed directly.
 *   [MatMoE]    "MatMoE: Matryoshka Mixture-of-Experts with Dynamic Mixed-Precision
 *               Quantization for Efficient Inference", abstract: floor-and-
 *               compensation quantisation; bit-width per expert from routing scores.
 *   [MoET]      "MoET in FP4 MoE Inference" (Q&A page), answer and references:
 *               FP4/INT4 expert weights, router at higher precision, NVFP4.
 *   [DuoRate]   "DuoRate: Two-Rate Per-Expert Precision Allocation for Mixture-of-
 *               Experts Serving", key concepts: a resident and a routing-weighted
 *               read rate; a distortion tensor baked offline, unlabeled profiling,
 *               one dot product per expert and a bisection to a read budget.
 *
 * Conventions shared by every entry point
 *   - bf16 values are passed as uint16_t bit patterns.
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise, owned
 *     by the caller; the library never allocates, frees or keeps a pointer after
 *     the call returns.  Device pointers must be 16-byte aligned unless a call
 *     states a smaller alignment.
 *   - Every call only enqueues work on `stream` (a cudaStream_t; NULL means the
 *     legacy default stream) and returns without synchronising.
 *   - All arguments are validated on the host before anything is launched; an
 *     invalid call launches nothing and returns an error code.  A failed launch
 *     returns MOE_ERR_CUDA.  No C++ exception crosses the ABI.
 *   - T = 0 (no tokens) is valid and launches nothing, except where a call
 *     requires T >= 1 (the activation moments).
 *   - Shapes: weights are row-major [E][N][K] with K contiguous.  The gate/up
 *     matrix w13 of expert e is [2I][H] (rows 0..I-1 gate, I..2I-1 up); the down
 *     matrix w2 is [H][I].
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 2

/* Size limits enforced by validation. */
#define MOE_MAX_EXPERTS 1024 /* E */
#define MOE_MAX_TOPK 32      /* k */

typedef void* moe_stream_t; /* cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* a size outside the limits stated per call */
  MOE_ERR_WORKSPACE = 3,         /* workspace pointer null or smaller than required */
  MOE_ERR_CUDA = 4,              /* a CUDA launch or runtime call failed */
  MOE_ERR_MISALIGNED = 5,        /* a device pointer is not 16-byte aligned */
  MOE_ERR_DEVICE_TIMEOUT = 6     /* a kernel gave up waiting (see moe_check_device_errors) */
} moe_status_t;

typedef enum {
  MOE_FMT_W4G128 = 0,   /* INT4, symmetric, one bf16 scale per 128 K-elements [ExactMoE] */
  MOE_FMT_BITPLANE8 = 1,/* 8-bit symmetric codes stored as 8 bitplanes [PagedMoE], read at b planes */
  MOE_FMT_NVFP4 = 2     /* E2M1 + E4M3 scale per 16 + fp32 scale per expert matrix [MoET] */
} moe_format_t;

/* Routing of T tokens to k experts each; every array is device memory.
 * Pair p = t*k + j is token t's j-th choice. */
typedef struct {
  int32_t* topk_ids;       /* [T*k]  expert of pair p; slots ordered by logit descending, ties by lower id */
  float* topk_w;           /* [T*k]  routing weight of pair p (softmax over the token's k logits) */
  int32_t* expert_offsets; /* [E+1]  pairs routed to experts < e; offsets[E] = T*k */
  int32_t* sorted_pair;    /* [T*k]  pair held by sorted row r; ascending p inside each expert */
  int32_t* pair_to_row;    /* [T*k]  inverse of sorted_pair */
  int32_t* expert_list;    /* [E+1]  [0] = number A of experts with >= 1 pair, [1..A] their ids ascending */
} moe_routing_t;

/* Quantised expert weights (device memory), as written by the quantisers below.
 *   W4G128:    w13 uint32 [E][2I][H/8],  w13_scale bf16 [E][2I][H/128];
 *              w2  uint32 [E][H][I/8],   w2_scale  bf16 [E][H][I/128].
 *   BITPLANE8: w13 uint32 [E][8][2I][H/32], w13_scale bf16 [E][2I][H/128];
 *              w2  uint32 [E][8][H][I/32],  w2_scale  bf16 [E][H][I/128].
 *   NVFP4:     w13 uint8 [E][2I][H/2], w13_scale E4M3 uint8 [E][2I][H/16], w13_gscale fp32 [E];
 *              w2  uint8 [E][H][I/2],  w2_scale  E4M3 uint8 [E][H][I/16],  w2_gscale  fp32 [E]. */
typedef struct {
  moe_format_t fmt;
  const void* w13;
  const void* w13_scale;
  const void* w2;
  const void* w2_scale;
  const float* w13_gscale; /* NVFP4 only, else NULL */
  const float* w2_gscale;  /* NVFP4 only, else NULL */
} moe_experts_t;

/* Static string for a status code (never NULL). */
const char* moe_status_string(moe_status_t status);

/* MOE_ABI_VERSION of the loaded library. */
int moe_abi_version(void);

/* ------------------------------------------------------------------------
 * Offline weight preparation (not part of a layer step).
 * ------------------------------------------------------------------------ */

/* INT4 symmetric group-128 quantisation [ExactMoE].
 * Per row and per group of 128 consecutive K elements: scale = bf16(max|w| / 7)
 * (fp32 division, round to nearest even); q = clamp(rint(w / scale), -8, 7)
 * (fp32 division, ties to even); an all-zero group has scale 0 and q = 0.
 * Storage: u = q + 8, element k of a row in bits 4*(k%8).. of uint32 word k/8.
 *   w      bf16 [E][N][K];  packed uint32 [E][N][K/8];  scales bf16 [E][N][K/128].
 * Requires E, N >= 1, K >= 128, K % 128 == 0.  Bit-exact (integer decisions in IEEE fp32). */
moe_status_t moe_quantize_w4g128(const uint16_t* w, int64_t E, int64_t N, int64_t K,
                                 uint32_t* packed, uint16_t* scales, moe_stream_t stream);

/* 8-bitplane variable-precision form [PagedMoE bitplane prefixes; MatMoE floor and
 * compensation].  Per group of 128: scale = bf16(max|w| / 127); q = clamp(rint(w /
 * scale), -127, 127); u = q + 128 in 1..255.  Plane p (0..7) holds bit 7-p of u
 * (plane 0 = most significant), element k of a row in bit k%32 of word k/32.
 * A b-plane prefix is reconstructed as u' = ((u >> (8-b)) << (8-b)) + (b < 8 ? 1 << (7-b) : 0),
 * w' = scale * (u' - 128).
 *   w bf16 [E][N][K];  planes uint32 [E][8][N][K/32];  scales bf16 [E][N][K/128].
 * Requires K % 128 == 0.  Bit-exact. */
moe_status_t moe_pack_bitplanes(const uint16_t* w, int64_t E, int64_t N, int64_t K,
                                uint32_t* planes, uint16_t* scales, moe_stream_t stream);

/* NVFP4 quantisation [MoET, NVFP4 reference].  Per expert matrix (one [N][K] slice):
 * g = amax / (6 * 448) (fp32).  Per block of 16 consecutive K elements:
 * sb = E4M3_satfinite(amax_block / (6 * g)); code = E2M1_satfinite(w / (float(sb) * g)),
 * round to nearest even, a magnitude that rounds to zero is +0 (code 0); g == 0 or
 * sb == 0 gives codes 0.  Element 2i sits in the low nibble of byte i.
 *   w bf16 [E][N][K];  codes uint8 [E][N][K/2];  block_scales uint8 [E][N][K/16];  gscale fp32 [E].
 * gscale is also used as scratch during the call.  Requires K % 32 == 0.  Bit-exact. */
moe_status_t moe_quantize_nvfp4(const uint16_t* w, int64_t E, int64_t N, int64_t K,
                                uint8_t* codes, uint8_t* block_scales, float* gscale,
                                moe_stream_t stream);

/* NVFP4 quantisation of one fp32 tensor as a single scale unit (the activations of the
 * W4A4 prefill path [MoET: NVFP4]; same recipe as moe_quantize_nvfp4, with the whole
 * [R][C] tensor in place of one expert matrix).  a fp32 [R][C]; codes uint8 [R][C/2];
 * block_scales uint8 E4M3 [R][C/16]; gscale fp32 [1] (amax / 2688, also scratch).
 * Requires C % 16 == 0.  Bit-exact. */
moe_status_t moe_quantize_nvfp4_f32(const float* a, int64_t R, int64_t C, uint8_t* codes, uint8_t* block_scales,
                                    float* gscale, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * One layer step: route -> (select_bits) -> grouped_ffn -> combine
 * ------------------------------------------------------------------------ */

/* Bytes of device workspace moe_route_topk needs for (T, E, k). */
size_t moe_route_workspace_bytes(int64_t T, int64_t E, int64_t k);

/* Router logits, top-k, softmax weights and the stable permutation [ExactMoE: BF16
 * router, unchanged top-k; nothing pruned or substituted].
 * logits[t][e] = sum_h x[t][h] * w_router[e][h] (+ bias[e]) in fp32, in one fixed
 * order: 32 partial sums, partial L accumulating h = 256j + 8L + i for j outer,
 * i = 0..7 inner, by fused multiply-add from +0; the partials then added pairwise
 * at lane distance 16, 8, 4, 2, 1; then + bias.  Top-k: logit descending, equal
 * logits by ascending expert id.  Weights: w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)
 * over the k chosen.  Permutation: stable counting sort of the pairs by expert.
 *   x bf16 [T][H];  w_router bf16 [E][H];  bias fp32 [E] or NULL;  out: see moe_routing_t.
 * Requires H % 256 == 0, 1 <= E <= MOE_MAX_EXPERTS, 1 <= k <= min(E, MOE_MAX_TOPK),
 * T >= 0; workspace >= moe_route_workspace_bytes(T, E, k).  Workspace contents: the
 * FIRST 256 bytes hold a completion counter (used by the one-launch router of small
 * batches) that must be zero before the first call that uses this workspace (allocate
 * it zero-filled once, e.g. cudaMemset); every call leaves it zero again.  The fp32
 * logits follow it and are scratch, overwritten.  The counter's place does not depend
 * on (T, E, k), so a workspace sized for (T_max, E_max) serves any number of later
 * calls of any T <= T_max, E <= E_max, in any order.  Calls whose kernels overlap on
 * one workspace race on it.  The first call on a device sets the router kernels'
 * shared-memory attributes for that device (once); make one call before capturing a
 * stream into a graph.  Ids and permutation are deterministic. */
moe_status_t moe_route_topk(const uint16_t* x, const uint16_t* w_router, const float* bias,
                            int64_t T, int64_t H, int64_t E, int64_t k,
                            const moe_routing_t* out, void* workspace, size_t workspace_bytes,
                            moe_stream_t stream);

/* Maximum T * E accepted by moe_route_topk_noalloc (floats in its fixed array). */
#define MOE_NOALLOC_MAX_LOGITS 65536

/* moe_route_topk without a workspace argument.  No counterpart on the source pages:
 * it exists for callers that cannot allocate device memory -- an engine that plans
 * all device memory up front and hands a layer only fixed buffers, a custom-op host
 * that passes just inputs and outputs, or code running while a stream is captured
 * into a CUDA graph in global mode, where cudaMalloc is not allowed.
 * Same computation, arguments, results and errors as moe_route_topk, except that
 * the fp32 logits scratch and the completion counter are a fixed device array inside
 * the library (256 KiB + 256 bytes per GPU that loads the library, held until exit):
 * the logits fill its first T * E floats and the counter is the word right after the
 * 256 KiB, the same place for every shape (zero when the library loads; every call
 * leaves it zero), so calls of different shapes may follow one another in any order.
 *   - T * E must be <= MOE_NOALLOC_MAX_LOGITS, else MOE_ERR_UNSUPPORTED_SHAPE;
 *   - the library allocates nothing and frees nothing during the call;
 *   - all calls share the array: calls whose kernels overlap on one GPU (e.g. on two
 *     streams) race on it; serialise them;
 *   - the first call on a device looks up the array's address (cudaGetSymbolAddress
 *     with that device current), caches it and sets the router kernels' shared-memory
 *     attributes for that device; make that first call before any stream capture. */
moe_status_t moe_route_topk_noalloc(const uint16_t* x, const uint16_t* w_router, const float* bias,
                                    int64_t T, int64_t H, int64_t E, int64_t k,
                                    const moe_routing_t* out, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Budgeted bit allocation for bitplane experts (replaces the fixed thresholds of
 * moe_select_bits with a per-expert choice under a read budget)
 * ------------------------------------------------------------------------ */

/* Offline distortion table [DuoRate: a distortion tensor baked offline].  For expert
 * e, prefix length b = 1..8 and input channel k:
 *   delta[e][b-1][k] = sum_{n<N} (s[e][n][k/128] * (u'_b[e][n][k] - u[e][n][k]))^2,
 * u the stored 8-bit code, u'_b its b-bit floor-and-compensation prefix (0 for b = 8),
 * fp64, rows n in order.  Pass the gate/up matrix (K = H: the matrix that reads x).
 *   planes uint32 [E][8][N][K/32] and scales bf16 [E][N][K/128] as written by
 *   moe_pack_bitplanes;  delta fp64 [E][8][K] (caller-allocated).
 * Requires E, N >= 1, K % 128 == 0. */
moe_status_t moe_bitplane_distortion(const uint32_t* planes, const uint16_t* scales, int64_t E, int64_t N,
                                     int64_t K, double* delta, moe_stream_t stream);

/* Activation second moments of a workload's tokens [DuoRate: online profiling of a
 * workload's prefill, without labels]: m[k] = (1/T) sum_t x[t][k]^2, fp64, tokens in
 * order.   x bf16 [T][H];  m fp64 [H].  Requires T, H >= 1. */
moe_status_t moe_activation_moments(const uint16_t* x, int64_t T, int64_t H, double* m, moe_stream_t stream);

/* Per-expert bit-widths under a read budget [DuoRate: a Lagrangian rate-distortion
 * allocation solved with one dot product per expert and a bisection to the read
 * budget; the routing frequency cancels from every per-expert decision].
 *   D[e][c] = sum_k m[k] * delta[e][choices[c]-1][k]  (one warp per dot product);
 *   at multiplier lam each expert takes argmin_c D[e][c] + lam * choices[c], ties to the
 *   larger width; 100 bisection steps on lam find the smallest lam whose read rate is
 *   within the budget -- the exact integer sum_e n_e * b_e (n_e pairs routed to e, from
 *   expert_offsets) against the fp64 product budget * sum_e n_e -- and bits_e receives
 *   the widths at the upper end of the final interval.  Experts with no pairs, and all
 *   experts when even the smallest width exceeds the budget, get the smallest choice.
 *   delta fp64 [E][8][K];  m fp64 [K];  expert_offsets int32 [E+1] (moe_route_topk);
 *   choices: HOST array of nchoices distinct widths in 1..8, 1 <= nchoices <= 8;
 *   budget: bits per weight, finite, >= 0;  bits_e uint8 [E];  lambda: fp64 device
 *   scalar that receives the final multiplier, or NULL.  One CTA; E <= MOE_MAX_EXPERTS. */
moe_status_t moe_allocate_bits(const double* delta, const double* m, const int32_t* expert_offsets, int64_t E,
                               int64_t K, const uint8_t* choices, int64_t nchoices, double budget,
                               uint8_t* bits_e, double* lambda, moe_stream_t stream);

/* Per-pair bit-widths from per-expert ones: bits[p] = bits_e[topk_ids[p]], p < T*k
 * (the bits array moe_grouped_ffn takes for BITPLANE8). */
moe_status_t moe_expand_bits(const int32_t* topk_ids, const uint8_t* bits_e, int64_t T, int64_t k,
                             uint8_t* bits, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Expert slot cache: planning (HOST functions: host memory only, no CUDA call)
 * [ExactMoE abstract: routed experts kept in pinned host memory and executed through a
 * configurable GPU-resident slot cache, every routed expert served; PagedMoE abstract:
 * a cached bitplane prefix is reused or extended by fetching only the missing planes,
 * the prefix length decided before any transfer].
 *
 * A step's demand need[e] (0 = nothing routed to e; else the planes its pairs read,
 * 1..planes) is served in ascending expert id:
 *   hit        resident with >= need[e] planes: nothing fetched;
 *   extension  resident with h < need[e] planes: fetch planes [h, need[e]);
 *   miss       fetch planes [0, need[e]) into the lowest free slot, else into the slot,
 *              among those not served in the current round, with the smallest
 *              (holds an expert needed later in the step, last step used, slot index).
 * When a miss finds every slot served in the current round, the round closes (the
 * caller computes its experts) and a new round starts; a step needing <= S experts is
 * one round.
 * ------------------------------------------------------------------------ */

/* Bytes of host memory for the state of a cache of S slots over E experts; 0 if
 * 1 <= S <= E <= MOE_MAX_EXPERTS does not hold. */
size_t moe_cache_state_bytes(int64_t E, int64_t S);

/* Initialise a cache state (all slots free) in caller-owned host memory, 8-byte aligned,
 * of at least moe_cache_state_bytes(E, S) bytes.  planes: 8 for bitplane experts, 1 for
 * whole-expert formats (W4 g128, NVFP4).  MOE_ERR_WORKSPACE if state_bytes is short. */
moe_status_t moe_cache_init(void* state, size_t state_bytes, int64_t E, int64_t S, int64_t planes);

/* Plan one step and update the state (host arrays throughout).  need uint8 [E], each
 * <= planes (checked before the state changes).  Outputs for the n routed experts, in
 * service order: served_expert int32 [n], served_slot int32 [n], fetch_lo / fetch_hi
 * uint8 [n] (planes [lo, hi) to copy into the slot; lo == hi: nothing); round_start
 * int32 [R + 1] (round r = entries [round_start[r], round_start[r+1])); *nrounds = R.
 * Capacities: E entries for the per-expert arrays, E + 1 for round_start. */
moe_status_t moe_cache_plan(void* state, const uint8_t* need, int32_t* served_expert, int32_t* served_slot,
                            uint8_t* fetch_lo, uint8_t* fetch_hi, int32_t* round_start, int32_t* nrounds);

/* The slots' contents: expert_of int32 [S] (-1 = free) and resident planes uint8 [S]. */
moe_status_t moe_cache_slots(const void* state, int32_t* expert_of, uint8_t* planes);

/* ------------------------------------------------------------------------
 * Expert slot cache on the device (device memory; graph-capturable, no host sync)
 * ------------------------------------------------------------------------ */

/* One step's plan on the device (device arrays, caller-allocated). */
typedef struct {
  int32_t* served_expert; /* [E]  routed experts in ascending id */
  int32_t* served_slot;   /* [E]  their slots */
  uint8_t* fetch_lo;      /* [E]  planes [lo, hi) to copy; lo == hi: nothing */
  uint8_t* fetch_hi;      /* [E] */
  int32_t* nserved;       /* [1]  number of routed experts */
  int32_t* overflow;      /* [1]  1 if the step needed more slots than exist (state unchanged) */
} moe_cache_plan_t;

/* Plans one step on a DEVICE copy of a state written by moe_cache_init (same bytes,
 * 8-byte aligned device memory), from the routing of the step: need[e] = the largest
 * bits[p] over e's pairs (bits NULL: 1 for whole experts), and writes every pair's slot
 * id (slot_ids int32 [T*k]) for moe_permute.  Requires S >= min(E, T*k): one round, in
 * which the plan equals moe_cache_plan's (no routed expert is evicted); E and S must be
 * the state's. */
moe_status_t moe_cache_step(void* state, int64_t E, int64_t S, const moe_routing_t* routing, const uint8_t* bits,
                            int64_t T, int64_t k, int32_t* slot_ids, const moe_cache_plan_t* plan,
                            moe_stream_t stream);

/* Copies the planned planes of the served experts from the host store into their slots,
 * with the expert's scales (and NVFP4 per-expert scale) on a miss.  host_store: the E
 * experts in the layouts of moe_experts_t, in page-locked host memory the device can read
 * (cudaHostAlloc, or cudaHostRegister with mapping); slots: the same layouts with S
 * experts, device memory.  Reads over the host link; returns without waiting. */
moe_status_t moe_cache_fetch(const moe_cache_plan_t* plan, int64_t E, const moe_experts_t* host_store,
                             const moe_experts_t* slots, int64_t H, int64_t I, moe_stream_t stream);

/* The permutation of moe_route_topk alone: from ids int32 [T*k] (each < E) writes
 * out->expert_offsets, sorted_pair, pair_to_row and expert_list (out->topk_ids and
 * topk_w are not touched).  With ids = moe_cache_step's slot ids and E = S, the routing
 * of the slot store for moe_grouped_ffn and moe_combine.  T = 0: nothing is written. */
moe_status_t moe_permute(const int32_t* ids, int64_t T, int64_t k, int64_t E, const moe_routing_t* out,
                         moe_stream_t stream);

/* Per-pair bit-width from the routing weight [MatMoE: precision per expert from
 * routing scores; PagedMoE: prefix length from current routing weights].
 * bits[p] = choices[0] if w < thresholds[0], choices[1] if w < thresholds[1],
 * choices[2] if w < thresholds[2], else choices[3] (fp32 compares; equality takes
 * the higher tier).  thresholds and choices are HOST arrays (copied at the call);
 * thresholds ascending, choices in 1..8.
 *   topk_w fp32 [T*k];  bits uint8 [T*k]. */
moe_status_t moe_select_bits(const float* topk_w, int64_t T, int64_t k,
                             const float thresholds[3], const uint8_t choices[4],
                             uint8_t* bits, moe_stream_t stream);

/* Bytes of device workspace moe_grouped_ffn needs. */
size_t moe_ffn_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k,
                               moe_format_t fmt);

/* Grouped SwiGLU expert FFN over the permuted pairs [ExactMoE: fused grouped
 * execution of all selected experts; PagedMoE: prefixes executed directly, no
 * full-precision expert materialised].
 * For sorted row r of expert e holding pair p = t*k + j:
 *   g = x[t] . deq(W_gate_e)^T, u = x[t] . deq(W_up_e)^T  (fp32 accumulation),
 *   h = bf16(silu(g) * u),  y_rows[r] = bf16(h . deq(W2_e)^T).
 * Two execution paths, chosen on the host from the shape alone (nothing is read back
 * from the device): with T*k >= 32*E and W4G128 or NVFP4 weights, a tensor-core GEMM
 * (weights dequantised into tensor memory once per tile of up to 192 routed rows, fp16
 * operands: W4 weights q*s, NVFP4 weights e2m1*e4m3) for the experts with more than 16
 * routed rows, followed by the weight-streaming GEMV for the others; otherwise the GEMV
 * alone (dequantisation in registers, weights read once per pass of up to 16 rows).  For
 * BITPLANE8 expert e is read at bits[p] planes for pair p (planes 0..bits[p]-1, floor
 * and compensation as above); expert e's weights are fetched to max_p bits[p].
 *   x bf16 [T][H];  routing: as written by moe_route_topk;  bits uint8 [T*k]
 *   (BITPLANE8 only, values 1..8, else may be NULL);  y_rows bf16 [T*k][H].
 * Requires H % 256 == 0, I % 128 == 0, the limits of moe_route_topk, and workspace
 * >= moe_ffn_workspace_bytes(...) (scratch: h, and for the GEMM path the token rows
 * gathered into routed order; contents need not be initialised).  Not bit-exact: fp32
 * accumulation order, the rounding of h (and, on the GEMM path, of each dequantised
 * W4 weight to fp16) differ from an fp64 reference (ExactMoE: the low-bit layer is
 * not numerically identical to BF16); the FFN tolerance covers both paths.
 * Range: the W4 paths stage activations as fp16 x/16 and x/256 (GEMV) or x/16 and h/16
 * (GEMM), the NVFP4 paths activations and h as fp16 * 2^-8, so |x|, |h| < 2^20 (W4) and
 * |x|, |h| < 2^24 (NVFP4) keep them finite; magnitudes below 2^-10 (W4) or 2^-6 (NVFP4)
 * fall into fp16's subnormal range (absolute error at most 2^-20 or 2^-16).  The W4 GEMM
 * rounds each weight q*s to fp16 (relative 2^-12 at most, for scales >= 2^-14).  Bitplane activations are staged in
 * bf16 scaled by up to 2^7 (|x| < 2^120). */
moe_status_t moe_grouped_ffn(const uint16_t* x, const moe_routing_t* routing,
                             const moe_experts_t* experts, const uint8_t* bits,
                             int64_t T, int64_t H, int64_t I, int64_t E, int64_t k,
                             uint16_t* y_rows, void* workspace, size_t workspace_bytes,
                             moe_stream_t stream);

/* Bytes of the weight-scale tiles moe_w4a4_prepare writes for E experts of H, I. */
size_t moe_w4a4_scale_tiles_bytes(int64_t H, int64_t I, int64_t E);

/* Lays out the E4M3 block scales of NVFP4 experts (as written by moe_quantize_nvfp4) in the
 * order the block-scaled FP4 tensor cores read them [MoET: NVFP4 for expert GEMMs]: per
 * 128-row weight tile and 64-element K block, 512 bytes holding the scale of tile row
 * m = m0 + 32 m1 and sub-block kk (16 elements) at byte 16 m0 + 4 m1 + kk.  Gate/up tiles
 * are 64 gate and 64 up rows, interleaved by 16 (tile row 32 q + j: gate row 64 t + 16 q + j
 * for j < 16, else up row I + 64 t + 16 q + j - 16); down tiles are 128 consecutive rows of w2.
 * Run once per set of experts (the tiles depend on the weights only); the result is read
 * by every moe_grouped_ffn_w4a4 call on those experts.
 *   scale_tiles: device, 16-byte aligned, >= moe_w4a4_scale_tiles_bytes(H, I, E) bytes.
 * Requires H % 256 == 0, I % 128 == 0. */
moe_status_t moe_w4a4_prepare(const moe_experts_t* experts, int64_t H, int64_t I, int64_t E, void* scale_tiles,
                              size_t scale_tiles_bytes, moe_stream_t stream);

/* Bytes of device workspace moe_grouped_ffn_w4a4 needs. */
size_t moe_ffn_w4a4_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k);

/* The grouped FFN with NVFP4 weights AND NVFP4 activations (W4A4) for prefill batches
 * [MoET: NVFP4 for expert GEMMs].  x is quantised on the fly as one tensor by the NVFP4
 * recipe (E2M1 codes, an E4M3 scale per 16 consecutive elements of a row, one fp32 scale
 * amax/2688 for the tensor); per expert g, u = x' W13'^T, h = silu(g) u kept in fp32; all
 * routed rows of h are quantised the same way, as one tensor, from those fp32 values; y_rows
 * = h' W2'^T (bf16).  The tensor cores take both operands as E2M1 codes with their E4M3
 * block scales (tcgen05 kind::mxf4nvf4, block16: every product e2m1 * e4m3 * e2m1 * e4m3 is
 * exact, fp32 accumulation); the two per-tensor scales multiply each sum once.  Always this
 * GEMM (any batch size): tiles of 128 weight rows x 128 routed rows, K stages of 256.
 *   experts: fmt must be MOE_FMT_NVFP4; scale_tiles: written by moe_w4a4_prepare for the
 *   same experts; other arguments and layouts as for moe_grouped_ffn; workspace >=
 *   moe_ffn_w4a4_workspace_bytes(...) (scratch: the quantised x and h, x's codes in routed
 *   order, the activation scales in tile order, h in fp32).
 * Requires H % 256 == 0, I % 128 == 0.
 * Tolerance against the W4A4 definition as for moe_grouped_ffn; an element of h within a
 * rounding of an E2M1 decision boundary may take the other code (fp32 order). */
moe_status_t moe_grouped_ffn_w4a4(const uint16_t* x, const moe_routing_t* routing, const moe_experts_t* experts,
                                  const void* scale_tiles, int64_t T, int64_t H, int64_t I, int64_t E, int64_t k,
                                  uint16_t* y_rows, void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* Routing-weighted combine [ExactMoE: the selected experts' outputs weighted by the
 * unchanged routing weights]: out[t] = bf16( sum_{j<k} topk_w[t*k+j] *
 * y_rows[pair_to_row[t*k+j]] (+ residual[t]) ), fp32 accumulation in slot order j.
 *   y_rows bf16 [T*k][H];  residual bf16 [T][H] or NULL;  out bf16 [T][H] (may alias residual).
 * Requires H % 8 == 0.  Deterministic. */
moe_status_t moe_combine(const uint16_t* y_rows, const moe_routing_t* routing,
                         const uint16_t* residual, int64_t T, int64_t H, int64_t k,
                         uint16_t* out, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Expert parallelism: the device side of the exchange [ExactMoE: every selected expert
 * is executed, wherever it is placed].  Rank r owns experts [r E/G, (r+1) E/G); a rank
 * sends its routed rows in sorted-row order (moe_gather_rows with idx = sorted_pair,
 * div = k); an owner receives runs in source-rank order, each grouped by local expert,
 * and labels them with moe_ids_from_counts for moe_permute (k = 1, E = E/G).
 * ------------------------------------------------------------------------ */

/* dst[i] = src[idx[i] / div] for i < n: rows of H bf16 (H % 8 == 0); idx int32 [n]
 * (4-byte aligned), every idx[i] / div a valid row of src. */
moe_status_t moe_gather_rows(const uint16_t* src, const int32_t* idx, int64_t n, int64_t div, int64_t H,
                             uint16_t* dst, moe_stream_t stream);

/* Local expert of each received row: counts int32 [S][El] (rows from source s for local
 * expert j); ids int32 [sum of counts] gets j for those rows, ordered by s then j.
 * One CTA; S * El <= 2^20. */
moe_status_t moe_ids_from_counts(const int32_t* counts, int64_t S, int64_t El, int32_t* ids, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Device error reporting
 * ------------------------------------------------------------------------ */

/* Synchronises `stream`, then reads and clears the library's device error word.
 * Kernels never trap: a kernel whose bounded wait on an asynchronous copy runs out
 * records the fact and returns.  Returns MOE_ERR_DEVICE_TIMEOUT if any kernel on
 * this device recorded one since the last call, MOE_ERR_CUDA if the stream reports
 * an error, else MOE_OK. */
moe_status_t moe_check_device_errors(moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
