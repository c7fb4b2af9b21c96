// Expert slot cache: the planning core shared by the host entry point and device code.
//
// After "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference" (abstract:
// routed experts live in pinned host memory and run through a GPU-resident slot cache,
// every routed expert served) and "PagedMoE: Cross-Precision Expert Caching for
// Token-Level Dynamic Precision in SSD-Resident MoE Inference" (abstract: a bitplane
// expert state is reused or extended by fetching only its missing planes, the prefix
// length decided before any transfer).
//
// One step's plan: the experts with need[e] > 0, in ascending id, are served into slots:
//   hit        resident with at least need[e] planes: nothing to fetch;
//   extension  resident with h < need[e] planes: fetch planes [h, need[e]);
//   miss       fetch planes [0, need[e]) into the lowest free slot, else into the
//              unpinned slot with the smallest (expert needed later in the step, last
//              step used, slot index);
// slots served in the current round are pinned; a miss with every slot pinned closes the
// round (its experts get computed) and opens a new one with nothing pinned.
//
// State (caller memory, 8-byte aligned): a header, then slot_of[E] (int32, -1 if not
// resident), expert_of[S] (int32, -1 if free), last_use[S] and pin_mark[S] (int64),
// planes[S] (uint8).
#pragma once
#include <stddef.h>
#include <stdint.h>

#ifdef __CUDACC__
#define MOE_HD __host__ __device__
#else
#define MOE_HD
#endif

namespace moe {

constexpr int32_t kCacheMagic = 0x43414348;  // "CACH"

struct CacheHeader {
  int32_t magic, E, S, P;  // P: planes per expert (8 for bitplanes, 1 for whole experts)
  int64_t step;            // steps planned so far
  int64_t mark;            // current round's pin mark
};

struct CacheView {
  CacheHeader* h;
  int32_t* slot_of;    // [E]
  int32_t* expert_of;  // [S]
  int64_t* last_use;   // [S]
  int64_t* pin_mark;   // [S]
  uint8_t* planes;     // [S]
};

MOE_HD inline size_t cache_align8(size_t b) { return (b + 7) / 8 * 8; }

MOE_HD inline size_t cache_state_bytes(int E, int S) {
  return cache_align8(sizeof(CacheHeader)) + cache_align8(size_t(E) * 4) + cache_align8(size_t(S) * 4) +
         size_t(S) * 8 * 2 + cache_align8(size_t(S));
}

MOE_HD inline CacheView cache_view(void* state, int E, int S) {
  uint8_t* p = static_cast<uint8_t*>(state);
  CacheView v;
  v.h = reinterpret_cast<CacheHeader*>(p);
  p += cache_align8(sizeof(CacheHeader));
  v.slot_of = reinterpret_cast<int32_t*>(p);
  p += cache_align8(size_t(E) * 4);
  v.expert_of = reinterpret_cast<int32_t*>(p);
  p += cache_align8(size_t(S) * 4);
  v.last_use = reinterpret_cast<int64_t*>(p);
  p += size_t(S) * 8;
  v.pin_mark = reinterpret_cast<int64_t*>(p);
  p += size_t(S) * 8;
  v.planes = p;
  return v;
}

MOE_HD inline void cache_reset(CacheView v, int E, int S, int P) {
  v.h->magic = kCacheMagic;
  v.h->E = E;
  v.h->S = S;
  v.h->P = P;
  v.h->step = 0;
  v.h->mark = 0;
  for (int e = 0; e < E; ++e) v.slot_of[e] = -1;
  for (int s = 0; s < S; ++s) {
    v.expert_of[s] = -1;
    v.last_use[s] = 0;
    v.pin_mark[s] = -1;
    v.planes[s] = 0;
  }
}

// the slot a miss of expert e goes to, or -1 when every slot is pinned in this round
MOE_HD inline int cache_victim(const CacheView& v, int e, const uint8_t* need) {
  const int S = v.h->S;
  for (int s = 0; s < S; ++s)
    if (v.expert_of[s] < 0) return s;
  int best = -1;
  int best_later = 0;
  int64_t best_use = 0;
  for (int s = 0; s < S; ++s) {
    if (v.pin_mark[s] == v.h->mark) continue;
    const int x = v.expert_of[s];
    const int later = (x > e && need[x] > 0) ? 1 : 0;
    // lexicographic (later, last_use, s); s only grows, so ties keep the first slot
    if (best < 0 || later < best_later || (later == best_later && v.last_use[s] < best_use)) {
      best = s;
      best_later = later;
      best_use = v.last_use[s];
    }
  }
  return best;
}

// Plans one step.  need[E] in 0..P.  Outputs, in service order, served_expert[n],
// served_slot[n], fetch_lo[n], fetch_hi[n] (lo == hi: nothing to fetch) for n < the number
// of routed experts, and round_start[0..R] (round r = [round_start[r], round_start[r+1]));
// returns R.
MOE_HD inline int cache_plan(CacheView v, const uint8_t* need, int32_t* served_expert, int32_t* served_slot,
                             uint8_t* fetch_lo, uint8_t* fetch_hi, int32_t* round_start) {
  const int E = v.h->E;
  v.h->step += 1;
  v.h->mark += 1;
  int n = 0, r = 0;
  round_start[0] = 0;
  for (int e = 0; e < E; ++e) {
    const int want = need[e];
    if (want == 0) continue;
    int s = v.slot_of[e];
    int lo = want, hi = want;
    if (s >= 0) {
      const int have = v.planes[s];
      if (have < want) {
        lo = have;
        v.planes[s] = uint8_t(want);
      }
    } else {
      s = cache_victim(v, e, need);
      if (s < 0) {  // every slot pinned: close the round, then serve e in a fresh one
        round_start[++r] = n;
        v.h->mark += 1;
        s = cache_victim(v, e, need);
      }
      const int old = v.expert_of[s];
      if (old >= 0) v.slot_of[old] = -1;
      v.expert_of[s] = e;
      v.slot_of[e] = s;
      v.planes[s] = uint8_t(want);
      lo = 0;
    }
    v.last_use[s] = v.h->step;
    v.pin_mark[s] = v.h->mark;
    served_expert[n] = e;
    served_slot[n] = s;
    fetch_lo[n] = uint8_t(lo);
    fetch_hi[n] = uint8_t(hi);
    ++n;
  }
  if (n > round_start[r]) round_start[++r] = n;
  return r;
}

}  // namespace moe
