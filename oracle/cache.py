"""Expert slot cache with plane-prefix reuse (test infrastructure, like the rest of
``oracle``): which routed experts are served from device slots, which must be fetched
from the host-resident expert store, and which planes.

Follows "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference", abstract
(experts kept in pinned host memory, executed through a configurable GPU-resident slot
cache; complete expert availability with unchanged top-k routing, so every routed expert
is served), and "PagedMoE: Cross-Precision Expert Caching for Token-Level Dynamic
Precision in SSD-Resident MoE Inference", abstract (one stored state per expert in a
bitplane layout; lower precisions are prefixes, so cached data is reused or extended by
fetching only the missing bitplanes; the prefix length is chosen before any transfer).
The pages fix no replacement policy; the plainest reading (R28-R31):

  R28  S slots; a slot holds at most one expert: for bitplane experts the prefix of its
       first h planes (h = 1..8) plus its scales, for whole-expert formats the expert
       (h = 1 of P = 1 "plane").
  R29  demand of a step: need[e] = 0 for an expert nothing is routed to, else the planes
       its pairs read (bitplanes: the largest width among them; whole experts: 1).
  R30  service: the routed experts in ascending id.  An expert already resident with
       h >= need is a hit; resident with h < need is an extension (fetch planes
       [h, need)); otherwise a miss (fetch planes [0, need)) into a victim slot: the
       lowest-index free slot, else, among slots not pinned in the current round, the
       one minimising (holds an expert needed later in this step, last step it was
       used, slot index).  Hits and extensions keep their slot.
  R31  rounds: experts served in a round are pinned until the round ends; when a miss
       finds no victim, the round closes (its experts are computed) and a new round
       begins with nothing pinned.  A step needing at most S experts is one round.
       last_use of a served slot is the step's index (steps count from 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass
class Served:
    expert: int
    slot: int
    lo: int      # first plane fetched (lo == hi: nothing fetched, a hit)
    hi: int      # one past the last plane fetched


@dataclass
class SlotCache:
    E: int
    S: int
    P: int = 1                   # planes per expert (8 for bitplanes, 1 for whole experts)
    step: int = 0
    slot_of: list = field(default_factory=list)    # [E] slot or -1
    expert_of: list = field(default_factory=list)  # [S] expert or -1
    planes: list = field(default_factory=list)     # [S] resident planes h
    last_use: list = field(default_factory=list)   # [S] step last served (0: never)

    def __post_init__(self):
        self.slot_of = [-1] * self.E
        self.expert_of = [-1] * self.S
        self.planes = [0] * self.S
        self.last_use = [0] * self.S

    def plan(self, need) -> list[list[Served]]:
        """Serve one step's demand (reading R29: need[e] in 0..P); returns the rounds,
        each the list of experts served in it, in service order (R30, R31)."""
        need = [int(v) for v in need]
        assert len(need) == self.E and all(0 <= v <= self.P for v in need)
        self.step += 1
        routed = [e for e in range(self.E) if need[e] > 0]
        rounds: list[list[Served]] = []
        cur: list[Served] = []
        pinned: set[int] = set()
        i = 0
        while i < len(routed):
            e = routed[i]
            s = self.slot_of[e]
            if s >= 0:  # hit or extension
                h = self.planes[s]
                lo, hi = (h, need[e]) if h < need[e] else (need[e], need[e])
                self.planes[s] = max(h, need[e])
            else:
                s = self._victim(pinned, set(routed[i + 1:]))
                if s < 0:  # every slot is pinned: close the round
                    assert cur, "a round always fits one expert (S >= 1)"
                    rounds.append(cur)
                    cur, pinned = [], set()
                    continue
                old = self.expert_of[s]
                if old >= 0:
                    self.slot_of[old] = -1
                self.expert_of[s], self.slot_of[e], self.planes[s] = e, s, need[e]
                lo, hi = 0, need[e]
            self.last_use[s] = self.step
            pinned.add(s)
            cur.append(Served(e, s, lo, hi))
            i += 1
        if cur:
            rounds.append(cur)
        return rounds

    def _victim(self, pinned: set, later: set) -> int:
        for s in range(self.S):
            if self.expert_of[s] < 0:
                return s
        best, key = -1, None
        for s in range(self.S):
            if s in pinned:
                continue
            k = (1 if self.expert_of[s] in later else 0, self.last_use[s], s)
            if key is None or k < key:
                best, key = s, k
        return best


def need_from_routing(offsets, sorted_pair, bits=None, planes: int = 1):
    """need[e] of one step (R29): 0 if no pair is routed to e, else the largest width
    among its pairs (bits per pair, bitplane experts) or 1 (whole experts)."""
    E = len(offsets) - 1
    need = [0] * E
    for e in range(E):
        for r in range(int(offsets[e]), int(offsets[e + 1])):
            w = 1 if bits is None else int(bits[int(sorted_pair[r])])
            need[e] = max(need[e], min(planes, w))
    return need


def fetched_planes(rounds) -> int:
    """Planes fetched over a step's rounds."""
    return sum(sv.hi - sv.lo for rnd in rounds for sv in rnd)
