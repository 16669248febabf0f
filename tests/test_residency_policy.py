"""The expert cache's replacement policy, on CPU: a plain model of the rule
that moe_layer_forward_cached applies on the GPU, pinned by hand-worked
sequences.  The GPU tests compare the device's decisions with this model.

Rule (per call, over the distinct experts the call selected, ascending):
a resident expert counts a use; a missing one takes an empty slot if there
is one (the lowest), else the slot with the fewest uses among the slots this
call does not need, ties to the least recently used, then to the lowest
slot; a newly loaded expert has one use."""


class CacheModel:
    def __init__(self, E, C):
        self.slot_of = [-1] * E
        self.expert_of = [-1] * C
        self.uses = [0] * C
        self.last = [0] * C
        self.tick = self.hits = self.misses = 0

    def call(self, experts):
        needed = sorted(set(experts))
        self.tick += 1
        pinned = {self.slot_of[e] for e in needed if self.slot_of[e] >= 0}
        loaded = []
        for e in needed:
            s = self.slot_of[e]
            if s >= 0:
                self.hits += 1
                self.uses[s] += 1
                self.last[s] = self.tick
                continue
            free = [c for c in range(len(self.expert_of)) if c not in pinned]
            empty = [c for c in free if self.expert_of[c] < 0]
            v = empty[0] if empty else min(free, key=lambda c: (self.uses[c], self.last[c], c))
            if self.expert_of[v] >= 0:
                self.slot_of[self.expert_of[v]] = -1
            self.expert_of[v], self.slot_of[e] = e, v
            self.uses[v], self.last[v] = 1, self.tick
            pinned.add(v)
            loaded.append((e, v))
            self.misses += 1
        return loaded


def test_hand_worked_sequence_two_slots():
    m = CacheModel(E=4, C=2)
    assert m.call([0]) == [(0, 0)]            # empty slots fill from the lowest
    assert m.call([1]) == [(1, 1)]
    assert m.call([0]) == []                  # hit: expert 0 now has 2 uses
    assert m.call([2]) == [(2, 1)]            # fewest uses: slot 1 (expert 1, 1 use)
    assert m.slot_of == [0, -1, 1, -1]
    assert m.call([3, 0]) == [(3, 1)]         # expert 0 is needed: its slot is not a victim
    assert (m.hits, m.misses) == (2, 4)


def test_recency_breaks_use_ties_then_the_lowest_slot():
    m = CacheModel(E=6, C=3)
    m.call([0, 1, 2])                         # all three loaded in one call: 1 use each, same tick
    m.call([1])                               # slot 1: 2 uses
    m.call([2])                               # slot 2: 2 uses, newer
    assert m.call([3]) == [(3, 0)]            # slot 0: fewest uses
    m.call([3])                               # slot 0 back to 2 uses, newest
    assert m.call([4]) == [(4, 1)]            # 2 uses each: slot 1 is the least recently used
    m2 = CacheModel(E=4, C=2)
    m2.call([0, 1])
    assert m2.call([2]) == [(2, 0)]           # equal uses and ticks: the lowest slot


def test_a_call_never_evicts_what_it_needs():
    m = CacheModel(E=8, C=4)
    for step in range(50):
        experts = [(step * 3 + j * 5) % 8 for j in range(3)]
        m.call(experts)
        for e in set(experts):
            assert m.slot_of[e] >= 0 and m.expert_of[m.slot_of[e]] == e
        assert sorted(e for e in m.expert_of if e >= 0) == sorted(e for e in range(8) if m.slot_of[e] >= 0)
