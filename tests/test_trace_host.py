"""Decoding of the step trace (include/eta.h) on the host: every slot is an
atomic maximum, a "first" slot holds the bitwise complement of the earliest
time, an unwritten slot is 0 and left out."""
import torch

import learned_threshold_sparse_b200 as eta


def _complement(t):
    return (~t) & 0xFFFFFFFFFFFFFFFF


def _as_signed(u):
    return u - (1 << 64) if u >= 1 << 63 else u


def test_slots_and_decoding():
    assert eta.ETA_TRACE_SLOTS == 24
    slots = {name: (slot, first) for name, slot, first in eta.TRACE_SLOTS}
    assert len({s for s, _ in slots.values()}) == len(slots)
    assert all(0 <= s < eta.ETA_TRACE_SLOTS for s, _ in slots.values())
    tr = torch.zeros(eta.ETA_TRACE_SLOTS, dtype=torch.int64)
    times = {"screen_first": 1_000, "screen_last": 5_000, "attend_first": 5_500, "tile_first": 9_000,
             "attend_last": 70_000, "append_first": 100, "append_last": 900}
    for name, t in times.items():
        slot, first = slots[name]
        # what the kernels leave after several CTAs: the max of complements
        # (earliest time) for a first slot, the max of times for a last slot
        vals = [t, t + 700, t + 30] if first else [t - 400, t, t - 10]
        v = max(_complement(x) for x in vals) if first else max(vals)
        tr[slot] = _as_signed(v)
    got = eta.trace_times(tr)
    assert got == times
