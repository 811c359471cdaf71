"""A model of the tensor-core kernels' barrier protocols, checked on the CPU.

Every warp role (TMA producer, feature map, MMA issuer, state group, scores/output group) is
written as the sequence of mbarrier waits (with the phase index it waits for) and arrivals it
performs, for the three kernels (0: the aggregate mode of tc_forward.cu, 1: the causal output
kernel of tc_causal.cu, 2: the non-causal output mode of tc_forward.cu) and any list of work
items of 1..16 chunks walked by one CTA.  A random scheduler interleaves the roles. The
test fails on a deadlock (no role can move) or on parity aliasing (a wait for a phase two or more
phases behind its barrier, which the hardware's parity test cannot tell from a pending one).
Each role's arrivals count as one (the kernel's thread counts are per role).  This model mirrors
the kernel's code by hand: change both together.
"""
import random
import sys

import pytest


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.completed = count, 0, 0


def roles(mode, NS, items):
    """Generators of ('w', barrier, phase) and ('a', barrier) events, one per warp role.

    Modes 0 and 2: tc_forward.cu (aggregate, non-causal output).  Mode 1: tc_causal.cu after
    the three-kernel pass's scan; mode 3: tc_causal.cu as the single pass (each item streams
    its aggregate chunks first; the look-back between CTAs is outside this model)."""
    causal = mode in (1, 3)
    fused = mode == 3

    def tma():
        g = 0
        for nc in items:
            for _ in range((2 if fused else 1) * nc):
                s = g % NS
                if g >= NS:
                    yield ("w", f"empty[{s}]", g // NS - 1)
                yield ("a", f"full[{s}]")
                g += 1
        for gg in range(max(0, g - NS), g):  # drain: every load has landed
            yield ("w", f"full[{gg % NS}]", gg // NS)

    def feature_map():
        g = 0
        for j, nc in enumerate(items):
            for c in range((2 if fused else 1) * nc):
                s = g % NS
                yield ("w", f"full[{s}]", g // NS)
                yield ("a", f"ready[{s}]")
                if causal:  # the column sums of every feature-map warp are in
                    yield ("a", "zsync")
                    yield ("w", "zsync", g)
                if fused and c + 1 == nc:  # the item's z published; its start z back
                    yield ("a", "zpub")
                    yield ("w", "zready", j)
                g += 1

    def mma():
        g = go = 0
        for j, nc in enumerate(items):
            b = j & 1
            if mode == 0 and j >= 2:
                yield ("w", f"item_empty[{b}]", (j >> 1) - 1)
            if mode == 2:
                yield ("w", f"item_full[{b}]", j >> 1)
            if fused:  # the aggregate chunks
                for _ in range(nc):
                    s = g % NS
                    yield ("w", f"ready[{s}]", g // NS)
                    yield ("a", f"empty[{s}]")  # the commit
                    yield ("a", f"empty[{s}]")  # on behalf of the output group
                    g += 1
                yield ("a", "s_full")
            for c in range(nc):
                s = g % NS
                yield ("w", f"ready[{s}]", g // NS)
                if mode == 0:
                    yield ("a", f"empty[{s}]")
                elif causal:
                    yield ("w", "s_ready", go)
                    if go >= 2:
                        yield ("w", f"o_empty[{go & 1}]", (go >> 1) - 1)
                    yield ("a", "p_full")
                    if not fused or c + 1 < nc:
                        yield ("a", "s_full")
                    yield ("w", "p_ready", go)
                    yield ("a", f"o_full[{go & 1}]")
                    yield ("a", f"empty[{s}]")
                else:
                    if g >= 2:
                        yield ("w", f"o_empty[{g & 1}]", (g >> 1) - 1)
                    yield ("a", f"o_full[{g & 1}]")
                    yield ("a", f"empty[{s}]")
                g += 1
                go += 1
            if mode == 0:
                yield ("a", f"item_full[{b}]")
            if mode == 2:
                yield ("a", f"item_empty[{b}]")
        yield ("a", "fin")
        yield ("w", "fin", 0)

    def state_group():
        if causal:
            gs = 0
            for j, nc in enumerate(items):
                if fused:  # the aggregate, the published z, then the start state
                    yield ("w", "s_full", gs)
                    gs += 1
                    yield ("w", "zpub", j)
                    yield ("a", "zready")
                elif j > 0:  # the previous item's last products are done with S
                    yield ("w", "s_full", gs)
                    gs += 1
                yield ("a", "s_ready")
                for c in range(nc):
                    if c + 1 < nc:
                        yield ("w", "s_full", gs)
                        gs += 1
                        yield ("a", "s_ready")
        elif mode == 2:
            for j in range(len(items)):
                b = j & 1
                if j >= 2:
                    yield ("w", f"item_empty[{b}]", (j >> 1) - 1)
                yield ("a", f"item_full[{b}]")
        else:
            for j in range(len(items)):
                b = j & 1
                yield ("w", f"item_full[{b}]", j >> 1)
                yield ("a", f"item_empty[{b}]")

    def score_group():
        if not causal:
            return
        g = go = 0
        for nc in items:
            g += nc if fused else 0
            for _ in range(nc):
                yield ("w", f"ready[{g % NS}]", g // NS)  # phi(q).z of this stage
                yield ("w", "p_full", go)
                yield ("a", "p_ready")
                yield ("a", f"den_ready[{go & 1}]")
                g += 1
                go += 1

    def output_group():
        g = go = 0
        if causal:
            for nc in items:
                g += nc if fused else 0
                for _ in range(nc):
                    yield ("w", f"o_full[{go & 1}]", go >> 1)
                    yield ("w", f"den_ready[{go & 1}]", go >> 1)
                    yield ("a", f"empty[{g % NS}]")  # the stage's last reader
                    yield ("a", f"o_empty[{go & 1}]")
                    g += 1
                    go += 1
        elif mode == 2:
            for nc in items:
                for _ in range(nc):
                    yield ("w", f"o_full[{g & 1}]", g >> 1)
                    yield ("a", f"o_empty[{g & 1}]")
                    g += 1

    return [tma(), feature_map(), mma(), state_group(), score_group(), output_group()]


def run(mode, NS, items, rng):
    # arrivals per phase: every barrier here is released by one role, except the causal kernel's
    # stages (the MMA commit and the output group)
    counts = {"empty": 2} if mode in (1, 3) else {}
    bars = {}

    def bar(name):
        if name not in bars:
            bars[name] = Barrier(counts.get(name.split("[")[0], 1))
        return bars[name]

    gens = roles(mode, NS, items)
    cur = [next(gen, None) for gen in gens]
    while True:
        runnable = []
        for r, ev in enumerate(cur):
            if ev is None:
                continue
            if ev[0] == "a":
                runnable.append(r)
                continue
            b, phase = bar(ev[1]), ev[2]
            assert b.completed < phase + 2, f"parity aliasing: {ev}, mode {mode}, items {items}"
            if b.completed > phase:  # the waited-for phase has completed
                runnable.append(r)
        if not runnable:
            assert all(ev is None for ev in cur), f"deadlock at {cur}, mode {mode}, items {items}"
            return True
        r = rng.choice(runnable)
        if cur[r][0] == "a":
            b = bar(cur[r][1])
            b.pending += 1
            if b.pending == b.count:
                b.pending, b.completed = 0, b.completed + 1
        cur[r] = next(gens[r], None)


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_protocol_has_no_deadlock_or_aliasing(mode):
    rng = random.Random(1000 + mode)
    for _ in range(1500):
        NS = rng.choice([2, 3, 4, 5, 6, 8])
        items = [rng.choice([1, 1, 2, 3, 5, 16]) for _ in range(rng.randint(1, 9))]
        assert run(mode, NS, items, rng)


def test_model_catches_a_missing_arrival(monkeypatch):
    """The check has teeth: a score group that never releases p_ready deadlocks the model."""
    original = roles

    def broken(mode, NS, items):
        gens = original(mode, NS, items)
        gens[4] = (ev for ev in gens[4] if ev != ("a", "p_ready"))
        return gens

    monkeypatch.setattr(sys.modules[__name__], "roles", broken)
    with pytest.raises(AssertionError, match="deadlock"):
        run(1, 3, [4, 2], random.Random(0))
