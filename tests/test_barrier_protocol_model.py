"""A model of the tensor-core kernels' barrier protocols, checked on the CPU.

Every warp role (TMA producer, feature map, MMA issuer, state group, scores/output group) is
written as the sequence of mbarrier waits (with the phase index it waits for) and arrivals it
performs, for the three modes of tc_forward.cu (0 aggregate, 1 causal output, 2 non-causal
output; 4 is the causal output with two MMA-issuing warps, as run at d = 64) and the causal
kernel on features of their own dimension, tc_causal.cu (mode 3), and
any list of work items of 1..16 chunks walked by one CTA.  A random scheduler interleaves the roles. The
test fails on a deadlock (no role can move) or on parity aliasing (a wait for a phase two or more
phases behind its barrier, which the hardware's parity test cannot tell from a pending one).
Each role's arrivals count as one (the kernel's thread counts are per role).  TMA loads and
tcgen05.commit arrivals ('i' events) are asynchronous: they land later, in any order, each as a
step of its own.  A wait may target only its barrier's pending phase or the one just completed
(the hardware tests a phase's parity): waiting further behind, or ahead, fails the test.  This
model mirrors the kernel's code by hand: change both together.
"""
import random
import sys

import pytest


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.completed = count, 0, 0


def roles_forward(mode, NS, items, two=False):
    """Generators of ('w', barrier, phase) and ('a', barrier) events, one per warp role."""

    def tma():
        g = 0
        for nc in items:
            for _ in range(nc):
                s = g % NS
                if g >= NS:
                    yield ("w", f"empty[{s}]", g // NS - 1)
                yield ("i", f"full[{s}]")
                g += 1
        for gg in range(max(0, g - NS), g):  # drain: every load has landed
            yield ("w", f"full[{gg % NS}]", gg // NS)

    def feature_map(team=0, teams=1):  # teams take alternate chunks
        g = 0
        for nc in items:
            for _ in range(nc):
                s = g % NS
                if g % teams == team:
                    yield ("w", f"full[{s}]", g // NS)
                    yield ("a", f"ready[{s}]")
                g += 1

    def mma():
        g = 0
        for j, nc in enumerate(items):
            b = j & 1
            if mode == 0 and j >= 2:
                yield ("w", f"item_empty[{b}]", (j >> 1) - 1)
            if mode == 2:
                yield ("w", f"item_full[{b}]", j >> 1)
            for _ in range(nc):
                s = g % NS
                yield ("w", f"ready[{s}]", g // NS)
                if mode == 0:
                    yield ("i", f"empty[{s}]")
                elif mode == 1:
                    yield ("w", "z_ready", g)
                    if g >= 1:  # the previous chunk's P V, interleaved with this chunk's scores
                        yield ("w", "p_ready", g - 1)
                        yield ("i", f"o_full[{(g - 1) & 1}]")
                        yield ("i", f"empty[{(g - 1) % NS}]")
                    yield ("i", "p_full")
                    if not two:  # else phi(Q) S_<c and the S update go to the second issuer
                        yield ("w", "s_ready", g)
                        if g >= 2:
                            yield ("w", f"o_empty[{g & 1}]", (g >> 1) - 1)
                        yield ("i", "s_full")
                else:
                    if g >= 2:
                        yield ("w", f"o_empty[{g & 1}]", (g >> 1) - 1)
                    yield ("i", f"o_full[{g & 1}]")
                    yield ("i", f"empty[{s}]")
                g += 1
            if mode == 0:
                yield ("i", f"item_full[{b}]")
            if mode == 2:
                yield ("i", f"item_empty[{b}]")
        if mode == 1 and g > 0:  # the last chunk's P V (after a second issuer's products)
            if two:
                yield ("w", "s_full", g - 1)
            yield ("w", "p_ready", g - 1)
            yield ("i", f"o_full[{(g - 1) & 1}]")
            yield ("i", f"empty[{(g - 1) % NS}]")
        yield ("i", "fin")
        yield ("w", "fin", 0)

    def mma2():  # causal: the second issuer, phi(Q) S_<c and the S update
        g = 0
        for nc in items:
            for _ in range(nc):
                yield ("w", f"ready[{g % NS}]", g // NS)
                yield ("w", "s_ready", g)
                if g >= 2:
                    yield ("w", f"o_empty[{g & 1}]", (g >> 1) - 1)
                yield ("i", "s_full")
                g += 1
        yield ("i", "fin2")
        yield ("w", "fin2", 0)

    def state_group():
        if mode == 1:
            g = 0
            for j, nc in enumerate(items):
                if j > 0:  # the previous item's last S and O products are done
                    yield ("w", "s_full", g - 1)
                yield ("a", "z_ready")
                yield ("a", "s_ready")
                for c in range(nc):
                    yield ("w", "p_full", g)
                    if not two:  # with two issuers the output group takes all the scores
                        yield ("a", "p_ready")
                        yield ("a", "rs_ready")
                    if c + 1 < nc:
                        yield ("w", "s_full", g)
                        yield ("a", "z_ready")
                        yield ("a", "s_ready")
                    g += 1
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

    def output_group():
        g = 0
        if mode == 1:
            for nc in items:
                for _ in range(nc):
                    yield ("w", "p_full", g)
                    if not two:
                        yield ("w", "rs_ready", g)
                    yield ("a", "p_ready")
                    if g >= 1:
                        yield ("w", f"o_full[{(g - 1) & 1}]", (g - 1) >> 1)
                        yield ("a", f"o_empty[{(g - 1) & 1}]")
                    g += 1
            if g > 0:
                yield ("w", f"o_full[{(g - 1) & 1}]", (g - 1) >> 1)
                yield ("a", f"o_empty[{(g - 1) & 1}]")
        elif mode == 2:
            for nc in items:
                for _ in range(nc):
                    yield ("w", f"o_full[{g & 1}]", g >> 1)
                    yield ("a", f"o_empty[{g & 1}]")
                    g += 1

    # the aggregate kernel splits its feature map into two teams when the stages divide evenly
    teams = 2 if mode == 0 and NS % 2 == 0 else 1
    roles = [tma(), feature_map(0, teams), mma(), state_group(), output_group()]
    if teams == 2:
        roles.append(feature_map(1, 2))
    return roles + [mma2()] if two else roles


def roles_features(NS, items):
    """tc_causal.cu: 128-token chunks, the scores rounded in tensor memory, z summed by the
    feature warps."""

    def tma():
        g = 0
        for nc in items:
            for _ in range(nc):
                s = g % NS
                if g >= NS:
                    yield ("w", f"empty[{s}]", g // NS - 1)
                yield ("i", f"full[{s}]")
                g += 1
        for gg in range(max(0, g - NS), g):
            yield ("w", f"full[{gg % NS}]", gg // NS)

    def features():
        g = 0
        for nc in items:
            for _ in range(nc):
                s = g % NS
                yield ("w", f"full[{s}]", g // NS)
                yield ("a", f"ready[{s}]")
                yield ("a", "zsync")  # every feature warp's column sums are in
                yield ("w", "zsync", g)
                g += 1

    def mma():
        g = 0
        for nc in items:
            for _ in range(nc):
                s = g % NS
                yield ("w", f"ready[{s}]", g // NS)
                yield ("w", "s_ready", g)
                if g >= 2:
                    yield ("w", f"o_empty[{g & 1}]", (g >> 1) - 1)
                yield ("i", "p_full")  # the scores
                yield ("i", "s_full")  # F(Q) S_<c and the state update
                yield ("w", "p_ready", g)
                yield ("i", f"o_full[{g & 1}]")  # P V
                yield ("i", f"empty[{s}]")
                g += 1
        yield ("i", "fin")
        yield ("w", "fin", 0)

    def state_group():
        g = 0
        for j, nc in enumerate(items):
            if j > 0:  # the previous item's last products are done with S and its operand
                yield ("w", "s_full", g - 1)
            yield ("a", "s_ready")
            for c in range(nc):
                if c + 1 < nc:
                    yield ("w", "s_full", g)
                    yield ("a", "s_ready")
                g += 1

    def output_group():
        g = 0
        for nc in items:
            for _ in range(nc):
                if g >= 1:
                    yield ("w", f"o_full[{(g - 1) & 1}]", (g - 1) >> 1)
                    yield ("a", f"o_empty[{(g - 1) & 1}]")
                yield ("w", f"ready[{g % NS}]", g // NS)  # F(q).z of this stage
                yield ("w", "p_full", g)
                yield ("a", "p_ready")
                g += 1
        if g > 0:
            yield ("w", f"o_full[{(g - 1) & 1}]", (g - 1) >> 1)
            yield ("a", f"o_empty[{(g - 1) & 1}]")

    return [tma(), features(), mma(), state_group(), output_group()]


def roles(mode, NS, items):
    if mode == 3:
        return roles_features(NS, items)
    if mode == 4:
        return roles_forward(1, NS, items, two=True)
    return roles_forward(mode, NS, items)


def run(mode, NS, items, rng):
    # arrivals per phase; tc_forward.cu's causal mode: both drain groups release p_ready
    counts = {"p_ready": 2} if mode == 1 else {}
    bars = {}

    def bar(name):
        if name not in bars:
            bars[name] = Barrier(counts.get(name.split("[")[0], 1))
        return bars[name]

    gens = roles(mode, NS, items)
    cur = [next(gen, None) for gen in gens]
    inflight = []  # asynchronous arrivals issued and not yet landed

    def arrive(name):
        b = bar(name)
        b.pending += 1
        if b.pending == b.count:
            b.pending, b.completed = 0, b.completed + 1

    while True:
        runnable = []
        for r, ev in enumerate(cur):
            if ev is None:
                continue
            if ev[0] in ("a", "i"):
                runnable.append(r)
                continue
            b, phase = bar(ev[1]), ev[2]
            assert b.completed < phase + 2, f"parity aliasing: {ev}, mode {mode}, items {items}"
            # the hardware tests a phase's parity, so a wait may only target the pending phase
            # or the one just completed: a wait two phases ahead would pass at once
            assert phase <= b.completed, f"wait ahead of its barrier: {ev}, mode {mode}, items {items}"
            if b.completed > phase:  # the waited-for phase has completed
                runnable.append(r)
        if not runnable and not inflight:
            assert all(ev is None for ev in cur), f"deadlock at {cur}, mode {mode}, items {items}"
            return True
        if inflight and (not runnable or rng.random() < 0.3):
            arrive(inflight.pop(rng.randrange(len(inflight))))  # one landing, in any order
            continue
        r = rng.choice(runnable)
        if cur[r][0] == "a":
            arrive(cur[r][1])
        elif cur[r][0] == "i":
            inflight.append(cur[r][1])
        cur[r] = next(gens[r], None)


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4])
def test_protocol_has_no_deadlock_or_aliasing(mode):
    rng = random.Random(1000 + mode)
    for _ in range(1500):
        NS = rng.choice([2, 3, 4, 5, 6, 8])
        items = [rng.choice([1, 1, 2, 3, 5, 16]) for _ in range(rng.randint(1, 9))]
        assert run(mode, NS, items, rng)


def test_model_catches_a_missing_arrival(monkeypatch):
    """The check has teeth: a state group that never releases p_ready deadlocks the model."""
    original = roles

    def broken(mode, NS, items):
        gens = original(mode, NS, items)
        gens[3] = (ev for ev in gens[3] if ev != ("a", "p_ready"))
        return gens

    monkeypatch.setattr(sys.modules[__name__], "roles", broken)
    with pytest.raises(AssertionError, match="deadlock"):
        run(1, 3, [4, 2], random.Random(0))
