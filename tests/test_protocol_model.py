"""A model of the mbarrier protocols of the persistent attention kernels
(roles as Python generators, run over random interleavings), checking the
rule that parity waits impose.

An mbarrier wait names the parity of the phase it waits for, so a wait for
phase k returns as soon as the barrier's completed-phase count has the other
parity.  It is therefore only correct while phase k - 1 has completed and
phase k + 1 has not: started earlier, it passes at once (EARLY); started after
phase k + 1 completed, it never returns (ALIAS).  The model flags both, and a
set of roles that can no longer move (DEADLOCK).

Each role below follows the order of waits and arrivals of one role of a
kernel, with the barrier counts of its plan (a softmax group or the producer
warp's lanes are one role; their per-thread arrivals are one arrival).  The
configurations are the ones the kernels' plans may choose, including the
rules the plans enforce (producer warps <= ring stages, S buffers a multiple
of the softmax groups and at least groups x epilogue depth; the flash
kernel's ring has an even number of stages).  Negative cases show that the
model catches real mistakes: a "result ready" barrier pair shared by four
softmax groups (which ended in a bounded-wait timeout on a B200 before it was
indexed per group), plans the rules reject, and an odd flash ring.
"""
import random

import pytest


class Bar:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, self.name
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


class ProtocolError(AssertionError):
    pass


def run(roles: dict, bars: dict, seed: int, max_steps: int = 10 ** 6) -> None:
    rng = random.Random(seed)
    state = {n: next(g, None) for n, g in roles.items()}
    for _ in range(max_steps):
        ready = []
        for n, op in state.items():
            if op is None:
                continue
            if op[0] == "wait":
                b, k = bars[op[1]], op[2]
                if b.done >= k + 2:
                    raise ProtocolError(f"ALIAS: {n} waits for phase {k} of {op[1]}, {b.done} completed")
                if b.done < k:
                    if (b.done & 1) != (k & 1):
                        raise ProtocolError(f"EARLY: {n} waits for phase {k} of {op[1]}, {b.done} completed")
                    continue
                if b.done == k + 1:
                    ready.append(n)
            else:
                ready.append(n)
        if not ready:
            live = {n: op for n, op in state.items() if op is not None}
            if not live:
                return
            raise ProtocolError(f"DEADLOCK: {live}")
        n = rng.choice(ready)
        op = state[n]
        if op[0] == "arrive":
            bars[op[1]].arrive()
        state[n] = next(roles[n], None)
    raise ProtocolError("step limit")


# --------------------------------------------------------------- stack kernel
def stack_kernel(tiles, stages, nsb, wgs, pdepth, nprod, lce=False, conv_bars=4):
    """Producers, the S = QK^T issuer, the P V issuer and the softmax groups.
    With ``lce`` the filter warps of the decoupled arrangement are added: a
    result ring of two buffers, "written" on barrier tile % conv_bars."""
    np_ = wgs * pdepth
    bars = {}

    def B(name, count=1):
        bars[name] = Bar(name, count)

    for s in range(stages):
        B(f"full{s}"), B(f"empty{s}")
    for b in range(nsb):
        B(f"s_full{b}"), B(f"o_full{b}"), B(f"s_free{b}")
    for b in range(np_):
        B(f"p_full{b}")
    for b in range(2):
        B(f"halo{b}"), B(f"conv_free{b}")
    for b in range(conv_bars):
        B(f"conv_full{b}")

    def producer(w):
        for i in range(w, tiles, nprod):
            s = i % stages
            if i >= stages:
                yield ("wait", f"empty{s}", i // stages - 1)
            yield ("arrive", f"full{s}")

    def s_issuer():
        for i in range(tiles):
            s, sb = i % stages, i % nsb
            yield ("wait", f"full{s}", i // stages)
            if i >= nsb:
                yield ("wait", f"s_free{sb}", i // nsb - 1)
            yield ("arrive", f"s_full{sb}")

    def pv_issuer():
        for i in range(tiles):
            yield ("wait", f"p_full{i % np_}", i // np_)
            yield ("arrive", f"o_full{i % nsb}")
            yield ("arrive", f"empty{i % stages}")

    def filter_warps():
        issued = 0
        for _ in range(min(2, tiles)):
            yield ("arrive", f"halo{issued & 1}")
            issued += 1
        for i in range(tiles):
            yield ("wait", f"halo{i & 1}", i >> 1)
            if i >= 2:
                yield ("wait", f"conv_free{i & 1}", (i >> 1) - 1)
            yield ("arrive", f"conv_full{i % conv_bars}")
            if issued < tiles:
                yield ("arrive", f"halo{issued & 1}")
                issued += 1

    def softmax(wg):
        def epilogue(j):
            yield ("wait", f"o_full{j % nsb}", j // nsb)
            if lce:
                yield ("wait", f"conv_full{j % conv_bars}", j // conv_bars)
            yield ("arrive", f"s_free{j % nsb}")
            if lce:
                yield ("arrive", f"conv_free{j & 1}")

        last = -1
        for i in range(wg, tiles, wgs):
            yield ("wait", f"full{i % stages}", i // stages)
            yield ("wait", f"s_full{i % nsb}", i // nsb)
            yield ("arrive", f"p_full{i % np_}")
            if pdepth == 2:
                if last >= 0:
                    yield from epilogue(last)
                last = i
            else:
                yield from epilogue(i)
        if last >= 0:
            yield from epilogue(last)

    roles = {"s_issuer": s_issuer(), "pv_issuer": pv_issuer()}
    for w in range(nprod):
        roles[f"producer{w}"] = producer(w)
    for w in range(wgs):
        roles[f"softmax{w}"] = softmax(w)
    if lce:
        roles["filter"] = filter_warps()
    return roles, bars


def plan_allows(stages, nsb, wgs, pdepth, nprod):
    return nprod <= stages and wgs <= stages and nsb % wgs == 0 and nsb >= wgs * pdepth


STACK_PLANS = [  # (stages, S buffers, softmax groups, epilogue depth, producer warps)
    (9, 8, 4, 1, 2),   # stage 1
    (6, 8, 4, 1, 2),
    (5, 8, 2, 1, 2),   # stage 1 with the local context term in the epilogue
    (3, 4, 2, 2, 2),
    (2, 4, 2, 2, 2),
    (3, 2, 1, 2, 2),
    (2, 2, 2, 1, 2),
    (2, 2, 1, 1, 1),
]


@pytest.mark.parametrize("plan", STACK_PLANS, ids=[str(p) for p in STACK_PLANS])
def test_stack_kernel_protocol(plan):
    assert plan_allows(*plan)
    for tiles in (1, 2, 3, 7, 21, 22):
        for seed in range(40):
            run(*stack_kernel(tiles, *plan), seed)


@pytest.mark.parametrize("plan", [(5, 8, 4, 1, 2), (5, 8, 2, 2, 2), (5, 8, 2, 1, 2), (5, 4, 1, 1, 2)])
def test_stack_kernel_with_filter_warps_protocol(plan):
    """The decoupled local-context arrangement with "written" barriers per tile % 4."""
    for tiles in (1, 2, 3, 9, 22):
        for seed in range(40):
            run(*stack_kernel(tiles, *plan, lce=True, conv_bars=4), seed)


def test_plan_rules_are_needed():
    """A plan the rules reject fails in the model: more producer warps than
    stages, or fewer S buffers than groups x epilogue depth."""
    for plan in ((2, 4, 2, 1, 4), (4, 2, 2, 2, 2)):
        assert not plan_allows(*plan)
        with pytest.raises(ProtocolError):
            for seed in range(200):
                run(*stack_kernel(12, *plan), seed)


def test_model_catches_shared_result_barriers():
    """Two "written" barriers shared by four softmax groups: a group can start
    waiting for phase k while phase k - 1 is still open (EARLY)."""
    with pytest.raises(ProtocolError, match="EARLY"):
        for seed in range(200):
            run(*stack_kernel(22, 5, 8, 4, 1, 2, lce=True, conv_bars=2), seed)


# --------------------------------------------------------------- slice kernel
def slice_kernel(slices, units_per_slice, full_count):
    """Producer (boxes, and with producer-built masks a second arrival), S
    issuer, P V issuer, two softmax groups; two stages, two TMEM buffers."""
    stages = groups = 2
    units = slices * units_per_slice
    bars = {}
    for s in range(stages):
        bars[f"full{s}"] = Bar(f"full{s}", full_count)
        bars[f"empty{s}"] = Bar(f"empty{s}")
    for b in range(groups):
        for n in ("s_full", "o_full", "s_free", "p_full"):
            bars[f"{n}{b}"] = Bar(f"{n}{b}")

    def producer():
        for j in range(slices):
            s = j % stages
            if j >= stages:
                yield ("wait", f"empty{s}", j // stages - 1)
            for _ in range(full_count):
                yield ("arrive", f"full{s}")

    def s_issuer():
        for u in range(units):
            j, b = u // units_per_slice, u % groups
            yield ("wait", f"full{j % stages}", j // stages)
            if u >= groups:
                yield ("wait", f"s_free{b}", u // groups - 1)
            yield ("arrive", f"s_full{b}")

    def pv_issuer():
        for u in range(units):
            j, m, b = u // units_per_slice, u % units_per_slice, u % groups
            yield ("wait", f"p_full{b}", u // groups)
            yield ("arrive", f"o_full{b}")
            if m == units_per_slice - 1:
                yield ("arrive", f"empty{j % stages}")

    def softmax(g):
        for u in range(g, units, groups):
            j, b = u // units_per_slice, u % groups
            yield ("wait", f"full{j % stages}", j // stages)
            yield ("wait", f"s_full{b}", u // groups)
            yield ("arrive", f"p_full{b}")
            yield ("wait", f"o_full{b}", u // groups)
            yield ("arrive", f"s_free{b}")

    roles = {"producer": producer(), "s_issuer": s_issuer(), "pv_issuer": pv_issuer(),
             "softmax0": softmax(0), "softmax1": softmax(1)}
    return roles, bars


@pytest.mark.parametrize("full_count", [1, 2], ids=["masks_in_softmax", "masks_by_producer"])
def test_slice_kernel_protocol(full_count):
    for slices in (1, 2, 4, 5):
        for units in (1, 2):
            for seed in range(60):
                run(*slice_kernel(slices, units, full_count), seed)


# ---------------------------------------------------------------- warp kernel
def warp_kernel(slices, compute_warps):
    """Producer loading slices into two buffers; compute warps taking items in
    turn, each waiting for every slice's load (with or without items in it)
    before arriving on its buffer's "empty" barrier."""
    bars = {f"{n}{b}": Bar(f"{n}{b}", compute_warps if n == "empty" else 1)
            for n in ("full", "empty") for b in range(2)}

    def producer():
        for k in range(slices):
            if k >= 2:
                yield ("wait", f"empty{k & 1}", (k - 2) >> 1)
            yield ("arrive", f"full{k & 1}")

    def compute():
        for k in range(slices):
            yield ("wait", f"full{k & 1}", k >> 1)  # before its items, or alone if it has none
            yield ("arrive", f"empty{k & 1}")

    roles = {"producer": producer()}
    for w in range(compute_warps):
        roles[f"compute{w}"] = compute()
    return roles, bars


def test_warp_kernel_ring_protocol():
    for slices in (1, 2, 3, 5):
        for seed in range(60):
            run(*warp_kernel(slices, 4), seed)


# --------------------------------------------------------------- flash kernel
def flash_kernel(tiles, nb, stages=4):
    """Two softmax groups on alternate tiles (group = tile & 1), each with its
    Q buffer and two S/O buffers; K/V blocks go through one ring indexed by the
    step number s, where the steps of a tile pair interleave the pair's blocks
    (s = 2 nb pair + 2 b + (tile & 1)).  Steps of a missing last odd tile are
    skipped by every role."""
    groups = 2
    steps = ((tiles + 1) // 2) * 2 * nb
    bars = {}
    for g in range(groups):
        bars[f"q_full{g}"], bars[f"q_empty{g}"] = Bar(f"q_full{g}"), Bar(f"q_empty{g}")
        for y in range(2):
            for n in ("s_full", "s_free", "p_full", "o_full"):
                bars[f"{n}{g}{y}"] = Bar(f"{n}{g}{y}")
    for x in range(stages):
        bars[f"kv_full{x}"], bars[f"kv_empty{x}"] = Bar(f"kv_full{x}"), Bar(f"kv_empty{x}")

    def step_at(s):
        pair, r = divmod(s, 2 * nb)
        b, tile = r >> 1, 2 * pair + (r & 1)
        return (tile, b) if tile < tiles else None

    def producer():
        for s in range(steps):
            st = step_at(s)
            if st is None:
                continue
            tile, b = st
            g, use = tile & 1, tile >> 1
            if b == 0:
                if use > 0:
                    yield ("wait", f"q_empty{g}", use - 1)
                yield ("arrive", f"q_full{g}")
            if s >= stages:
                yield ("wait", f"kv_empty{s % stages}", s // stages - 1)
            yield ("arrive", f"kv_full{s % stages}")

    def s_issuer():
        for s in range(steps):
            st = step_at(s)
            if st is None:
                continue
            tile, b = st
            g, use = tile & 1, tile >> 1
            k = use * nb + b
            if b == 0:
                yield ("wait", f"q_full{g}", use)
            yield ("wait", f"kv_full{s % stages}", s // stages)
            if k >= 2:
                yield ("wait", f"s_free{g}{k & 1}", (k >> 1) - 1)
            yield ("arrive", f"s_full{g}{k & 1}")
            if b == nb - 1:
                yield ("arrive", f"q_empty{g}")

    def pv_issuer():
        for s in range(steps):
            st = step_at(s)
            if st is None:
                continue
            tile, b = st
            g, use = tile & 1, tile >> 1
            k = use * nb + b
            yield ("wait", f"p_full{g}{k & 1}", k >> 1)
            yield ("arrive", f"o_full{g}{k & 1}")
            yield ("arrive", f"kv_empty{s % stages}")

    def softmax(g):
        def fold(k):
            yield ("wait", f"o_full{g}{k & 1}", k >> 1)
            yield ("arrive", f"s_free{g}{k & 1}")

        for tile in range(g, tiles, groups):
            use = tile >> 1
            for b in range(nb):
                k = use * nb + b
                yield ("wait", f"s_full{g}{k & 1}", k >> 1)
                yield ("arrive", f"p_full{g}{k & 1}")
                if b > 0:
                    yield from fold(k - 1)
            yield from fold(use * nb + nb - 1)

    roles = {"producer": producer(), "s_issuer": s_issuer(), "pv_issuer": pv_issuer(),
             "softmax0": softmax(0), "softmax1": softmax(1)}
    return roles, bars


@pytest.mark.parametrize("nb", [1, 2, 8])
def test_flash_kernel_protocol(nb):
    """Four ring stages (even, like the steps of a pair), odd and even tile counts."""
    for tiles in (1, 2, 3, 5, 6):
        for seed in range(40):
            run(*flash_kernel(tiles, nb), seed)


def test_flash_ring_needs_an_even_stage_count_with_a_missing_tile():
    """With an odd number of stages a skipped step and a later real one can
    share a stage (here steps +1 and +4 of the last pair, four blocks per
    tile, three stages): the stage's phase count falls behind, and the real
    step's load waits for a release that never comes."""
    with pytest.raises(ProtocolError):
        for seed in range(100):
            run(*flash_kernel(3, 4, stages=3), seed)
