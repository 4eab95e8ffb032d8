"""Model check of the GEMM kernels' barrier protocol (gemm_sm100.cuh,
gemm_pair_sm100.cuh), on the CPU.

Every warp role of one CTA is played as a coroutine against mbarriers with the
hardware's phase semantics: a barrier completes a phase when its arrival count
is reached, and a parity wait passes while the current (incomplete) phase's
parity differs from the one asked for, so it only tells the latest two phases
apart.  Random schedules (including a tensor pipe that completes MMAs, in
order, at arbitrary times) check that

* no schedule deadlocks, and
* every wait passes on exactly the phase its role means (not an older phase
  still showing the right parity, nor a newer one that reused the buffer).

The roles: code-tile producer (empty -> full), scale-tile producer (sfree
-> sfload, groups of two stages that never span two tiles), gate (full +
sf_full -> ready count), MMA issuer (ready, acc_empty -> commits to empty /
acc_full / mma_done), scale warps (sfload and empty of stage kg - slots ->
sf_full, sfree after a group's last stage; with GELU they drain a share of
each tile's shared accumulator columns and arrive on acc_empty; the last tile
after mma_done), epilogue warps (acc_full -> acc_empty), and the producers'
tail waits before exit.  The CTA-pair form is modelled too: per-CTA empty,
scale-group, accumulator and MMA-done barriers; the leader's full, sf_full and
acc_empty counting both CTAs; the MMA commits arriving at both CTAs.  The
abort paths (a bounded wait running out) are not modelled.

The planted variants re-create three mistakes this protocol rules out and
must be caught: the scale warps' last-tile wait as a parity wait on acc_full
(an older tile's phase can satisfy it when K spans few stages), waiting on
every tile's acc_full in order after the slots are written (a warp that far
behind no longer tells the phases apart), and the GELU share drained after,
instead of before, the wait on a stage of the next tile (that stage's MMAs
wait for the release the share is part of: a deadlock)."""
import itertools
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.completed = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def passes(self, phase):
        # the hardware parity test for "phase `phase` has completed"
        return (self.completed & 1) != (phase & 1)


class Violation(AssertionError):
    pass


def wait(bar, phase, what):
    return ("wait", bar, phase, what)


def until(cond):
    return ("until", cond)


SF_GROUP = 2  # stages per scale-tile copy


def run_protocol(T, num_kt, stages, slots, gelu, seed, n_epi=2, n_scale=2, groups=3, pair=False,
                 last_wait="mma_done", in_order_waits=False, help_before_wait=True):
    """One CTA, or a CTA pair (pair=True): each CTA has its own empty, sfload,
    sfree, acc_full and mma_done barriers; the leader's full, sf_full and
    acc_empty count both CTAs' arrivals; the leader's gate and MMA issuer run
    alone, and the MMA commits arrive at both CTAs' barriers."""
    rng = random.Random(seed)
    ctas = 2 if pair else 1
    G = T * num_kt  # stages each CTA walks
    U = T * -(-num_kt // SF_GROUP)  # scale-tile groups (a group never spans two tiles)
    # per CTA
    sfload = [[Bar(1) for _ in range(groups)] for _ in range(ctas)]
    sfree = [[Bar(n_scale) for _ in range(groups)] for _ in range(ctas)]
    empty = [[Bar(1) for _ in range(stages)] for _ in range(ctas)]
    acc_full = [[Bar(1), Bar(1)] for _ in range(ctas)]
    mma_done = [Bar(1) for _ in range(ctas)]
    # the leader's, counting both CTAs
    full = [Bar(ctas) for _ in range(stages)]  # each CTA's tile landing
    sf_full = [Bar(n_scale * ctas) for _ in range(slots)]
    acc_empty = Bar((n_epi + (n_scale if gelu else 0)) * ctas)
    st = {"ready": 0}
    pipe = []  # commits (lists of barriers), completed in issue order by the tensor pipe

    def producer(c):
        for g in range(G):
            yield wait(empty[c][g % stages], g // stages - 1, "producer empty")
            full[g % stages].arrive()  # this CTA's TMA fill completing
        if c == 0:  # no exit with copies in flight (the leader's barriers count both)
            for u in range(max(0, G - stages), G):
                yield wait(full[u % stages], u // stages, "producer tail full")

    def sf_producer(c):
        for u in range(U):
            yield wait(sfree[c][u % groups], u // groups - 1, "sf producer sfree")
            sfload[c][u % groups].arrive()
        for u in range(max(0, U - groups), U):
            yield wait(sfload[c][u % groups], u // groups, "sf producer tail sfload")

    def gate():
        for g in range(G):
            yield wait(full[g % stages], g // stages, "gate full")
            yield wait(sf_full[g % slots], g // slots, "gate sf_full")
            st["ready"] = g + 1

    def mma():
        g = 0
        for t in range(T):
            for kt in range(num_kt):
                yield until(lambda g=g: st["ready"] > g)
                if kt == 0 and t > 0:
                    yield wait(acc_empty, t - 1, "mma acc_empty")
                pipe.append([empty[c][g % stages] for c in range(ctas)])
                g += 1
            pipe.append([acc_full[c][t & 1] for c in range(ctas)])
        pipe.append([mma_done[c] for c in range(ctas)])

    def epilogue(c):
        for t in range(T):
            yield wait(acc_full[c][t & 1], t // 2, "epilogue acc_full")
            if t == T - 1:
                break  # the last tile: nothing waits for its release
            acc_empty.arrive()

    def scale_warp(c):
        help_next = 0
        u = 0  # scale-tile groups consumed

        def help_one(t):
            yield wait(acc_full[c][t & 1], t // 2, "help acc_full")
            acc_empty.arrive()

        for g in range(G):
            kt = g % num_kt
            if kt % SF_GROUP == 0:
                yield wait(sfload[c][u % groups], u // groups, "scale sfload")
            if g >= slots:
                # before_wait(kg): drain shared columns of every tile whose
                # release the awaited stage's MMAs may need
                if not help_before_wait:
                    yield wait(empty[c][(g - slots) % stages], (g - slots) // stages, "scale empty")
                while gelu and help_next < T - 1 and g - slots >= (help_next + 1) * num_kt:
                    yield from help_one(help_next)
                    help_next += 1
                if help_before_wait:
                    yield wait(empty[c][(g - slots) % stages], (g - slots) // stages, "scale empty")
            sf_full[g % slots].arrive()
            if kt % SF_GROUP == SF_GROUP - 1 or kt == num_kt - 1:
                sfree[c][u % groups].arrive()
                u += 1
        while gelu and help_next < T - 1:
            yield from help_one(help_next)
            help_next += 1
        if in_order_waits:
            for t in range(help_next, T - 1):
                yield wait(acc_full[c][t & 1], t // 2, "in-order acc_full")
        if T > 0:
            if last_wait == "mma_done":
                yield wait(mma_done[c], 0, "last-tile mma_done")
            else:
                yield wait(acc_full[c][(T - 1) & 1], (T - 1) // 2, "last-tile acc_full")

    actors = [gate(), mma()]
    for c in range(ctas):
        actors += [producer(c), sf_producer(c)] + [epilogue(c) for _ in range(n_epi)] + \
                  [scale_warp(c) for _ in range(n_scale)]
    pending = {}
    for a in actors:
        try:
            pending[a] = next(a)
        except StopIteration:
            pass
    while pending or pipe:
        runnable = [a for a, cnd in pending.items() if
                    (cnd[0] == "wait" and cnd[1].passes(cnd[2])) or (cnd[0] == "until" and cnd[1]())]
        choices = runnable + (["pipe"] if pipe else [])
        if not choices:
            raise Violation("deadlock: " + ", ".join(cnd[3] for cnd in pending.values() if cnd[0] == "wait"))
        a = rng.choice(choices)
        if a == "pipe":
            for bar in pipe.pop(0):
                bar.arrive()
            continue
        cnd = pending[a]
        if cnd[0] == "wait" and cnd[1].completed != cnd[2] + 1:
            kind = "an older" if cnd[1].completed < cnd[2] + 1 else "a newer"
            raise Violation(f"{cnd[3]} for phase {cnd[2]} passed on {kind} phase "
                            f"({cnd[1].completed} completed)")
        try:
            pending[a] = next(a)
        except StopIteration:
            del pending[a]
    return True


# STAGES >= slots, as the kernels assert; num_kt from one stage up to past the
# slot count; 1 to 5 tiles per CTA (both accumulators, the last-tile split)
# and 2 to 4 scale-tile groups in flight
CASES = [(T, kt, s, sl, gelu) for T, kt, (s, sl), gelu in
         itertools.product([1, 2, 3, 5], [1, 2, 3, 7], [(4, 4), (5, 4), (6, 6)], [False, True])]


@pytest.mark.parametrize("pair", [False, True])
@pytest.mark.parametrize("T,num_kt,stages,slots,gelu", CASES)
def test_protocol_has_no_deadlock_or_phase_alias(T, num_kt, stages, slots, gelu, pair):
    for seed in range(12):
        run_protocol(T, num_kt, stages, slots, gelu, seed, groups=2 + seed % 3, pair=pair)


def _caught(gelu=False, **kw):
    for pair in (False, True):
        for T, num_kt in [(3, 1), (5, 1), (4, 2), (5, 3), (3, 7)]:
            for seed in range(40):
                try:
                    run_protocol(T, num_kt, 6, 6, gelu, seed, pair=pair, **kw)
                except Violation as e:
                    return str(e)
    return None


def test_planted_last_tile_parity_wait_is_caught():
    msg = _caught(last_wait="acc_full")
    assert msg is not None and "older phase" in msg, msg


def test_planted_in_order_waits_are_caught():
    msg = _caught(in_order_waits=True)
    assert msg is not None, msg


def test_planted_help_after_the_wait_is_caught():
    msg = _caught(gelu=True, help_before_wait=False)
    assert msg is not None and msg.startswith("deadlock"), msg
