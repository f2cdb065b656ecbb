"""Model check of the query-major kernel's barrier protocol (host-side, no GPU).

paged_prefill_kernel coordinates a load warp, one MMA-issuing thread and two
softmax warpgroups through mbarriers waited on by phase parity.  A parity wait
is only meaningful while the barrier is at most one phase away from the phase
waited for: if it is behind, the wait passes at once (an earlier phase has the
same parity); if it is two ahead, it blocks for good.  This test runs a
discrete-event model of the kernel's schedule (the same order of waits,
arrivals, loads and tcgen05 commits as the kernel; tcgen05 MMAs execute in
issue order and a commit completes once every earlier MMA has) under random
interleavings and latencies, and checks that

  * every actor finishes (no deadlock) for any number of key tiles and ring
    depth;
  * every parity wait starts with the barrier at the phase waited for or one
    past it;
  * a ring entry is refilled only after every MMA that reads its previous tile
    has completed, and an MMA reads a tile only after it has landed (and, for
    the last V tile past the context, after its rows were zeroed);
  * a softmax warpgroup reads S_x(j) only after that MMA completed and writes
    P_x(j) only after P_x(j-1) . V has completed.
"""
import random

import pytest


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0   # done = completed phases

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


class Violation(AssertionError):
    pass


def run_model(nk, kE, tail, seed, mutation=None):
    rng = random.Random(seed)
    full = [Barrier(1) for _ in range(kE)]
    empty = [Barrier(1) for _ in range(kE)]
    s_full, p_full = [Barrier(1), Barrier(1)], [Barrier(1), Barrier(1)]
    o_full, v_tail = Barrier(1), Barrier(1)

    landed = set()            # ring entries' tiles whose load completed: index i (K_j = 2j, V_j = 2j + 1)
    tail_zeroed = [False]
    mma_done = set()          # completed MMA groups: ("S", x, j) / ("PV", x, j)
    pipe = []                 # in-order tensor pipe: ("mma", key, reads) or ("commit", barrier)
    loads = []                # in-flight TMA loads: [remaining steps, tile index]
    entry_tile = {}           # entry -> tile index it holds

    def wait(bar, phase):
        """Generator: parity wait for `phase` of `bar`; checks the one-phase window."""
        if bar.done not in (phase, phase + 1):
            raise Violation(f"parity wait for phase {phase} started at phase {bar.done}")
        while bar.done <= phase:
            yield

    def issue_mma(key, reads):
        for i in reads:
            if i not in landed:
                raise Violation(f"{key} issued before tile {i} landed")
        pipe.append(("mma", key, reads))

    def load_warp():
        for i in range(2 * nk):
            e = i % kE
            if i >= kE:
                yield from wait(empty[e], (i - kE) // kE)
                prev = i - kE
                j, is_v = prev // 2, prev % 2 == 1
                readers = [("PV", x, j) for x in (0, 1)] if is_v else [("S", x, j) for x in (0, 1)]
                if not all(r in mma_done for r in readers):
                    raise Violation(f"entry {e} refilled with tile {i} before {readers} completed")
            entry_tile[e] = i
            loads.append([rng.randint(1, 6), i])
            yield
        if tail:
            i = 2 * nk - 1
            yield from wait(full[i % kE], i // kE)
            for _ in range(rng.randint(1, 8)):   # the warp's stores of zeros
                yield
            tail_zeroed[0] = True
            v_tail.arrive()

    def mma_thread():
        yield from wait(full[0], 0)
        for x in (0, 1):
            issue_mma(("S", x, 0), [0])
            pipe.append(("commit", s_full[x]))
        pipe.append(("commit", empty[0]))
        for j in range(nk):
            vi = 2 * j + 1
            yield from wait(full[vi % kE], vi // kE)
            if tail and j == nk - 1 and mutation != "no_tail_wait":
                yield from wait(v_tail, 0)
            more = j + 1 < nk
            ki = 2 * (j + 1)
            for x in (0, 1):
                yield from wait(p_full[x], j)
                if tail and j == nk - 1 and not tail_zeroed[0]:
                    raise Violation("last P . V issued before the V tail was zeroed")
                if mutation == "early_v_release" and x == 1:
                    pipe.append(("commit", empty[vi % kE]))
                if more and mutation == "s_before_pv":
                    if x == 0:
                        yield from wait(full[ki % kE], ki // kE)
                    issue_mma(("S", x, j + 1), [ki])
                    pipe.append(("commit", s_full[x]))
                issue_mma(("PV", x, j), [vi])
                if x == 1 and mutation != "early_v_release":
                    pipe.append(("commit", empty[vi % kE]))
                if more:
                    if mutation != "s_before_pv":
                        if x == 0:
                            yield from wait(full[ki % kE], ki // kE)
                        issue_mma(("S", x, j + 1), [ki])
                        pipe.append(("commit", s_full[x]))
                    if x == 1:
                        pipe.append(("commit", empty[ki % kE]))
                yield
            if not more:
                pipe.append(("commit", o_full))

    def softmax(x):
        for j in range(nk):
            yield from wait(s_full[x], j)
            if ("S", x, j) not in mma_done:
                raise Violation(f"softmax {x} read S({j}) before it completed")
            for _ in range(rng.randint(1, 4)):   # exponentials
                yield
            if j > 0 and ("PV", x, j - 1) not in mma_done:
                raise Violation(f"softmax {x} wrote P({j}) before P({j - 1}) . V completed")
            p_full[x].arrive()
        yield from wait(o_full, 0)

    actors = [load_warp(), mma_thread(), softmax(0), softmax(1)]
    alive = list(range(len(actors)))
    for _ in range(200000):
        if not alive and not pipe and not loads:
            return
        # loads land after their latency
        for ld in loads:
            ld[0] -= 1
        for ld in [ld for ld in loads if ld[0] <= 0]:
            loads.remove(ld)
            landed.add(ld[1])
            full[ld[1] % kE].arrive()
        # the tensor pipe retires its head with some probability
        if pipe and rng.random() < 0.5:
            kind, a, *_ = pipe.pop(0)
            if kind == "mma":
                mma_done.add(a)
            else:
                a.arrive()
        # a random actor takes one step
        if alive:
            k = rng.choice(alive)
            try:
                next(actors[k])
            except StopIteration:
                alive.remove(k)
    raise Violation(f"no progress (deadlock): actors still waiting {alive}, pipe {len(pipe)}, loads {len(loads)}")


@pytest.mark.parametrize("kE", [5, 8])
@pytest.mark.parametrize("nk", [1, 2, 3, 4, 5, 6, 9, 17])
@pytest.mark.parametrize("tail", [False, True])
def test_protocol_has_no_deadlock_aliasing_or_hazard(nk, kE, tail):
    for seed in range(12):
        run_model(nk, kE, tail, seed * 1000 + nk * 10 + kE)


@pytest.mark.parametrize("mutation", ["early_v_release", "no_tail_wait", "s_before_pv"])
def test_model_catches_a_broken_schedule(mutation):
    # the check itself: each of these reorderings breaks the protocol, and
    # some interleaving must expose it
    caught = 0
    for seed in range(40):
        try:
            run_model(6, 5, True, seed, mutation)
        except Violation:
            caught += 1
    assert caught > 0
