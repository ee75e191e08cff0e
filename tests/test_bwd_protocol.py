"""A discrete-event model of the dK/dV backward kernel's barrier protocol, checked on the CPU.

attn_bwd_dkdv_kernel's roles talk only through mbarriers: the TMA producer (K and V once, then query tiles of
Q, dO, LSE and Delta through a 3-slot ring), the MMA warp (in the order A(0), A(1), B(0), A(2), B(1), ...,
B(n-1): A writes dP^T, then S^T into tensor-memory buffer i % 2, B computes dQ^T, then dV and dK), and two softmax groups
that take the tiles in turn (group g owns the tiles i = g mod 2 and buffer g). Each group hands the 32 KB dQ
staging buffer to the other in tile order through one barrier. Barrier counts follow the kernel: the
softmax-side barriers count warps, so a group of four warps is one actor arriving 4. MMAs, commits and copies
complete at once (timing does not matter for these properties). Over random step counts and interleavings the
model checks that

  * every role runs to the end (no deadlock: a role only waits for something another role will still do), and
  * no parity wait can be fooled: when a wait for phase n of a barrier succeeds, phase n + 1 has not completed
    yet (a parity wait only sees the current phase's parity, so a waiter two phases behind would hang or pass
    on the wrong phase).

Two negative controls must fail: the dQ staging hand-off waiting for the tile's own release (an off-by-one)
deadlocks, and a producer that refills ring slots without waiting for their release runs the softmax groups'
waits two phases behind.
"""
import random

import pytest

STAGES = 3  # Q / dO / LSE / Delta ring depth


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        assert self.pending <= self.count, "more arrivals than the phase expects"
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


class Model:
    def __init__(self, ns, bug=None):
        self.ns, self.bug = ns, bug
        self.b = {"kv_full": Barrier(1), "stage_free": Barrier(1), "acc_done": Barrier(1), "drain": Barrier(1)}
        for s in range(STAGES):
            self.b[f"q_full{s}"] = Barrier(1)
            self.b[f"q_empty{s}"] = Barrier(1)
        for r in range(2):
            for name, count in (("s_full", 1), ("p_full", 4), ("dq_full", 1), ("dq_empty", 4), ("b_done", 1)):
                self.b[f"{name}{r}"] = Barrier(count)
        self.epilogue_named = 0  # groups that reached the epilogue's named barrier
        self.violations = []

    def wait(self, name, n):
        """Wait for completion n (0-based) of a barrier: the kernel's parity wait on phase n."""
        bar = self.b[name]

        def ready():
            if bar.done > n + 1:
                self.violations.append((name, n, bar.done))
            return bar.done > n
        return ready


def producer(m):
    m.b["kv_full"].arrive()
    for i in range(m.ns):
        s = i % STAGES
        if i >= STAGES and m.bug != "no_ring_release_wait":
            yield m.wait(f"q_empty{s}", (i - STAGES) // STAGES)
        m.b[f"q_full{s}"].arrive()


def mma(m):
    yield m.wait("kv_full", 0)

    def issue_a(i):
        s, rb = i % STAGES, i & 1
        yield m.wait(f"q_full{s}", i // STAGES)
        if i >= 2:
            yield m.wait(f"dq_empty{rb}", (i - 2) >> 1)  # dP^T overwrites the dQ^T columns
            yield m.wait(f"b_done{rb}", (i - 2) >> 1)    # S^T overwrites P^T, dS^T
        m.b[f"s_full{rb}"].arrive()

    def issue_b(i):
        s, rb = i % STAGES, i & 1
        yield m.wait(f"p_full{rb}", i >> 1)
        m.b[f"dq_full{rb}"].arrive()
        m.b[f"b_done{rb}"].arrive()
        m.b[f"q_empty{s}"].arrive()

    yield from issue_a(0)
    for i in range(1, m.ns):
        yield from issue_a(i)
        yield from issue_b(i - 1)
    yield from issue_b(m.ns - 1)
    m.b["acc_done"].arrive()
    m.b["drain"].arrive()
    yield m.wait("drain", 0)


def softmax_group(m, g):
    for i in range(g, m.ns, 2):
        s, rb = i % STAGES, g
        yield m.wait(f"q_full{s}", i // STAGES)
        yield m.wait(f"s_full{rb}", i >> 1)
        m.b[f"p_full{rb}"].arrive(4)
        yield m.wait(f"dq_full{rb}", i >> 1)
        m.b[f"dq_empty{rb}"].arrive(4)
        if m.bug == "stage_wait_own_release":
            yield m.wait("stage_free", i)
        elif i > 0:
            yield m.wait("stage_free", i - 1)
        m.b["stage_free"].arrive()  # the group leader, once the bulk reduction has read the staging buffer
    yield m.wait("acc_done", 0)
    m.epilogue_named += 1
    yield lambda: m.epilogue_named == 2  # named barrier of both groups before the dK / dV stores


def run(ns, seed, bug=None):
    """Random interleaving of the roles; returns (finished, violations)."""
    m = Model(ns, bug)
    rng = random.Random(seed)
    roles = {"tma": producer(m), "mma": mma(m), "g0": softmax_group(m, 0), "g1": softmax_group(m, 1)}
    waiting = {name: None for name in roles}
    alive = set(roles)
    while alive:
        runnable = [name for name in sorted(alive) if waiting[name] is None or waiting[name]()]
        if not runnable:
            return False, m.violations
        name = rng.choice(runnable)
        try:
            waiting[name] = next(roles[name])
        except StopIteration:
            alive.discard(name)
    return True, m.violations


def test_protocol_has_no_deadlock_and_no_ambiguous_parity_wait():
    """Step counts of every shape the kernel meets: one tile, odd counts (a lone last A/B), the G * n steps of
    grouped-query heads, and long walks."""
    rng = random.Random(99)
    for trial in range(1500):
        ns = rng.choice([1, 2, 3, 4, 5]) if rng.random() < 0.4 else rng.randint(1, 64)
        finished, violations = run(ns, trial)
        assert finished, f"deadlock with {ns} steps (schedule seed {trial})"
        assert not violations, f"parity wait two phases behind with {ns} steps: {violations[:3]}"


@pytest.mark.parametrize("ns", [1, 2, 3, 6, 7, 32, 33])
def test_protocol_corner_step_counts(ns):
    for seed in range(100):
        finished, violations = run(ns, seed)
        assert finished and not violations


def test_model_catches_a_deadlocking_hand_off():
    """Negative control: tile i waiting for its own release of the staging buffer never proceeds."""
    assert not run(1, 0, bug="stage_wait_own_release")[0]
    assert not any(run(ns, seed, bug="stage_wait_own_release")[0] for ns in (2, 5) for seed in range(20))


def test_model_catches_a_ring_overrun():
    """Negative control: without the wait for a slot's release the producer can complete a slot's phases two
    ahead of a softmax group's wait."""
    rng = random.Random(3)
    caught = sum(bool(run(rng.randint(7, 40), seed, bug="no_ring_release_wait")[1]) for seed in range(200))
    assert caught > 0
