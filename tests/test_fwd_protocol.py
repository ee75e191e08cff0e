"""A discrete-event model of the persistent forward kernel's barrier protocol, checked on the CPU.

attn_fwd_kernel's roles talk only through mbarriers (and, between its two softmax groups, three named barriers
per work item). This model replays each role's waits and arrivals in the kernel's order -- the K and V
producers with the one Q buffer, the MMA warp, the two softmax groups with their epilogue, the output-store
warp -- with barrier counts as in the kernel (softmax-side barriers count warps: a group of four warps is one
actor arriving 4). Loads and MMAs complete at once (timing does not matter for these properties). Over random
work-item mixes and random interleavings it checks that

  * every role runs to the end (no deadlock: a role only waits for something another role will still do), and
  * no parity wait can be fooled: when a wait for phase n of a barrier succeeds, phase n + 1 has not completed
    yet (a parity wait only sees the current phase's parity, so a waiter two phases behind would hang).

A negative control (an MMA issue order, tried during development, that ran the S tiles of item k+2 before the
last PVs of item k) must deadlock in the model.
"""
import random

import pytest

STAGES = 3  # K and V ring depth


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        assert self.pending <= self.count, "more arrivals than the phase expects"
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


class Model:
    def __init__(self, items):
        self.items = items
        self.b = {}
        for name, count in [("q_full", 1), ("q_tmem", 8), ("q_free", 1), ("o_staged", 8), ("o_final", 1)]:
            self.b[name] = Barrier(count)
        for s in range(STAGES):
            for name in ("k_full", "k_empty", "v_full", "v_empty"):
                self.b[f"{name}{s}"] = Barrier(1)
        for s in range(2):
            for name, count in (("s_full", 1), ("s_free", 4), ("p_full", 4), ("xchg", 4), ("pv_done", 1)):
                self.b[f"{name}{s}"] = Barrier(count)
        self.named = {"A": [0, 0], "B": [0, 0], "C": [0, 0]}  # passes of each named barrier, per group
        self.violations = []

    def wait(self, name, n):
        """Wait for completion n (0-based) of a barrier: the kernel's parity wait on phase n."""
        bar = self.b[name]

        def ready():
            if bar.done > n + 1:
                self.violations.append((name, n, bar.done))
            return bar.done > n
        return ready

    def named_barrier(self, which, g, k):
        self.named[which][g] += 1
        return lambda: min(self.named[which]) > k


def producer(m, is_k):
    t0 = 0
    for k, n in enumerate(m.items):
        if is_k:  # one Q buffer, shared with the output staging of item k-2
            if k == 1:
                yield m.wait("q_tmem", 0)
            if k >= 2:
                yield m.wait("q_free", k - 2)
            m.b["q_full"].arrive()
        for j in range(n):
            t = t0 + j
            s = t % STAGES
            if t >= STAGES:
                yield m.wait(("k_empty" if is_k else "v_empty") + str(s), (t - STAGES) // STAGES)
            m.b[("k_full" if is_k else "v_full") + str(s)].arrive()
        t0 += n


def mma(m, order="per_item"):
    def issue_s(t):
        if t >= 2:
            yield m.wait(f"s_free{t & 1}", (t - 2) // 2)
        yield m.wait(f"k_full{t % STAGES}", t // STAGES)
        m.b[f"s_full{t & 1}"].arrive()
        m.b[f"k_empty{t % STAGES}"].arrive()

    def issue_pv(t):
        yield m.wait(f"p_full{t & 1}", t // 2)
        yield m.wait(f"v_full{t % STAGES}", t // STAGES)
        m.b[f"pv_done{t & 1}"].arrive()
        m.b[f"v_empty{t % STAGES}"].arrive()

    if order == "per_item":  # the kernel: per item S(0), S(1), S(2), PV(0), ..., PV(n-1), then o_final
        t0 = 0
        for k, n in enumerate(m.items):
            yield m.wait("q_tmem", k)
            for j in range(n + 2):
                if j < n:
                    yield from issue_s(t0 + j)
                if j >= 2:
                    yield from issue_pv(t0 + j - 2)
            m.b["o_final"].arrive()
            t0 += n
    else:  # negative control: one stream over all items, PVs two tiles behind, no flush at item starts
        starts = [sum(m.items[:k]) for k in range(len(m.items))]
        ends = {starts[k] + n - 1 for k, n in enumerate(m.items)}
        total = sum(m.items)
        tp = 0
        for ts in range(total):
            if ts in starts:
                yield m.wait("q_tmem", starts.index(ts))
            yield from issue_s(ts)
            if ts + 1 - tp >= 3:
                yield from issue_pv(tp)
                if tp in ends:
                    m.b["o_final"].arrive()
                tp += 1
        while tp < total:
            yield from issue_pv(tp)
            if tp in ends:
                m.b["o_final"].arrive()
            tp += 1


def softmax_group(m, g):
    def copy_q(k):
        yield m.wait("q_full", k)
        m.b["q_tmem"].arrive(4)

    yield from copy_q(0)
    t0 = 0
    for k, n in enumerate(m.items):
        have_next = k + 1 < len(m.items)
        t = t0 + ((g - t0) & 1)
        while t < t0 + n:  # the group's tiles of the item
            j = t - t0
            yield m.wait(f"s_full{g}", t // 2)
            m.b[f"s_free{g}"].arrive(4)
            if j > 0:
                yield m.wait(f"xchg{g ^ 1}", (t - 1) // 2)
            m.b[f"xchg{g}"].arrive(4)
            if t > 0:
                yield m.wait(f"pv_done{(t - 1) & 1}", (t - 1) // 2)
            m.b[f"p_full{g}"].arrive(4)
            t += 2
        yield m.named_barrier("A", g, k)
        yield m.named_barrier("B", g, k)
        yield m.wait("o_final", k)
        if have_next:
            yield from copy_q(k + 1)
        if k > 0:
            yield m.wait("q_free", k - 1)
        m.b["o_staged"].arrive(4)
        yield m.named_barrier("C", g, k)
        t0 += n


def store_warp(m):
    for k in range(len(m.items)):
        yield m.wait("o_staged", k)
        m.b["q_free"].arrive()


def run(items, seed, order="per_item"):
    """Random interleaving of the roles; returns (finished, violations)."""
    m = Model(items)
    rng = random.Random(seed)
    roles = {"k": producer(m, True), "v": producer(m, False), "mma": mma(m, order),
             "g0": softmax_group(m, 0), "g1": softmax_group(m, 1), "store": store_warp(m)}
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


def random_items(rng):
    """A CTA's work items: KV tiles per item, long and short ones mixed (short ones stress the boundaries)."""
    return [rng.randint(1, 16) if rng.random() < 0.6 else rng.randint(1, 3) for _ in range(rng.randint(1, 8))]


def test_protocol_has_no_deadlock_and_no_ambiguous_parity_wait():
    rng = random.Random(2024)
    for trial in range(1500):
        items = random_items(rng)
        finished, violations = run(items, trial)
        assert finished, f"deadlock with items {items} (schedule seed {trial})"
        assert not violations, f"parity wait two phases behind with items {items}: {violations[:3]}"


@pytest.mark.parametrize("items", [[1], [16], [1, 1, 1, 1], [3, 1, 2, 16, 1], [16] * 4])
def test_protocol_corner_item_mixes(items):
    for seed in range(50):
        finished, violations = run(items, seed)
        assert finished and not violations


def test_model_catches_a_deadlocking_issue_order():
    """Negative control: the continuous S/PV stream without a flush deadlocks once a one-tile item follows."""
    rng = random.Random(7)
    deadlocks = sum(not run(random_items(rng), trial, order="stream")[0] for trial in range(300))
    assert deadlocks > 0
    assert not run([2, 1, 2], 0, order="stream")[0]
