"""A discrete-event model of the persistent forward kernel's barrier protocol, checked on the CPU.

attn_fwd_kernel runs as CTA pairs whose roles talk only through mbarriers (and, between the two softmax groups
of a CTA, three named barriers per work item). This model replays each role's waits and arrivals in the
kernel's order -- in each CTA the K and V producers with the one Q buffer, the two softmax groups with their
epilogue and the output-store warp; in the even CTA the MMA warp -- with barrier counts as in the kernel
(softmax-side barriers count warps: a group of four warps is one actor arriving 4; the pair barriers of the even
CTA count the arrivals of both CTAs; a multicast commit arrives once in each CTA). Loads and MMAs complete at once (timing does not matter for these properties). Over random
work-item mixes and random interleavings it checks that

  * every role runs to the end (no deadlock: a role only waits for something another role will still do), and
  * no parity wait can be fooled: when a wait for phase n of a barrier succeeds, phase n + 1 has not completed
    yet (a parity wait only sees the current phase's parity, so a waiter two phases behind would hang).

The group without an item's last tile copies the next item's Q into tensor memory as soon as the item's last S
MMA has completed (s_done), so the next item's first S tiles queue right behind the item's last PV; the model
also checks that the epilogue never stages the output over a Q that has not been copied yet. Negative controls:
an MMA issue order tried during development (the S tiles of item k+2 before the last PVs of item k) must
deadlock, and a Q copy that does not wait for s_done must be caught.
"""
import random

import pytest

STAGES = 4  # K and V ring depth


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self, n=1):
        self.pending += n
        assert self.pending <= self.count, "more arrivals than the phase expects"
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


class Model:
    """Barriers of both CTAs of a pair. Local and multicast-completed barriers exist once per CTA (suffix r);
    the pair barriers live in the even CTA. A K or V ring slot's pair barrier completes after the even CTA's
    arming arrival and the two halves' copy completions (modelled as three arrivals, in any order)."""

    def __init__(self, items):
        self.items = items
        self.b = {"q_ready": Barrier(8)}
        for r in range(2):
            for name, count in [("q_full", 1), ("q_tmem", 4), ("q_free", 1), ("o_staged", 8), ("o_final", 1),
                                ("s_done", 1)]:
                self.b[f"{name}{r}"] = Barrier(count)
            for s in range(STAGES):
                for name in ("k_empty", "v_empty"):
                    self.b[f"{name}{s}_{r}"] = Barrier(1)
            for s in range(2):
                for name, count in (("s_full", 1), ("xchg", 4), ("pv_done", 1)):
                    self.b[f"{name}{s}_{r}"] = Barrier(count)
        for s in range(STAGES):
            for name in ("k_full", "v_full"):
                self.b[f"{name}{s}"] = Barrier(3)
        for s in range(2):
            for name in ("s_free", "p_full"):
                self.b[f"{name}{s}"] = Barrier(8)
        self.named = {(w, r): [0, 0] for w in "ABC" for r in range(2)}  # passes of each named barrier, per group
        self.q_copied = [-1, -1]  # per CTA: the last item whose Q is in tensor memory
        self.violations = []

    def wait(self, name, n):
        """Wait for completion n (0-based) of a barrier: the kernel's parity wait on phase n."""
        bar = self.b[name]

        def ready():
            if bar.done > n + 1:
                self.violations.append((name, n, bar.done))
            return bar.done > n
        return ready

    def both(self, name):
        """A multicast commit: one arrival on the barrier at the same offset in each CTA."""
        for r in range(2):
            self.b[f"{name}_{r}" if name[-1].isdigit() else f"{name}{r}"].arrive()

    def named_barrier(self, which, r, g, k):
        self.named[(which, r)][g] += 1
        return lambda: min(self.named[(which, r)]) > k


def producer(m, r, is_k):
    t0 = 0
    for k, n in enumerate(m.items):
        if is_k:  # one Q buffer per CTA, shared with the output staging of item k-2
            if k == 1:
                yield m.wait(f"q_tmem{r}", 0)
            if k >= 2:
                yield m.wait(f"q_free{r}", k - 2)
            m.b[f"q_full{r}"].arrive()
        for j in range(n):
            t = t0 + j
            s = t % STAGES
            if t >= STAGES:
                yield m.wait(("k_empty" if is_k else "v_empty") + f"{s}_{r}", (t - STAGES) // STAGES)
            full = m.b[("k_full" if is_k else "v_full") + str(s)]
            if r == 0:
                full.arrive()  # arm the pair barrier with both halves' bytes
            full.arrive()      # this CTA's half landed
        t0 += n


def mma(m, order="dynamic"):
    def ready(name, n):
        bar = m.b[name]
        if bar.done > n + 1:
            m.violations.append((name, n, bar.done))
        return bar.done > n

    def s_ready(t):
        return (t < 2 or ready(f"s_free{t & 1}", (t - 2) // 2)) and ready(f"k_full{t % STAGES}", t // STAGES)

    def pv_ready(t):
        return ready(f"p_full{t & 1}", t // 2) and ready(f"v_full{t % STAGES}", t // STAGES)

    def issue_s(t):
        m.both(f"s_full{t & 1}")
        m.both(f"k_empty{t % STAGES}")

    def issue_pv(t):
        m.both(f"pv_done{t & 1}")
        m.both(f"v_empty{t % STAGES}")

    if order == "dynamic":  # the kernel: per item, whichever of PV(jp), S(js) is ready (PV first), then o_final
        t0 = 0
        for k, n in enumerate(m.items):
            yield m.wait("q_ready", k)
            js = jp = 0
            while jp < n:
                yield lambda: (js < n and s_ready(t0 + js)) or (jp < js and pv_ready(t0 + jp))
                if jp < js and pv_ready(t0 + jp):
                    issue_pv(t0 + jp)
                    jp += 1
                else:
                    issue_s(t0 + js)
                    js += 1
                    if js == n:
                        m.both("s_done")  # the item's Q in tensor memory is no longer read
            m.both("o_final")
            t0 += n
    else:  # negative control: one stream over all items, PVs two tiles behind, no flush at item starts
        starts = [sum(m.items[:k]) for k in range(len(m.items))]
        ends = {starts[k] + n - 1 for k, n in enumerate(m.items)}
        total = sum(m.items)
        tp = 0
        for ts in range(total):
            if ts in starts:
                yield m.wait("q_ready", starts.index(ts))
            yield lambda: s_ready(ts)
            issue_s(ts)
            if ts + 1 - tp >= 3:
                yield lambda: pv_ready(tp)
                issue_pv(tp)
                if tp in ends:
                    m.both("o_final")
                tp += 1
        while tp < total:
            yield lambda: pv_ready(tp)
            issue_pv(tp)
            if tp in ends:
                m.both("o_final")
            tp += 1


def softmax_group(m, r, g, bug=None):
    def copy_q(k):  # one group copies both head-dim halves of the item's Q into this CTA's tensor memory
        yield m.wait(f"q_full{r}", k)
        m.q_copied[r] = k
        m.b[f"q_tmem{r}"].arrive(4)
        m.b["q_ready"].arrive(4)

    if g == 0:
        yield from copy_q(0)
    t0 = 0
    for k, n in enumerate(m.items):
        have_next = k + 1 < len(m.items)
        t = t0 + ((g - t0) & 1)
        while t < t0 + n:  # the group's tiles of the item (a tile above the diagonal takes the same steps)
            j = t - t0
            yield m.wait(f"s_full{g}_{r}", t // 2)
            m.b[f"s_free{g}"].arrive(4)
            if j > 0:
                yield m.wait(f"xchg{g ^ 1}_{r}", (t - 1) // 2)
            m.b[f"xchg{g}_{r}"].arrive(4)
            if t > 0:
                yield m.wait(f"pv_done{(t - 1) & 1}_{r}", (t - 1) // 2)
            m.b[f"p_full{g}"].arrive(4)
            t += 2
        # the group without the item's last tile copies the next item's Q once the item's last S has completed
        if have_next and g == ((t0 + n - 1) & 1) ^ 1:
            if bug != "copy_before_last_s":
                yield m.wait(f"s_done{r}", k)
            elif m.b[f"s_done{r}"].done <= k:
                m.violations.append(("next Q copied over a Q still read by this item's S", k))
            yield from copy_q(k + 1)
        yield m.named_barrier("A", r, g, k)
        yield m.named_barrier("B", r, g, k)
        yield m.wait(f"o_final{r}", k)
        if k > 0:
            yield m.wait(f"q_free{r}", k - 1)
        if have_next and m.q_copied[r] < k + 1:  # the staging below overwrites the Q buffer
            m.violations.append(("output staged over a Q not yet copied", k))
        m.b[f"o_staged{r}"].arrive(4)
        yield m.named_barrier("C", r, g, k)
        t0 += n


def store_warp(m, r):
    for k in range(len(m.items)):
        yield m.wait(f"o_staged{r}", k)
        m.b[f"q_free{r}"].arrive()


def run(items, seed, order="dynamic", bug=None):
    """Random interleaving of the roles of both CTAs; returns (finished, violations)."""
    m = Model(items)
    rng = random.Random(seed)
    roles = {"mma": mma(m, order)}
    for r in range(2):
        roles.update({f"k{r}": producer(m, r, True), f"v{r}": producer(m, r, False),
                      f"g0_{r}": softmax_group(m, r, 0, bug), f"g1_{r}": softmax_group(m, r, 1, bug),
                      f"store{r}": store_warp(m, r)})
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


def test_model_catches_a_q_copy_that_does_not_wait_for_the_last_s():
    """Negative control: copying the next item's Q without waiting for the item's last S MMA can overwrite a Q
    that an S MMA still reads."""
    rng = random.Random(9)
    caught = sum(bool(run(random_items(rng), trial, bug="copy_before_last_s")[1]) for trial in range(300))
    assert caught > 0
