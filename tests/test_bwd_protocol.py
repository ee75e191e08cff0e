"""A discrete-event model of the dK/dV backward kernel's barrier protocol, checked on the CPU.

attn_bwd_dkdv_kernel is persistent: a CTA walks several work items (key tiles), and its roles talk only through
mbarriers: the TMA producer of query tiles (Q, dO, LSE and Delta of every step through a 3-slot ring, running on
across items; an item's first two tiles go out as soon as their slots free, the later ones queue behind the
item's K and V loads), the K/V producer (each item's V once the last dP^T of the previous item is done, its K
once the last dQ^T is; then the previous item's dK and dV stores), the MMA warp (per item in the order A(0),
A(1), B(0), A(2), B(1), ..., B(n-1): A writes dP^T, then S^T into tensor-memory buffer gs % 2 of the running
step gs, B computes dQ^T, then dV and dK), and two softmax
groups that take the steps in turn (group g owns the steps gs = g mod 2 and buffer g) and after each item stage
its dV and dK in shared memory (the next item's first dV, dK MMAs wait until they have been read out of tensor
memory): the group of the item's last step stages dV in the dQ staging buffer (after its own last reduction
has read it), the other group dK in the two dS^T buffers. The K/V producer stores dK once it is staged
(dk_staged) and reports when the store has read the dS^T buffers (ds_read), then does the same for dV
(dv_staged, dq_read); each group waits for those reports before its first write to the same buffers in the next
item. The groups hand the 32 KB dQ staging buffer to each other in step order: a group's leader reports a
staged tile on dq_staged[gs % 2], the reduction warp issues the step's bulk reduction and reports its read on
stage_free[gs % 2]. Barrier counts follow the kernel: the softmax-side barriers count warps, and each group is
two actors -- the leader's warp, which also reports the staged tiles, and the other three warps, which can run
ahead of it. MMAs, commits and copies complete at once (timing does not matter for these properties). Over random item
mixes and interleavings the model checks that

  * every role runs to the end (no deadlock: a role only waits for something another role will still do),
  * no parity wait can be fooled: when a wait for phase n of a barrier succeeds, phase n + 1 has not completed
    yet (a parity wait only sees the current phase's parity, so a waiter two phases behind would hang or pass
    on the wrong phase), and
  * the staging buffer is never written (dQ of a step, or an item's dV) while a reduction is still reading it,
    and neither it nor a dS^T buffer is written while the previous item's dV, dK stores are reading them.

Negative controls must fail: a producer that refills ring slots without waiting for their release runs the
softmax groups' waits two phases behind; one stage barrier shared by both groups, with dV always staged by
group 0, lets a warp wait two phases ahead of it and stage over a tile being read; an epilogue that stages dV
without waiting for the item's last reductions does the same; a first step that does not wait for the previous
item's stores writes over them.
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
    def __init__(self, items, bug=None):
        self.items, self.bug = items, bug  # items: steps of each work item of the CTA
        self.b = {name: Barrier(1) for name in ("k_full", "v_full", "k_free", "v_free", "kv_issued", "stage_free0",
                                                 "stage_free1", "dq_staged0", "dq_staged1", "acc_done", "drain",
                                                 "ds_read", "dq_read")}
        self.b["acc_free"] = Barrier(8)
        self.b["dk_staged"] = Barrier(4)  # the four warps of the group that stages dK
        self.b["dv_staged"] = Barrier(4)
        for s in range(STAGES):
            self.b[f"q_full{s}"] = Barrier(1)
            self.b[f"q_empty{s}"] = Barrier(1)
        for r in range(2):
            for name, count in (("s_full", 1), ("p_full", 4), ("dq_full", 1), ("dq_empty", 4), ("b_done", 1)):
                self.b[f"{name}{r}"] = Barrier(count)
        self.named = {}  # named barrier instance -> actors that reached it
        self.single_done = 0  # completions of a single stage barrier for both groups (negative control)
        self.staged_reads_pending = set()  # steps whose dQ staging has been written but not yet read
        self.ds_reads_pending = set()      # items whose dK staging (the dS^T buffers) the stores have not read
        self.dq_reads_pending = set()      # items whose dV staging (the dQ staging buffer) they have not read
        self.violations = []

    def wait_single(self, n):
        """The parity wait of one stage barrier shared by both groups: it passes when the barrier's current
        phase has the other parity, also when it is two phases behind completion n."""
        return lambda: (self.single_done & 1) != (n & 1) or self.single_done > n

    def wait(self, name, n):
        """Wait for completion n (0-based) of a barrier: the kernel's parity wait on phase n."""
        bar = self.b[name]

        def ready():
            if bar.done > n + 1:
                self.violations.append((name, n, bar.done))
            return bar.done > n
        return ready


def producer(m):
    gs = 0
    for k, ns in enumerate(m.items):
        for i in range(ns):
            if i == (0 if k == 0 else min(2, ns - 1)):  # once per item: its later tiles queue behind its K and V
                yield m.wait("kv_issued", k)
            s = gs % STAGES
            if gs >= STAGES and m.bug != "no_ring_release_wait":
                yield m.wait(f"q_empty{s}", (gs - STAGES) // STAGES)
            m.b[f"q_full{s}"].arrive()
            gs += 1


def kv_producer(m):
    def store_epilogue(k):  # item k's dK store once dK is staged, then its dV store once dV is
        yield m.wait("dk_staged", k)
        m.ds_reads_pending.add(k)
        yield lambda: True
        m.ds_reads_pending.discard(k)  # the dK stores have read the dS^T buffers
        m.b["ds_read"].arrive()
        yield m.wait("dv_staged", k)
        m.dq_reads_pending.add(k)
        yield lambda: True
        m.dq_reads_pending.discard(k)  # the dV stores have read the dQ staging buffer
        m.b["dq_read"].arrive()

    for k, _ in enumerate(m.items):
        if k >= 1:
            yield m.wait("v_free", k - 1)
        m.b["v_full"].arrive()
        if k >= 1:
            yield m.wait("k_free", k - 1)
        m.b["k_full"].arrive()
        m.b["kv_issued"].arrive()
        if k >= 1:
            yield from store_epilogue(k - 1)
    yield from store_epilogue(len(m.items) - 1)


def mma(m):
    def issue_a(gs, first, k):
        s, rb = gs % STAGES, gs & 1
        yield m.wait(f"q_full{s}", gs // STAGES)
        if gs >= 2:
            yield m.wait(f"dq_empty{rb}", (gs - 2) >> 1)  # dP^T overwrites the dQ^T columns
        if first:
            yield m.wait("v_full", k)
        if gs >= 2:
            yield m.wait(f"b_done{rb}", (gs - 2) >> 1)    # S^T overwrites P^T, dS^T
        if first:
            yield m.wait("k_full", k)
        m.b[f"s_full{rb}"].arrive()

    def issue_b(gs, first, last, k):
        s, rb = gs % STAGES, gs & 1
        yield m.wait(f"p_full{rb}", gs >> 1)
        m.b[f"dq_full{rb}"].arrive()
        if last:
            m.b["k_free"].arrive()
        if first and k >= 1:
            yield m.wait("acc_free", k - 1)
        m.b[f"b_done{rb}"].arrive()
        m.b[f"q_empty{s}"].arrive()

    gs = 0
    for k, ns in enumerate(m.items):
        yield from issue_a(gs, True, k)
        for i in range(1, ns):
            yield from issue_a(gs + i, False, k)
            yield from issue_b(gs + i - 1, i == 1, False, k)
        m.b["v_free"].arrive()
        yield from issue_b(gs + ns - 1, ns == 1, True, k)
        m.b["acc_done"].arrive()
        gs += ns
    m.b["drain"].arrive()
    yield m.wait("drain", 0)


def named_barrier(m, key, actor, n_actors):
    m.named.setdefault(key, set()).add(actor)
    return lambda: len(m.named[key]) == n_actors


def softmax_warps(m, g, lead):
    """The warps of softmax group g: the group leader's warp (lead) or the other three. They run the same waits;
    the leader also reports each staged dQ tile to the reduction warp (dq_staged[g]) after the group's staging
    barrier, so the other warps can run ahead of it."""
    n = 1 if lead else 3
    actor = (g, lead)

    def wait_staged(step):
        return m.wait(f"stage_free{step & 1}", step >> 1)

    def wait_read(name, k):  # the previous item's dK (ds_read) or dV (dq_read) stores have read their staging
        if k >= 1 and m.bug != "no_epilogue_read_wait":
            yield m.wait(name, k - 1)

    gs0 = 0
    for k, ns in enumerate(m.items):
        first = True
        for gs in range(gs0 + ((g - gs0) & 1), gs0 + ns, 2):
            s, rb = gs % STAGES, g
            yield m.wait(f"q_full{s}", gs // STAGES)
            yield m.wait(f"s_full{rb}", gs >> 1)
            if first:
                yield from wait_read("ds_read", k)
            if m.ds_reads_pending:
                m.violations.append(("dS^T written over an unread dK staging", gs))
            m.b[f"p_full{rb}"].arrive(n)
            yield m.wait(f"dq_full{rb}", gs >> 1)
            m.b[f"dq_empty{rb}"].arrive(n)
            if gs > 0:
                if m.bug == "single_stage_barrier":  # one barrier for both groups, waited at its own parity
                    yield m.wait_single(gs - 1)
                else:
                    yield wait_staged(gs - 1)
            if first:
                yield from wait_read("dq_read", k)
                first = False
            if m.staged_reads_pending or m.dq_reads_pending:
                m.violations.append(("dQ staged over an unread tile", gs))
            yield named_barrier(m, ("stage", gs), actor, 2)
            if lead:
                m.staged_reads_pending.add(gs)  # staged; the reduction warp reads it
                m.b[f"dq_staged{g}"].arrive()
        # epilogue, after the item's last MMA: the group of the item's last step (late: its last reduction still
        # reads the dQ staging buffer) stages dV there, the other group stages dK in the two dS^T buffers
        yield m.wait("acc_done", k)
        gs_last = gs0 + ns - 1
        # (the negative control "single_stage_barrier" keeps the dV staging on group 0, where one stage barrier
        # for both groups is unsafe)
        dv_group = (g == 0) if m.bug == "single_stage_barrier" else (gs_last & 1) == g
        if dv_group and m.bug != "epilogue_skips_stage_wait":
            if m.bug == "single_stage_barrier":
                yield m.wait_single(gs_last)
            else:
                yield wait_staged(gs_last)
                if gs_last > 0:
                    yield wait_staged(gs_last - 1)
        yield from wait_read("dq_read" if dv_group else "ds_read", k)  # a group without a step here has not waited
        if dv_group and m.staged_reads_pending:
            m.violations.append(("dV staged over a dQ tile not yet read", k))
        if (dv_group and m.dq_reads_pending) or (not dv_group and m.ds_reads_pending):
            m.violations.append(("dV or dK staged over the previous item's unread staging", k))
        m.b["acc_free"].arrive(n)
        m.b["dv_staged" if dv_group else "dk_staged"].arrive(n)  # the K/V producer issues that store
        yield named_barrier(m, ("epilogue", k, g), actor, 2)  # the group leaves the item together
        gs0 += ns


def reducer(m):
    """The reduction warp: in step order, once a step's dQ tile is staged, one bulk reduction reads the staging
    buffer; then stage_free[gs % 2] hands the buffer on."""
    gs = 0
    for ns in m.items:
        for _ in range(ns):
            yield m.wait(f"dq_staged{gs & 1}", gs >> 1)
            yield lambda: True
            m.staged_reads_pending.discard(gs)  # the reduction has read the buffer
            m.b[f"stage_free{gs & 1}"].arrive()
            m.single_done += 1
            gs += 1


def run(items, seed, bug=None):
    """Random interleaving of the roles; returns (finished, violations)."""
    m = Model(items, bug)
    rng = random.Random(seed)
    roles = {"tma": producer(m), "kv": kv_producer(m), "mma": mma(m), "reduce": reducer(m)}
    for g in range(2):
        for lead in (True, False):
            roles[f"g{g}{'lead' if lead else 'rest'}"] = softmax_warps(m, g, lead)
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
    """A CTA's work items: steps per item, long and short ones mixed (one-step items stress the boundaries)."""
    return [rng.randint(1, 32) if rng.random() < 0.6 else rng.randint(1, 3) for _ in range(rng.randint(1, 6))]


def test_protocol_has_no_deadlock_and_no_ambiguous_parity_wait():
    """Item mixes of every shape the kernel meets: one-step items, odd step counts (a lone last A/B), the G * n
    steps of grouped-query heads, and long walks, several items per CTA."""
    rng = random.Random(99)
    for trial in range(1500):
        items = random_items(rng)
        finished, violations = run(items, trial)
        assert finished, f"deadlock with items {items} (schedule seed {trial})"
        assert not violations, f"parity wait two phases behind with items {items}: {violations[:3]}"


@pytest.mark.parametrize("items", [[1], [2], [3], [1, 1, 1], [32, 1, 2], [6, 7], [33, 32, 31]])
def test_protocol_corner_item_mixes(items):
    for seed in range(100):
        finished, violations = run(items, seed)
        assert finished and not violations


def test_model_catches_a_single_stage_barrier_race():
    """Negative control: with one stage barrier for both groups and dV always staged by group 0, a warp of group
    0 whose group did not run the item's last step can wait two phases ahead of it (its own leader's arrival
    still pending), pass at once and stage over a tile that is still being read."""
    rng = random.Random(11)
    caught = sum(bool(run(random_items(rng), seed, bug="single_stage_barrier")[1]) for seed in range(300))
    assert caught > 0


def test_model_catches_a_ring_overrun():
    """Negative control: without the wait for a slot's release the producer can complete a slot's phases two
    ahead of a softmax group's wait."""
    rng = random.Random(3)
    caught = sum(bool(run(random_items(rng), seed, bug="no_ring_release_wait")[1]) for seed in range(200))
    assert caught > 0


def test_model_catches_an_epilogue_overwriting_the_last_dq_tile():
    """Negative control: group 0's dV staging without the wait for the item's last bulk reduction can overwrite
    a dQ tile that the other group's reduction has not read yet."""
    rng = random.Random(5)
    caught = sum(bool(run(random_items(rng), seed, bug="epilogue_skips_stage_wait")[1]) for seed in range(200))
    assert caught > 0


def test_model_catches_a_step_writing_over_the_previous_items_stores():
    """Negative control: a group whose first step of an item does not wait for the previous item's dV, dK stores
    to have read their staging writes dS^T (or stages dQ) over it."""
    rng = random.Random(7)
    caught = sum(bool(run(random_items(rng), seed, bug="no_epilogue_read_wait")[1]) for seed in range(300))
    assert caught > 0
