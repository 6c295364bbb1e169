"""CPU model of the tensor-core heatmap kernel's mbarrier protocol (no GPU).

The kernel in csrc/heatmap_tc.cu runs six roles per CTA over the work units
it is given (one unit = 128 output pixels of one crop):

  scheduler          takes units from the hardware's CTA queue, drops those
                     of crops with no valid row, and publishes the others into
                     a ring of U slots: waits uempty[slot] before reusing a
                     slot (from the (U+1)-th unit on), fills it, arrives on
                     ufull[slot]; a stop marker follows the last unit;
  every other warp   per unit waits ufull[slot], reads the slot, arrives once
                     on uempty[slot] (also for the stop marker), then:

  feature-slab TMA   waits sempty[s] to reuse slab slot s, arms sfull[s] with
                     the slab's bytes (one arrival plus transaction bytes);
  kernel-row TMA     waits empty[s] to reuse stage s, arms bfull[s] with the
                     kernel rows' bytes; at exit waits bfull[] of its last
                     stages (its own copies only);
  MMA (one thread)   per unit waits accempty[buf] before reusing accumulator
                     buf (from the third unit on); per stage waits bfull[s]
                     and ready[s], issues, and commits to empty[s]; at the
                     unit's end commits to accfull[buf]; finally commits to
                     drain;
  epilogue warps     per unit wait accfull[buf], then each arrives once on
                     accempty[buf];
  producer warps     in G groups of P warps; group g takes every stage i with
                     i % G == g: waits sfull[slab slot] and (from the fourth
                     stage on) empty[s], then each warp of the group arrives
                     once on sempty[slab slot] and ready[s].

Barrier counts: ufull 1, uempty = every warp but the scheduler, sfull 1,
sempty = P, bfull 1, ready = P, empty 1, accfull 1, accempty = epilogue warps,
drain 1. Ring depths: 8 unit slots, 6 slab slots, 3 stages, 2 accumulators.

Hardware semantics modelled: a phase completes when its pending arrival count
and its pending transaction bytes both reach zero; a parity wait on P
succeeds iff the completed-phase count's parity differs from P; transaction
bytes land asynchronously in any order; a commit arrives once every earlier
MMA of its thread is done, i.e. commits are delivered in issue order.

Checked under random schedules (each role given a random speed per run): every successful wait sees exactly the phase
it means (a parity wait cannot tell phase k from k + 2), every arrival lands
in the phase it is meant for (none counts toward an earlier one), nothing
over-arrives, the drains end, and no configuration deadlocks.
"""
import random

import pytest

SLAB, STAGES, UNIT_SLOTS = 6, 3, 8


class Bar:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.completed = count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def arrive(self, phase, who):
        assert self.completed == phase, f"{who}: arrival for phase {phase} on {self.name} in phase {self.completed}"
        self.pending -= 1
        assert self.pending >= 0, f"{who}: over-arrival on {self.name}"
        self._maybe_complete()

    def expect_tx(self, phase, who):
        assert self.completed == phase, f"{who}: tx armed for phase {phase} on {self.name} in phase {self.completed}"
        self.tx += 1

    def land_tx(self):
        assert self.tx > 0
        self.tx -= 1
        self._maybe_complete()


def simulate(units, nchunks, nprod, nepi, seed, async_bias, bad_reuse_parity=False, skip_acc_wait=False,
             check_waits=True, groups=1, skip_slot_wait=False):
    """units: valid-row counts per unit of this CTA (0 = skipped). Returns the
    number of stages run; raises AssertionError on a protocol violation.
    `bad_reuse_parity` plants a wrong parity in the producers' reuse wait;
    `skip_acc_wait` drops the MMA's wait for a drained accumulator. With
    `check_waits` False only the data-hazard checks at each access run.
    `nprod` counts the warps of one producer group; `groups` groups take the
    stages in turn. `skip_slot_wait` drops the scheduler's wait for a read
    unit slot."""
    rnd = random.Random(seed)
    bars = {}

    def bar(name, count):
        bars[name] = Bar(name, count)

    for s in range(SLAB):
        bar(("sfull", s), 1)
        bar(("sempty", s), nprod)
    for s in range(STAGES):
        bar(("bfull", s), 1)
        bar(("ready", s), nprod)
        bar(("empty", s), 1)
    for t in range(2):
        bar(("accfull", t), 1)
        bar(("accempty", t), nepi)
    bar(("drain",), 1)
    nreaders = 3 + nepi + groups * nprod
    for s in range(UNIT_SLOTS):
        bar(("ufull", s), 1)
        bar(("uempty", s), nreaders)
    live = [n for n in units if n > 0]
    stages = len(live) * nchunks
    tx_in_flight = []          # barriers with transaction bytes still landing
    commits = []               # commit targets in issue order: (barrier, phase)

    # each role yields ("wait", bar, parity, expected_completed) | ("arrive", bar, phase)
    #                 | ("tx", bar, phase) | ("commit", bar, phase)
    #                 | ("access", bar, phases_needed, what): a read or overwrite of the
    #                   buffer that `bar` guards, legal once `bar` has completed that many phases
    def scheduler():
        for v in range(len(live) + 1):                            # the units, then the stop marker
            s, k = v % UNIT_SLOTS, v // UNIT_SLOTS
            if v >= UNIT_SLOTS:
                if not skip_slot_wait:
                    yield ("wait", ("uempty", s), (k - 1) & 1, k)
                yield ("access", ("uempty", s), k, "unit slot overwritten before every warp read it")
            yield ("arrive", ("ufull", s), k)

    def take_unit(v):
        s, k = v % UNIT_SLOTS, v // UNIT_SLOTS
        yield ("wait", ("ufull", s), k & 1, k + 1)
        yield ("access", ("ufull", s), k + 1, "unit slot read before it was published")
        yield ("arrive", ("uempty", s), k)

    def tma_slab():
        it = 0
        for v in range(len(live) + 1):
            yield from take_unit(v)
            if v == len(live):
                break
            for _ in range(nchunks):
                s, k = it % SLAB, it // SLAB
                if it >= SLAB:
                    yield ("wait", ("sempty", s), (k - 1) & 1, k)
                    yield ("access", ("sempty", s), k, "slab slot overwritten before the producers read it")
                yield ("tx", ("sfull", s), k)
                it += 1
        for last in range(max(0, stages - SLAB), stages):          # drain
            yield ("wait", ("sfull", last % SLAB), (last // SLAB) & 1, last // SLAB + 1)

    def tma_rows():
        it = 0
        for v in range(len(live) + 1):
            yield from take_unit(v)
            if v == len(live):
                break
            for _ in range(nchunks):
                s, k = it % STAGES, it // STAGES
                if it >= STAGES:
                    yield ("wait", ("empty", s), (k - 1) & 1, k)
                    yield ("access", ("empty", s), k, "kernel rows overwritten before the MMA read them")
                yield ("tx", ("bfull", s), k)
                it += 1
        for last in range(max(0, stages - STAGES), stages):        # drain
            yield ("wait", ("bfull", last % STAGES), (last // STAGES) & 1, last // STAGES + 1)

    def mma():
        it = 0
        for v in range(len(live) + 1):
            yield from take_unit(v)
            if v == len(live):
                break
            buf, use = v & 1, v >> 1
            if v >= 2 and not skip_acc_wait:
                yield ("wait", ("accempty", buf), (use - 1) & 1, use)
            if v >= 2:
                yield ("access", ("accempty", buf), use, "accumulator overwritten before the epilogue drained it")
            for _ in range(nchunks):
                s, k = it % STAGES, it // STAGES
                yield ("wait", ("bfull", s), k & 1, k + 1)
                yield ("access", ("bfull", s), k + 1, "kernel rows read before they landed")
                yield ("wait", ("ready", s), k & 1, k + 1)
                yield ("access", ("ready", s), k + 1, "stage read before its A operand was written")
                yield ("commit", ("empty", s), k)
                it += 1
            yield ("commit", ("accfull", buf), use)
        if it > 0:
            yield ("commit", ("drain",), 0)
            yield ("wait", ("drain",), 0, 1)

    def epilogue():
        for v in range(len(live) + 1):
            yield from take_unit(v)
            if v == len(live):
                break
            buf, use = v & 1, v >> 1
            yield ("wait", ("accfull", buf), use & 1, use + 1)
            yield ("access", ("accfull", buf), use + 1, "accumulator read before its MMAs completed")
            yield ("arrive", ("accempty", buf), use)

    def producer(g):
        for v in range(len(live) + 1):
            yield from take_unit(v)
            if v == len(live):
                break
            yield from produce(g, range(v * nchunks, (v + 1) * nchunks))

    def produce(g, its):
        for it in its:
            if it % groups != g:
                continue
            ss, ks = it % SLAB, it // SLAB
            s, k = it % STAGES, it // STAGES
            yield ("wait", ("sfull", ss), ks & 1, ks + 1)
            yield ("access", ("sfull", ss), ks + 1, "slab read before its bytes landed")
            if it >= STAGES:
                yield ("wait", ("empty", s), (k & 1) if bad_reuse_parity else ((k - 1) & 1), k)
                yield ("access", ("empty", s), k, "A stage overwritten before the MMA read it")
            yield ("arrive", ("sempty", ss), ks)
            yield ("arrive", ("ready", s), k)

    roles = {"scheduler": scheduler(), "tma_slab": tma_slab(), "tma_rows": tma_rows(), "mma": mma()}
    roles.update({f"epi{i}": epilogue() for i in range(nepi)})
    roles.update({f"prod{g}.{i}": producer(g) for g in range(groups) for i in range(nprod)})
    cur = {name: next(g, None) for name, g in roles.items()}
    # per-run role speeds, so that skewed interleavings (a slow epilogue, a fast
    # issuer) are explored too, not only evenly mixed ones
    speed = {name: rnd.choice([0.02, 1.0, 50.0]) for name in roles}

    while True:
        runnable = [n for n, op in cur.items()
                    if op is not None and (op[0] != "wait" or (bars[op[1]].completed & 1) != op[2])]
        pending = len(tx_in_flight) + (1 if commits else 0)
        if not runnable and not pending:
            break
        if pending and (not runnable or rnd.random() < async_bias):
            pick = rnd.randrange(pending)
            if pick < len(tx_in_flight):
                bars[tx_in_flight.pop(pick)].land_tx()
            else:
                target, phase = commits.pop(0)        # commits complete in issue order
                bars[target].arrive(phase, "commit")
            continue
        name = rnd.choices(runnable, weights=[speed[n] for n in runnable])[0]
        op = cur[name]
        if op[0] == "wait":
            got = bars[op[1]].completed
            if check_waits:
                assert got == op[3], f"{name}: wait on {op[1]} passed with {got} phases done, meant {op[3]}"
        elif op[0] == "access":
            got = bars[op[1]].completed
            assert got >= op[2], f"{name}: {op[3]} ({op[1]}: {got} phases done, needs {op[2]})"
        elif op[0] == "arrive":
            bars[op[1]].arrive(op[2], name)
        elif op[0] == "tx":
            b = bars[op[1]]
            b.expect_tx(op[2], name)
            b.arrive(op[2], name)                     # arrive.expect_tx: one arrival plus the bytes
            tx_in_flight.append(op[1])
        elif op[0] == "commit":
            commits.append((op[1], op[2]))
        cur[name] = next(roles[name], None)

    stuck = {n: op for n, op in cur.items() if op is not None}
    assert not stuck, f"deadlock: {stuck}"
    return stages


@pytest.mark.parametrize("async_bias", [0.05, 0.3, 0.8])
def test_protocol_random_schedules(async_bias):
    rnd = random.Random(int(async_bias * 1000))
    total = 0
    for trial in range(120):
        units = [rnd.choice([0, 16, 48, 96, 160]) for _ in range(rnd.randint(0, 9))]
        total += simulate(units, rnd.randint(1, 9), nprod=rnd.randint(1, 3), nepi=rnd.randint(1, 2),
                          seed=trial, async_bias=async_bias, groups=rnd.choice([1, 2, 3]))
    assert total > 0


def test_protocol_with_the_kernels_warp_counts():
    # 4 producer groups of 4 warps and 4 epilogue warps, as launched; long unit
    # runs wrap every ring many times (6 slab slots, 3 stages, 2 accumulators),
    # and unit lengths that are not multiples of the group count rotate which
    # group starts each unit
    for trial in range(6):
        units = [0, 96, 160, 0, 48, 16, 96, 96, 160, 32]
        simulate(units, 8, nprod=4, nepi=4, seed=trial, async_bias=0.3, groups=3)
        simulate(units, 4, nprod=4, nepi=4, seed=trial, async_bias=0.3, groups=3)
        simulate(units, 10, nprod=4, nepi=4, seed=trial, async_bias=0.3, groups=3)
        # two epilogue sets (8 warps) with 3 or 2 producer groups
        simulate(units, 8, nprod=4, nepi=8, seed=trial, async_bias=0.3, groups=3)
        simulate(units, 8, nprod=4, nepi=8, seed=trial, async_bias=0.3, groups=2)


def test_model_catches_four_producer_groups():
    """Four groups over three A slots: a group that last built stage i - 4 can
    find empty[i % 3] two phases short of the one it needs, and a parity wait
    cannot tell those apart. The model reports it (this is why the kernel runs
    three groups)."""
    failures = 0
    for trial in range(20):
        try:
            simulate([96, 48, 160, 16, 96], 8, nprod=2, nepi=1, seed=trial, async_bias=0.3, groups=4)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_model_catches_a_wrong_reuse_parity():
    """The check has teeth: producers that wait on empty[s] with the parity of
    the phase they are about to need, instead of the previous use's, pass on a
    phase that has not completed, and the model reports it."""
    for trial in range(20):
        with pytest.raises(AssertionError):
            simulate([96, 48, 160, 16], 6, nprod=2, nepi=1, seed=trial, async_bias=0.3,
                     bad_reuse_parity=True, groups=1 + trial % 4)


def test_model_catches_a_missing_accumulator_wait():
    """Without the MMA's wait on accempty it starts a third unit in an
    accumulator the epilogue may not have drained: the access check reports the
    overwrite on some schedule even with the phase-accounting checks off."""
    failures = 0
    for trial in range(30):
        try:
            simulate([96, 96, 96, 96, 96], 2, nprod=1, nepi=1, seed=trial, async_bias=0.3, skip_acc_wait=True,
                     check_waits=False)
        except AssertionError as e:
            assert "accumulator overwritten" in str(e) or "deadlock" in str(e), str(e)
            failures += 1
    assert failures > 0


def test_access_checks_alone_catch_a_wrong_reuse_parity():
    failures = 0
    for trial in range(20):
        try:
            simulate([96, 48, 160, 16], 6, nprod=2, nepi=1, seed=trial, async_bias=0.3, bad_reuse_parity=True,
                     check_waits=False)
        except AssertionError as e:
            assert "overwritten" in str(e) or "deadlock" in str(e) or "phase" in str(e), str(e)
            failures += 1
    assert failures > 0


def test_model_catches_a_missing_unit_slot_wait():
    """A scheduler that refills a unit slot without waiting for every other
    warp to have read it overwrites a unit some warp has not taken yet: the
    access check reports it on some schedule (with more units than slots)."""
    failures = 0
    for trial in range(30):
        try:
            simulate([96, 16, 48] * 5, 1, nprod=1, nepi=1, seed=trial, async_bias=0.3, skip_slot_wait=True,
                     check_waits=False, groups=2)
        except AssertionError as e:
            assert "unit slot" in str(e) or "deadlock" in str(e), str(e)
            failures += 1
    assert failures > 0


def _epilogue_set_decisions(seed, agree):
    """Four epilogue warps of a set wait on accfull with a bounded wait that
    tests the phase first and, while it is incomplete, gives up once the abort
    flag is set. The MMA's commit and another role's abort land at random times,
    and the warps reach their wait at random times. A warp that arrives after
    the commit succeeds; one that arrives before it succeeds only if the commit
    comes before the abort. With `agree` the set takes one decision (the AND
    over its warps, as bar.red.and gives); without it each warp acts alone."""
    rnd = random.Random(seed)
    commit_at, abort_at = rnd.randint(0, 9), rnd.randint(0, 9)
    starts = [rnd.randint(0, 9) for _ in range(4)]
    own = [t >= commit_at or commit_at <= abort_at for t in starts]
    return [all(own)] * 4 if agree else own


def test_epilogue_set_takes_one_decision_on_abort():
    """The kernel's epilogue warps meet at named barriers after the accumulator
    wait, so every warp of a set must take the same path when an abort lands as
    the commit completes; the AND-reduced decision guarantees it, per-warp
    decisions do not (on some schedule a warp would wait at a barrier the others
    skipped)."""
    split = 0
    for seed in range(400):
        assert len(set(_epilogue_set_decisions(seed, agree=True))) == 1
        split += len(set(_epilogue_set_decisions(seed, agree=False))) > 1
    assert split > 0
