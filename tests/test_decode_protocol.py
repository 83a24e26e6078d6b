"""Model check, on the CPU, of the mbarrier and cross-CTA protocols of the tensor-core decode
kernels: the fused block-scaled decode (`decode_mx_fused_kernel`, csrc/decode_mx_mma.cu), its
two-launch form, and the BF16 tensor-core decode (`decode_mma_kernel`, csrc/decode_mma.cu).

Each role of the CTA -- TMA producer, MMA issuer, scale copier, atom builders, epilogue -- is a
sequence of steps written from the kernel: waits (mbarrier parity waits with the hardware's
semantics: waiting on parity P passes once the barrier's completed-phase count has parity
other than P), plain arrivals, and asynchronous commits (tcgen05.commit) that complete later
but in issue order per issuing thread.  Random interleavings of the roles are run for many item
sequences (gate/up items, then down items of one or more groups), and the checker asserts:

* every schedule finishes (no deadlock);
* no wait is ever satisfied by a phase other than the one it means (a barrier never runs two
  phases ahead of a waiter, which a parity wait could not tell apart);
* no buffer -- ring stage, scale-atom region in shared memory, weight / activation scale columns
  and accumulators in TMEM -- is written while a reader may still use it (write after read);
* every reader finds the data of the item it is for (read after write).

The two-launch form (`decode_mx_mma_kernel<0/1>`) is checked the same way at each of its buffer
plans.  Planted mistakes (one wait dropped from one role) must each be caught.  The single-CTA
checks take every group's h as written; a multi-CTA check runs whole launches with the
cross-CTA counters (waits for all of a group's gate/up epilogues, two counted reads per down
item, reset by the last).
"""
import random

import pytest

ST = 4  # ring stages


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.done = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending, self.done = 0, self.done + 1


class Violation(AssertionError):
    pass


class Regions:
    """Live readers and current contents of every buffer region."""

    def __init__(self):
        self.readers, self.content = {}, {}

    def write(self, r, who):
        if self.readers.get(r):
            raise Violation(f"{who} writes {r} while {sorted(self.readers[r])} may still read it")

    def fill(self, r, tag):
        self.content[r] = tag

    def read(self, r, tag, want):
        if self.content.get(r) != want:
            raise Violation(f"{tag} reads {r} holding {self.content.get(r)}, expected {want}")
        self.readers.setdefault(r, set()).add(tag)

    def done(self, r, tag):
        self.readers.setdefault(r, set()).discard(tag)


class Groups:
    """The cross-CTA counters of a launch: per group, the gate/up epilogue arrivals (ready once
    all of the group's gate/up items have written their h planes) and the reads of down items
    (two per down item: its producer after the wait, its copier once the item's atoms exist);
    the last read resets both."""

    def __init__(self, n_groups, gu_blocks, dn_blocks):
        self.h, self.reads = [0] * n_groups, [0] * n_groups
        self.gu, self.dn = gu_blocks, dn_blocks

    def ready(self, g):
        return self.h[g] >= self.gu

    def h_done(self, g):
        self.h[g] += 1

    def read_done(self, g):
        if not self.ready(g):
            raise Violation(f"a read of group {g} counted before all its h was written")
        self.reads[g] += 1
        if self.reads[g] == 2 * self.dn:
            self.h[g], self.reads[g] = 0, 0


def build_protocol(items, nk, drop=None, glob=None):
    """Roles of one CTA for `items` = [(down, group)] (its items in order) and nk(down) = the
    item's 256-deep stages.  drop = (role, barrier name): leave that role's waits on that barrier
    out (a planted mistake).  glob: the launch's Groups when several CTAs are modelled (without
    it every group's h counts as written).  Returns (roles, barriers, regions)."""
    n = len(items)
    keys = [(g if d else -1) for d, g in items]
    act_new = [j == 0 or keys[j] != keys[j - 1] for j in range(n)]
    first_down = [items[j][0] and j > 0 and not items[j - 1][0] for j in range(n)]
    drun, r = [], -1
    for j in range(n):
        if items[j][0] and act_new[j]:
            r += 1
        drun.append(r)
    act_of = [None] * n                       # the item whose activation atoms item j reads
    for j in range(n):
        act_of[j] = j if act_new[j] else act_of[j - 1]

    bars = {}
    for s in range(ST):
        bars[("full", s)] = Bar(1)
        bars[("empty", s)] = Bar(1)
    for b in range(2):
        bars[("tfull", b)] = Bar(1)
        bars[("tempty", b)] = Bar(1)          # four epilogue warps, modelled as one arrival
        bars[("atoms_full", b)] = Bar(1)      # four builder warps, modelled as one arrival
        bars[("atoms_free", b)] = Bar(1)
        bars[("sf_ready", b)] = Bar(1)
    R = Regions()

    # The kernel's layout as sub-regions.  Shared memory: weight-atom buffers b at b x 16 KB, a
    # lower and an upper 8 KB half each (down items, K <= 2048, fill the lower half; gate/up
    # items both); the x atoms take buffer 1's place; the down activation atoms the upper half of
    # buffer 0.  TMEM: the x scale columns span both down activation-scale buffers; the weight-
    # scale buffers and the accumulators lie apart.
    def smem_w(j):
        b = j & 1
        return [("smem", b, "lo")] if items[j][0] else [("smem", b, "lo"), ("smem", b, "hi")]

    def smem_act(j):
        return [("smem", 0, "hi")] if items[j][0] else [("smem", 1, "lo"), ("smem", 1, "hi")]

    def tmem_act(j):
        return [("tmem_act", drun[j] & 1)] if items[j][0] else [("tmem_act", 0), ("tmem_act", 1)]

    def W(role, bar, parity, means):
        return None if drop == (role, bar[0]) else ("wait", bar, parity, means)

    def A(bar):
        return ("arrive", bar)

    def F(fn):
        return ("fn", fn)

    def producer():
        step = 0
        for j in range(n):
            if glob and items[j][0]:
                g = items[j][1]
                if drop != ("producer", "group"):
                    yield ("spin", lambda g=g: glob.ready(g))
                yield F(lambda g=g: glob.read_done(g))
            for kb in range(nk(items[j][0])):
                s, ph = step % ST, (step // ST) & 1
                yield W("producer", ("empty", s), ph ^ 1, step // ST - 1)
                yield F(lambda s=s, j=j: R.write(("stage", s), f"TMA of item {j}"))
                yield F(lambda s=s, j=j, kb=kb: R.fill(("stage", s), (j, kb)))
                yield A(("full", s))
                step += 1

    def mma():
        step = 0
        for j in range(n):
            b = j & 1
            yield W("mma", ("sf_ready", b), (j >> 1) & 1, j >> 1)
            yield W("mma", ("tempty", b), ((j >> 1) & 1) ^ 1, (j >> 1) - 1)
            yield F(lambda j=j, b=b: R.write(("acc", b), f"MMAs of item {j}"))
            yield F(lambda j=j, b=b: R.read(("tmem_w", b), ("mma", j), j))
            for t in tmem_act(j):
                yield F(lambda t=t, j=j: R.read(t, ("mma", j), act_of[j]))
            for kb in range(nk(items[j][0])):
                s, ph = step % ST, (step // ST) & 1
                yield W("mma", ("full", s), ph, step // ST)
                yield F(lambda s=s, j=j, kb=kb: R.read(("stage", s), ("mma", j, kb), (j, kb)))
                # the stage is released once the MMAs that read it completed
                yield ("commit", "mma", [F(lambda s=s, j=j, kb=kb: R.done(("stage", s), ("mma", j, kb))),
                                         A(("empty", s))])
                step += 1
            # the finished accumulator has a reader, the epilogue, until it hands the buffer back
            yield ("commit", "mma", [F(lambda j=j, b=b: [R.done(t, ("mma", j)) for t in [("tmem_w", b)] + tmem_act(j)]),
                                     F(lambda j=j, b=b: R.fill(("acc", b), j)),
                                     F(lambda j=j, b=b: R.readers.setdefault(("acc", b), set()).add(("epi", j))),
                                     A(("tfull", b))])

    def copier():
        for j in range(n):
            b = j & 1
            yield W("copier", ("atoms_full", b), (j >> 1) & 1, j >> 1)
            if glob and items[j][0]:
                yield F(lambda g=items[j][1]: glob.read_done(g))
            if j >= 2:
                yield W("copier", ("tfull", b), ((j - 2) >> 1) & 1, (j - 2) >> 1)
            if first_down[j]:
                yield W("copier", ("tfull", (j - 1) & 1), ((j - 1) >> 1) & 1, (j - 1) >> 1)
            src = [(x, j) for x in smem_w(j)] + ([(x, act_of[j]) for x in smem_act(j)] if act_new[j] else [])
            dst = [(("tmem_w", b), j)] + ([(t, act_of[j]) for t in tmem_act(j)] if act_new[j] else [])
            for t, _ in dst:
                yield F(lambda t=t, j=j: R.write(t, f"scale copies of item {j}"))
            for x, want in src:
                yield F(lambda x=x, want=want, j=j: R.read(x, ("cp", j), want))
            yield ("commit", "cp", [F(lambda src=src, j=j: [R.done(x, ("cp", j)) for x, _ in src]),
                                    F(lambda dst=dst: [R.fill(t, tag) for t, tag in dst]),
                                    A(("sf_ready", b)), A(("atoms_free", b))])

    def builders():
        def copied(x):
            return W("builders", ("atoms_free", x & 1), (x >> 1) & 1, x >> 1)
        for j in range(n):
            if j >= 2:
                yield copied(j - 2)
            if j == 1 and not items[0][0]:
                yield copied(0)
            if j >= 1 and act_new[j] and items[j][0]:
                yield copied(j - 1)
            if glob and act_new[j] and items[j][0] and drop != ("builders", "group"):   # h scales are read
                yield ("spin", lambda g=items[j][1]: glob.ready(g))
            regions = smem_w(j) + (smem_act(j) if act_new[j] else [])
            for x in regions:
                yield F(lambda x=x, j=j: R.write(x, f"builders of item {j}"))
            yield F(lambda j=j: [R.fill(x, j) for x in smem_w(j) + (smem_act(j) if act_new[j] else [])])
            yield A(("atoms_full", j & 1))

    def epilogue():
        for j in range(n):
            b = j & 1
            yield W("epilogue", ("tfull", b), (j >> 1) & 1, j >> 1)
            yield F(lambda j=j, b=b: R.read(("acc", b), ("epi", j), j))
            yield F(lambda j=j, b=b: R.done(("acc", b), ("epi", j)))
            yield A(("tempty", b))
            if glob and not items[j][0]:                    # h planes stored, then the count
                yield F(lambda g=items[j][1]: glob.h_done(g))

    def strip(gen):
        return (a for a in gen if a is not None)

    roles = {"producer": strip(producer()), "mma": strip(mma()), "copier": strip(copier()),
             "builders": strip(builders()), "epilogue": strip(epilogue())}
    return roles, bars, R


def run(items, nk, seed, drop=None, protocol=None):
    rng = random.Random(seed)
    roles, bars, _ = (protocol or build_protocol)(items, nk, drop)
    cur = {name: next(g, None) for name, g in roles.items()}
    inflight = {"mma": [], "cp": []}          # per issuing thread: commit effects, in issue order

    def wait_ok(bar, parity, means):
        b = bars[bar]
        if (b.done & 1) == parity:
            return False
        if b.done != means + 1:
            raise Violation(f"wait on {bar} for phase {means} passed with {b.done} phases completed")
        return True

    def do(act):
        if act[0] == "arrive":
            bars[act[1]].arrive()
        elif act[0] == "fn":
            act[1]()

    # each schedule gives the roles and the two commit streams random speeds, so that some
    # schedules keep one of them far behind the others
    speed = {k: rng.choice([0.02, 0.3, 1.0, 1.0, 3.0]) for k in list(roles) + list(inflight)}
    for _ in range(10 ** 6):
        runnable = [("role", name) for name, act in cur.items()
                    if act is not None and (act[0] != "wait" or wait_ok(*act[1:]))]
        runnable += [("complete", t) for t, q in inflight.items() if q]
        if not runnable:
            break
        kind, who = rng.choices(runnable, weights=[speed[w] for _, w in runnable])[0]
        if kind == "complete":
            for act in inflight[who].pop(0):
                do(act)
            continue
        act = cur[who]
        if act[0] == "commit":
            inflight[act[1]].append(act[2])
        elif act[0] != "wait":
            do(act)
        cur[who] = next(roles[who], None)
    stuck = {name: act for name, act in cur.items() if act is not None}
    if stuck:
        raise Violation(f"deadlock: {stuck}")


def build_protocol_two(mode, nact, nwb):
    """Roles of one CTA of `decode_mx_mma_kernel<mode>` (the two-launch form): a contiguous run
    of items; the epilogue warps also lay out the next item's atoms (before the current item's
    epilogue); nwb weight-atom buffers in shared memory and nact activation-scale buffers in
    TMEM (1 of each when the contraction is too long for two).  Gate/up (mode 0): every item
    multiplies x, whose atoms sit in weight buffer 1's place until item 0's copies are done;
    down (mode 1): the group's activation atoms have a region of their own."""
    def protocol(items, nk, drop=None):
        n = len(items)
        keys = [(g if mode else -1) for _, g in items]
        act_new = [j == 0 or keys[j] != keys[j - 1] for j in range(n)]
        run_of, r = [], -1
        for j in range(n):
            r += act_new[j]
            run_of.append(r)
        act_of = [None] * n
        for j in range(n):
            act_of[j] = j if act_new[j] else act_of[j - 1]
        bars = {}
        for s in range(ST):
            bars[("full", s)] = Bar(1)
            bars[("empty", s)] = Bar(1)
        for b in range(2):
            for nm in ("tfull", "tempty", "atoms_full", "atoms_free", "sf_ready"):
                bars[(nm, b)] = Bar(1)
        R = Regions()

        def smem_w(j):
            return [("smem_w", j % nwb)]

        def smem_act(j):
            return [("smem_w", 1)] if mode == 0 else [("smem_act",)]

        def tmem_act(j):
            return [("tmem_act", run_of[j] % nact)]

        def W(role, bar, parity, means):
            return None if drop == (role, bar[0]) else ("wait", bar, parity, means)

        def A(bar):
            return ("arrive", bar)

        def F(fn):
            return ("fn", fn)

        def producer():
            step = 0
            for j in range(n):
                for kb in range(nk(mode == 1)):
                    s, ph = step % ST, (step // ST) & 1
                    yield W("producer", ("empty", s), ph ^ 1, step // ST - 1)
                    yield F(lambda s=s, j=j: R.write(("stage", s), f"TMA of item {j}"))
                    yield F(lambda s=s, j=j, kb=kb: R.fill(("stage", s), (j, kb)))
                    yield A(("full", s))
                    step += 1

        def mma():
            step = 0
            for j in range(n):
                b = j & 1
                yield W("mma", ("sf_ready", b), (j >> 1) & 1, j >> 1)
                yield W("mma", ("tempty", b), ((j >> 1) & 1) ^ 1, (j >> 1) - 1)
                yield F(lambda j=j, b=b: R.write(("acc", b), f"MMAs of item {j}"))
                yield F(lambda j=j, b=b: R.read(("tmem_w", b), ("mma", j), j))
                for t in tmem_act(j):
                    yield F(lambda t=t, j=j: R.read(t, ("mma", j), act_of[j]))
                for kb in range(nk(mode == 1)):
                    s, ph = step % ST, (step // ST) & 1
                    yield W("mma", ("full", s), ph, step // ST)
                    yield F(lambda s=s, j=j, kb=kb: R.read(("stage", s), ("mma", j, kb), (j, kb)))
                    yield ("commit", "mma", [F(lambda s=s, j=j, kb=kb: R.done(("stage", s), ("mma", j, kb))),
                                             A(("empty", s))])
                    step += 1
                yield ("commit", "mma", [F(lambda j=j, b=b: [R.done(t, ("mma", j)) for t in [("tmem_w", b)] + tmem_act(j)]),
                                         F(lambda j=j, b=b: R.fill(("acc", b), j)),
                                         F(lambda j=j, b=b: R.readers.setdefault(("acc", b), set()).add(("epi", j))),
                                         A(("tfull", b))])

        def copier():
            for j in range(n):
                b, wb = j & 1, j % nwb
                yield W("copier", ("atoms_full", wb), (j // nwb) & 1, j // nwb)
                if j >= 2:
                    yield W("copier", ("tfull", b), ((j - 2) >> 1) & 1, (j - 2) >> 1)
                if act_new[j] and nact == 1 and j >= 1:
                    yield W("copier", ("tfull", (j - 1) & 1), ((j - 1) >> 1) & 1, (j - 1) >> 1)
                src = [(x, j) for x in smem_w(j)] + ([(x, act_of[j]) for x in smem_act(j)] if act_new[j] else [])
                dst = [(("tmem_w", b), j)] + ([(t, act_of[j]) for t in tmem_act(j)] if act_new[j] else [])
                for t, _ in dst:
                    yield F(lambda t=t, j=j: R.write(t, f"scale copies of item {j}"))
                for x, want in src:
                    yield F(lambda x=x, want=want, j=j: R.read(x, ("cp", j), want))
                yield ("commit", "cp", [F(lambda src=src, j=j: [R.done(x, ("cp", j)) for x, _ in src]),
                                        F(lambda dst=dst: [R.fill(t, tag) for t, tag in dst]),
                                        A(("sf_ready", b)), A(("atoms_free", wb))])

        def epilogue_builders():
            def copied(x):
                return W("epilogue", ("atoms_free", x % nwb), (x // nwb) & 1, x // nwb)

            def build(j):
                regions = smem_w(j) + (smem_act(j) if act_new[j] else [])
                for x in regions:
                    yield F(lambda x=x, j=j: R.write(x, f"atoms of item {j}"))
                yield F(lambda j=j, regions=regions: [R.fill(x, j) for x in regions])
                yield A(("atoms_full", j % nwb))
            yield from build(0)
            for j in range(n):
                if j + 1 < n:
                    if j + 1 >= nwb:
                        yield copied(j + 1 - nwb)
                    if act_new[j + 1] or (mode == 0 and j == 0):
                        yield copied(j)
                    yield from build(j + 1)
                b = j & 1
                yield W("epilogue", ("tfull", b), (j >> 1) & 1, j >> 1)
                yield F(lambda j=j, b=b: R.read(("acc", b), ("epi", j), j))
                yield F(lambda j=j, b=b: R.done(("acc", b), ("epi", j)))
                yield A(("tempty", b))

        def strip(gen):
            return (a for a in gen if a is not None)

        roles = {"producer": strip(producer()), "mma": strip(mma()), "copier": strip(copier()),
                 "epilogue": strip(epilogue_builders())}
        return roles, bars, R
    return protocol


@pytest.mark.parametrize("mode,nact,nwb", [(0, 1, 2), (1, 2, 2), (1, 1, 1), (1, 2, 1), (1, 1, 2)])
def test_two_launch_decode_protocol_random_interleavings(mode, nact, nwb):
    """The two-launch kernel at every buffer plan its host side can pick: gate/up (one x scale
    buffer, two weight-atom buffers), down with K <= 3072 (two and two) and longer K (one
    activation-scale buffer in TMEM, one weight-atom buffer), plus the mixed plans."""
    rng = random.Random(mode * 7 + nact * 3 + nwb)
    proto = build_protocol_two(mode, nact, nwb)
    for _ in range(40):
        n = rng.choice([1, 2, 3, 5, 9, 14])
        g, groups = rng.randrange(4), []
        for _ in range(n):
            if rng.random() < 0.3:
                g += 1
            groups.append(g)
        items = [(mode == 1, gg) for gg in groups]
        for seed in range(10):
            run(items, lambda down: 3 if down else 5, seed, protocol=proto)


# (In this form the MMA thread's wait for the epilogue to hand an accumulator back is implied:
# item j + 2's scale atoms are laid out by the same warps only after item j's epilogue, so the
# model finds no race without it; the waits below are the ones whose absence is one.)
@pytest.mark.parametrize("drop", [("copier", "tfull"), ("epilogue", "atoms_free"), ("mma", "sf_ready"),
                                  ("copier", "atoms_full"), ("producer", "empty")])
def test_two_launch_checker_catches_a_dropped_wait(drop):
    proto = build_protocol_two(1, 1, 1)
    items = [(True, 0), (True, 0), (True, 1), (True, 1), (True, 2), (True, 3)]
    for seed in range(400):
        try:
            run(items, lambda down: 3, seed, drop=drop, protocol=proto)
        except Violation:
            return
    raise AssertionError(f"dropping the {drop[0]}'s wait on {drop[1]} went unnoticed")


def item_lists(rng, count=60):
    """Item sequences of one CTA: gate/up items, then down items of groups that may change at
    every item or repeat (CTAs with only gate/up or only down items included)."""
    out = []
    while len(out) < count:
        n_gu = rng.choice([0, 1, 2, 3, 5, 9])
        n_dn = rng.choice([0, 1, 2, 4, 9])
        if n_gu + n_dn == 0:
            continue
        groups, g = [], rng.randrange(3)
        for _ in range(n_dn):
            if rng.random() < 0.6:
                g += 1 + rng.randrange(3)
            groups.append(g)
        out.append([(False, 0)] * n_gu + [(True, gg) for gg in groups])
    return out


@pytest.mark.parametrize("nk_gu,nk_dn", [(16, 8), (4, 2), (1, 1), (2, 5)])
def test_fused_decode_protocol_random_interleavings(nk_gu, nk_dn):
    rng = random.Random(nk_gu * 31 + nk_dn)
    for items in item_lists(rng):
        for seed in range(12):
            run(items, lambda down: nk_dn if down else nk_gu, seed)


# each planted mistake, with an item sequence that exposes it
MISTAKES = [
    (("copier", "tfull"), [(False, 0)] * 6),                          # weight scales rewritten under MMAs
    (("builders", "atoms_free"), [(False, 0)] * 3 + [(True, 1), (True, 2), (True, 3)]),   # atoms rewritten under copies
    (("mma", "tempty"), [(False, 0)] * 6),                            # accumulator rewritten under the epilogue
    (("mma", "sf_ready"), [(False, 0)] * 4),                          # MMAs read scales not yet copied
    (("epilogue", "tfull"), [(False, 0)] * 3),                        # epilogue reads an unfinished accumulator
    (("producer", "empty"), [(False, 0)] * 3),                        # TMA overwrites a stage under MMAs
    (("copier", "atoms_full"), [(False, 0)] * 3),                     # copies of atoms not yet laid out
]


@pytest.mark.parametrize("drop,items", MISTAKES, ids=[f"{r}-{b}" for (r, b), _ in MISTAKES])
def test_checker_catches_a_dropped_wait(drop, items):
    caught = False
    for seed in range(400):
        try:
            run(items, lambda down: 3 if down else 6, seed, drop=drop)
        except Violation:
            caught = True
            break
    assert caught, f"dropping the {drop[0]}'s wait on {drop[1]} went unnoticed"


def test_checker_catches_the_missing_first_down_wait():
    """Without the copier's wait for the last gate/up item before the first down item's
    activation scales, the x scale columns are overwritten while that item's MMAs may read them."""
    import types
    items = [(False, 0)] * 3 + [(True, 1), (True, 2)]
    orig = build_protocol

    def variant(items, nk, drop=None):
        roles, bars, R = orig(items, nk, drop)
        gen = roles["copier"]
        # the first-down wait is the second tfull wait of that item: drop waits on the previous
        # item's buffer (parity of item j - 1) at the first down item j = 3
        def filtered():
            seen_atoms = 0
            for a in gen:
                if a[0] == "wait" and a[1][0] == "atoms_full":
                    seen_atoms += 1
                if seen_atoms == 4 and a[0] == "wait" and a[1] == ("tfull", 0) and a[3] == 1:
                    continue
                yield a
        roles["copier"] = filtered()
        return roles, bars, R

    caught = False
    g = globals()
    g["build_protocol"] = variant
    try:
        for seed in range(600):
            try:
                run(items, lambda down: 3 if down else 6, seed)
            except Violation:
                caught = True
                break
    finally:
        g["build_protocol"] = orig
    assert caught


def run_launch(ctas, nk, glob, seed, drop=None, protocol=None):
    """Several CTAs' roles under one random schedule (CTA roles and commit streams with random
    speeds); the launch must finish and leave every group's counters at zero."""
    rng = random.Random(seed)
    roles, bars, inflight, cur, speed = {}, {}, {}, {}, {}
    for c, items in enumerate(ctas):
        r, b, _ = (protocol or build_protocol)(items, nk, drop=drop, glob=glob)
        for name, gen in r.items():
            roles[(c, name)] = gen
            cur[(c, name)] = next(gen, None)
            speed[(c, name)] = rng.choice([0.02, 0.3, 1.0, 1.0, 3.0])
        bars[c] = b
        for t in ("mma", "cp"):                      # commit streams, keyed apart from the roles
            inflight[(c, t, "q")] = []
            speed[(c, t, "q")] = rng.choice([0.05, 1.0, 3.0])

    def ok(key, act):
        if act[0] == "spin":
            return act[1]()
        if act[0] != "wait":
            return True
        bar, parity, means = act[1:]
        b = bars[key[0]][bar]
        if (b.done & 1) == parity:
            return False
        if b.done != means + 1:
            raise Violation(f"CTA {key[0]}: wait on {bar} for phase {means} passed after {b.done}")
        return True

    for _ in range(10 ** 7):
        runnable = [k for k, a in cur.items() if a is not None and ok(k, a)]
        runnable += [k for k, q in inflight.items() if q]
        if not runnable:
            break
        k = rng.choices(runnable, weights=[speed[x] for x in runnable])[0]
        if k in inflight:
            for act in inflight[k].pop(0):
                if act[0] == "arrive":
                    bars[k[0]][act[1]].arrive()
                else:
                    act[1]()
            continue
        act = cur[k]
        if act[0] == "commit":
            inflight[(k[0], act[1], "q")].append(act[2])
        elif act[0] == "arrive":
            bars[k[0]][act[1]].arrive()
        elif act[0] == "fn":
            act[1]()
        cur[k] = next(roles[k], None)
    stuck = {k: a for k, a in cur.items() if a is not None}
    if stuck:
        raise Violation(f"deadlock: {stuck}")
    if any(glob.h) or any(glob.reads):
        raise Violation(f"counters left at h={glob.h} reads={glob.reads}")


@pytest.mark.parametrize("n_act,gu_blocks,dn_blocks,grid", [(3, 2, 3, 4), (2, 4, 2, 3), (5, 1, 1, 7),
                                                             (1, 3, 5, 9), (4, 3, 2, 5)])
def test_fused_decode_launch_cross_cta(n_act, gu_blocks, dn_blocks, grid):
    """The whole launch: items b, b + grid, ... of [gate/up items | down items] per CTA (some
    CTAs start on down items), down items waiting for their group's gate/up epilogues in other
    CTAs and their own; every schedule finishes with the counters back at zero."""
    gu = [(False, g) for g in range(n_act) for _ in range(gu_blocks)]
    dn = [(True, g) for g in range(n_act) for _ in range(dn_blocks)]
    lst = gu + dn
    ctas = [lst[b::grid] for b in range(min(grid, len(lst)))]
    for seed in range(40):
        run_launch(ctas, lambda down: 2, Groups(n_act, gu_blocks, dn_blocks), seed)


class EarlyReset(Groups):
    """A planted counting mistake: the counters reset after the producers' reads alone."""

    def read_done(self, g):
        if not self.ready(g):
            raise Violation(f"a read of group {g} counted before all its h was written")
        self.reads[g] += 1
        if self.reads[g] == self.dn:
            self.h[g], self.reads[g] = 0, 0


@pytest.mark.parametrize("mistake", ["producer-wait", "builders-wait", "early-reset"])
def test_cross_cta_checker_catches_mistakes(mistake):
    n_act, gu_blocks, dn_blocks, grid = 3, 2, 3, 4
    gu = [(False, g) for g in range(n_act) for _ in range(gu_blocks)]
    dn = [(True, g) for g in range(n_act) for _ in range(dn_blocks)]
    lst = gu + dn
    ctas = [lst[b::grid] for b in range(grid)]
    drop = {"producer-wait": ("producer", "group"), "builders-wait": ("builders", "group")}.get(mistake)
    kind = EarlyReset if mistake == "early-reset" else Groups
    for seed in range(300):
        try:
            run_launch(ctas, lambda down: 2, kind(n_act, gu_blocks, dn_blocks), seed, drop=drop)
        except Violation:
            return
    raise AssertionError(f"{mistake} went unnoticed")


class GroupsBF16(Groups):
    """The BF16 tensor-core decode counts one read per down item (its producer's): the last of
    dn_blocks resets the group."""

    def read_done(self, g):
        if not self.ready(g):
            raise Violation(f"a read of group {g} counted before all its h was written")
        self.reads[g] += 1
        if self.reads[g] == self.dn:
            self.h[g], self.reads[g] = 0, 0


def build_protocol_bf16(items, nk, drop=None, glob=None, stages=3):
    """Roles of one CTA of the BF16 tensor-core decode (`decode_mma_kernel`, csrc/decode_mma.cu):
    a 3-stage ring, two accumulators, no scale factors; items b, b + grid, ... of [gate/up |
    down]; the producer waits for a down item's group before its first load and counts the read;
    the gate/up epilogue hands the accumulator back, stores h and counts itself."""
    n = len(items)
    bars = {}
    for s_ in range(stages):
        bars[("full", s_)] = Bar(1)
        bars[("empty", s_)] = Bar(1)
    for b in range(2):
        bars[("tfull", b)] = Bar(1)
        bars[("tempty", b)] = Bar(1)
    R = Regions()

    def W(role, bar, parity, means):
        return None if drop == (role, bar[0]) else ("wait", bar, parity, means)

    def producer():
        step = 0
        for j in range(n):
            if glob and items[j][0]:
                g = items[j][1]
                if drop != ("producer", "group"):
                    yield ("spin", lambda g=g: glob.ready(g))
                yield ("fn", lambda g=g: glob.read_done(g))
            for kb in range(nk(items[j][0])):
                s_, ph = step % stages, (step // stages) & 1
                yield W("producer", ("empty", s_), ph ^ 1, step // stages - 1)
                yield ("fn", lambda s_=s_, j=j: R.write(("stage", s_), f"TMA of item {j}"))
                yield ("fn", lambda s_=s_, j=j, kb=kb: R.fill(("stage", s_), (j, kb)))
                yield ("arrive", ("full", s_))
                step += 1

    def mma():
        step = 0
        for j in range(n):
            b = j & 1
            yield W("mma", ("tempty", b), ((j >> 1) & 1) ^ 1, (j >> 1) - 1)
            yield ("fn", lambda j=j, b=b: R.write(("acc", b), f"MMAs of item {j}"))
            for kb in range(nk(items[j][0])):
                s_, ph = step % stages, (step // stages) & 1
                yield W("mma", ("full", s_), ph, step // stages)
                yield ("fn", lambda s_=s_, j=j, kb=kb: R.read(("stage", s_), ("mma", j, kb), (j, kb)))
                yield ("commit", "mma", [("fn", lambda s_=s_, j=j, kb=kb: R.done(("stage", s_), ("mma", j, kb))),
                                         ("arrive", ("empty", s_))])
                step += 1
            yield ("commit", "mma", [("fn", lambda j=j, b=b: R.fill(("acc", b), j)),
                                     ("fn", lambda j=j, b=b: R.readers.setdefault(("acc", b), set()).add(("epi", j))),
                                     ("arrive", ("tfull", b))])

    def epilogue():
        for j in range(n):
            b = j & 1
            yield W("epilogue", ("tfull", b), (j >> 1) & 1, j >> 1)
            yield ("fn", lambda j=j, b=b: R.read(("acc", b), ("epi", j), j))
            yield ("fn", lambda j=j, b=b: R.done(("acc", b), ("epi", j)))
            yield ("arrive", ("tempty", b))
            if glob and not items[j][0]:
                yield ("fn", lambda g=items[j][1]: glob.h_done(g))

    def strip(gen):
        return (a for a in gen if a is not None)

    roles = {"producer": strip(producer()), "mma": strip(mma()), "epilogue": strip(epilogue())}
    return roles, bars, R


@pytest.mark.parametrize("n_act,gu_blocks,dn_blocks,grid", [(3, 2, 3, 4), (2, 4, 2, 3), (5, 1, 1, 7),
                                                             (1, 3, 5, 9), (6, 2, 4, 12)])
def test_bf16_decode_launch_cross_cta(n_act, gu_blocks, dn_blocks, grid):
    """The BF16 tensor-core decode's whole launch (several CTAs per SM in the kernel: here as
    many independent CTAs), with its producer-only read count."""
    gu = [(False, g) for g in range(n_act) for _ in range(gu_blocks)]
    dn = [(True, g) for g in range(n_act) for _ in range(dn_blocks)]
    lst = gu + dn
    ctas = [lst[b::grid] for b in range(min(grid, len(lst)))]
    for seed in range(40):
        run_launch(ctas, lambda down: 2 if down else 3, GroupsBF16(n_act, gu_blocks, dn_blocks), seed,
                   protocol=build_protocol_bf16)


@pytest.mark.parametrize("drop", [("producer", "group"), ("mma", "tempty"), ("producer", "empty"),
                                  ("epilogue", "tfull"), ("mma", "full")])
def test_bf16_checker_catches_mistakes(drop):
    n_act, gu_blocks, dn_blocks, grid = 3, 2, 3, 4
    gu = [(False, g) for g in range(n_act) for _ in range(gu_blocks)]
    dn = [(True, g) for g in range(n_act) for _ in range(dn_blocks)]
    lst = gu + dn
    ctas = [lst[b::grid] for b in range(grid)]
    for seed in range(300):
        try:
            run_launch(ctas, lambda down: 2, GroupsBF16(n_act, gu_blocks, dn_blocks), seed, drop=drop,
                       protocol=build_protocol_bf16)
        except Violation:
            return
    raise AssertionError(f"dropping the {drop[0]}'s wait on {drop[1]} went unnoticed")
