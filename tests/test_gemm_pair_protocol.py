"""Model check, on the CPU, of the cross-CTA protocols of the CTA-pair grouped GEMMs
(`moe_gemm_pair_kernel`, csrc/gemm_sm100.cu, and `moe_gemm_mx_pair_kernel`, csrc/gemm_mx_sm100.cu,
whose code-unit ring, scale buffers and converter groups are modelled below the BF16 part): two
CTAs share every MMA (`cta_group::2`).

Written from the kernel:
* both CTAs' producers wait on their own `empty[s]` and issue TMA copies whose bytes complete on
  the LEADER's `full[s]`; only the leader's producer arrives there, expecting both CTAs' bytes
  (`mbarrier.arrive.expect_tx`), so the peer's bytes may land before or after that arrival;
* the leader's MMA thread waits on `tempty[b]` (both CTAs' epilogues arrive there) and on
  `full[s]`, reads both CTAs' stages, writes both CTAs' accumulators, and its commits arrive on
  `empty[s]` and `tfull[b]` in both CTAs;
* each CTA's epilogue waits on its own `tfull[b]`, reads its accumulator half, and arrives on the
  leader's `tempty[b]`.

mbarrier phases complete when every expected arrival has come and the transaction count is
back to zero (it may go below zero in between).  TMA completions are independent events (any
order); a thread's commits complete in issue order.  Random schedules with random per-role speeds
must all finish; every wait must be satisfied by its own phase; every copy's bytes must land in
the phase they were issued for; no stage or accumulator may be overwritten under a live reader,
and every reader must find the tile and K step it expects.  Planted mistakes must be caught.
"""
import random

import pytest


class Violation(AssertionError):
    pass


class TxBar:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.done = count, 0, 0, 0

    def _check(self):
        if self.pending == self.count and self.tx == 0:
            self.pending, self.done = 0, self.done + 1

    def arrive(self, expect=0):
        self.tx += expect
        self.pending += 1
        if self.pending > self.count:
            raise Violation("more arrivals than the barrier expects in one phase")
        self._check()

    def complete_tx(self, n, phase, what):
        if self.done != phase:
            raise Violation(f"{what}: bytes of phase {phase} landed while the barrier is in phase {self.done}")
        self.tx -= n
        self._check()


def build(tiles, nk, ST=4, NBUF=2, mistake=None):
    """Roles of one CTA pair for `tiles` tiles of nk K steps each."""
    bars = {("full", s): TxBar(1) for s in range(ST)}                 # the leader's
    for c in (0, 1):
        for s in range(ST):
            bars[("empty", c, s)] = TxBar(1)
        for b in range(NBUF):
            bars[("tfull", c, b)] = TxBar(1)
    for b in range(NBUF):
        bars[("tempty", b)] = TxBar(1 if mistake == "tempty-count" else 2)   # both CTAs' epilogues
    readers, content = {}, {}
    BYTES = 7                                                          # per CTA and stage

    def write(r, who):
        if readers.get(r):
            raise Violation(f"{who} writes {r} under readers {sorted(readers[r])}")

    def read(r, tag, want):
        if content.get(r) != want:
            raise Violation(f"{tag} reads {r} = {content.get(r)}, expected {want}")
        readers.setdefault(r, set()).add(tag)

    def done(r, tag):
        readers.get(r, set()).discard(tag)

    def W(bar, parity, means):
        return ("wait", bar, parity, means)

    def producer(c):
        step = 0
        for t in range(tiles):
            for kb in range(nk):
                s, ph = step % ST, (step // ST) & 1
                if not (mistake == "peer-skips-empty" and c == 1):
                    yield W(("empty", c, s), ph ^ 1, step // ST - 1)
                yield ("fn", lambda c=c, s=s, t=t: write(("stage", c, s), f"TMA of CTA {c}"))
                if c == 0:
                    n = (1 if mistake == "leader-expects-own-bytes" else 2) * BYTES
                    yield ("fn", lambda s=s, n=n: bars[("full", s)].arrive(expect=n))
                # the copy lands later, on the leader's barrier, in this step's phase of it
                yield ("tma", [("fn", lambda c=c, s=s, t=t, kb=kb: content.__setitem__(("stage", c, s), (t, kb))),
                               ("fn", lambda s=s, k=step // ST: bars[("full", s)].complete_tx(BYTES, k, f"copy to stage {s}"))])
                step += 1

    def mma():
        step = 0
        for t in range(tiles):
            b = t % NBUF
            if mistake != "mma-skips-tempty":
                yield W(("tempty", b), ((t // NBUF) & 1) ^ 1, t // NBUF - 1)
            for c in (0, 1):
                yield ("fn", lambda c=c, b=b, t=t: write(("acc", c, b), f"MMAs of tile {t}"))
            for kb in range(nk):
                s, ph = step % ST, (step // ST) & 1
                yield W(("full", s), ph, step // ST)
                for c in (0, 1):
                    yield ("fn", lambda c=c, s=s, t=t, kb=kb: read(("stage", c, s), ("mma", t, kb), (t, kb)))
                yield ("commit", [("fn", lambda s=s, t=t, kb=kb: [done(("stage", c, s), ("mma", t, kb)) for c in (0, 1)])]
                       + [("arrive", ("empty", c, s)) for c in (0, 1)])
                step += 1
            yield ("commit", [("fn", lambda b=b, t=t: [content.__setitem__(("acc", c, b), t) for c in (0, 1)]),
                              ("fn", lambda b=b, t=t: [readers.setdefault(("acc", c, b), set()).add(("epi", c, t))
                                                       for c in (0, 1)])]
                   + [("arrive", ("tfull", c, b)) for c in (0, 1)])

    def epilogue(c):
        for t in range(tiles):
            b = t % NBUF
            yield W(("tfull", c, b), (t // NBUF) & 1, t // NBUF)
            yield ("fn", lambda c=c, b=b, t=t: read(("acc", c, b), ("epi", c, t), t))
            yield ("fn", lambda c=c, b=b, t=t: done(("acc", c, b), ("epi", c, t)))
            yield ("arrive", ("tempty", b))

    roles = {("prod", 0): producer(0), ("prod", 1): producer(1), ("mma",): mma(),
             ("epi", 0): epilogue(0), ("epi", 1): epilogue(1)}
    return roles, bars


def run(tiles, nk, seed, mistake=None):
    rng = random.Random(seed)
    roles, bars = build(tiles, nk, mistake=mistake)
    cur = {k: next(g, None) for k, g in roles.items()}
    tma, commits = [], []                       # in-flight copies (any order), commits (in order)
    speed = {k: rng.choice([0.02, 0.3, 1.0, 1.0, 3.0]) for k in list(roles) + ["tma", "commit"]}

    def ok(act):
        if act[0] != "wait":
            return True
        bar, parity, means = act[1:]
        b = bars[bar]
        if (b.done & 1) == parity:
            return False
        if b.done != means + 1:
            raise Violation(f"wait on {bar} for phase {means} passed after {b.done} phases")
        return True

    def do(act):
        if act[0] == "arrive":
            bars[act[1]].arrive()
        elif act[0] == "fn":
            act[1]()

    for _ in range(10 ** 6):
        cands = [k for k, a in cur.items() if a is not None and ok(a)]
        if tma:
            cands.append("tma")
        if commits:
            cands.append("commit")
        if not cands:
            break
        k = rng.choices(cands, weights=[speed[x] for x in cands])[0]
        if k == "tma":
            for act in tma.pop(rng.randrange(len(tma))):
                do(act)
            continue
        if k == "commit":
            for act in commits.pop(0):
                do(act)
            continue
        act = cur[k]
        if act[0] == "tma":
            tma.append(act[1])
        elif act[0] == "commit":
            commits.append(act[1])
        elif act[0] != "wait":
            do(act)
        cur[k] = next(roles[k], None)
    stuck = {k: a for k, a in cur.items() if a is not None}
    if stuck or tma or commits:
        raise Violation(f"deadlock: {stuck}, {len(tma)} copies and {len(commits)} commits pending")


@pytest.mark.parametrize("tiles,nk", [(1, 1), (3, 2), (5, 7), (9, 3), (2, 13)])
def test_pair_gemm_protocol_random_interleavings(tiles, nk):
    for seed in range(150):
        run(tiles, nk, seed)


@pytest.mark.parametrize("mistake", ["leader-expects-own-bytes", "peer-skips-empty", "mma-skips-tempty",
                                     "tempty-count"])
def test_pair_gemm_checker_catches_mistakes(mistake):
    """The leader expecting only its own bytes (the peer's half may be read before it lands),
    the peer's producer not waiting for the leader's release of a stage, the MMA thread not
    waiting for both epilogues, and a hand-back barrier that completes on one CTA's arrival."""
    for seed in range(500):
        try:
            run(4, 3, seed, mistake=mistake)
        except Violation:
            return
    raise AssertionError(f"{mistake} went unnoticed")


# ---------------------------------------------------------------- MXFP4 CTA pair
def build_mx(tiles, nk, mistake=None):
    """Roles of one CTA pair of `moe_gemm_mx_pair_kernel` (csrc/gemm_mx_sm100.cu): per CTA a
    token producer (its half of the token tile, bytes on the leader's bfull), a code producer
    (units of two K steps into a 3-deep ring on its own cfull, every fourth unit also the next
    scale tile into one of two scale buffers), and two converter groups taking alternate K steps
    (read their half of the unit -- and at a scale group's first unit the scales -- release the
    unit, wait for the stage, write the A tile, arrive on the leader's afull), which also run the
    epilogue of every tile; the leader's MMA thread waits on tempty (all four groups), bfull and
    afull, and commits to empty and tfull in both CTAs.  nk % 8 == 0."""
    ST, CST, BY, CBY = 3, 3, 5, 11
    nsteps, nunits = tiles * nk, tiles * nk // 2
    bars = {}
    for s in range(ST):
        bars[("bfull", s)] = TxBar(1)
        bars[("afull", s)] = TxBar(1 if mistake == "afull-one-cta" else 2)
        for c in (0, 1):
            bars[("empty", c, s)] = TxBar(1)
    for c in (0, 1):
        for s in range(CST):
            bars[("cfull", c, s)] = TxBar(1)
            bars[("cempty", c, s)] = TxBar(2)
        bars[("tfull", c)] = TxBar(1)
    bars[("tempty",)] = TxBar(4)
    readers, content = {}, {}

    def write(r, who):
        if readers.get(r):
            raise Violation(f"{who} writes {r} under readers {sorted(readers[r])}")

    def read(r, tag, want):
        if content.get(r) != want:
            raise Violation(f"{tag} reads {r} = {content.get(r)}, expected {want}")

    def W(bar, parity, means):
        return ("wait", bar, parity, means)

    def arrive(bar, phase):
        b = bars[bar]
        if b.done != phase:
            raise Violation(f"arrival for phase {phase} on {bar} while it is in phase {b.done}")
        b.arrive()

    def tok_prod(c):
        for n in range(nsteps):
            s = n % ST
            yield W(("empty", c, s), ((n // ST) & 1) ^ 1, n // ST - 1)
            yield ("fn", lambda c=c, s=s: write(("B", c, s), f"token copy of CTA {c}"))
            if c == 0:
                yield ("fn", lambda s=s: bars[("bfull", s)].arrive(expect=2 * BY))
            yield ("tma", [("fn", lambda c=c, s=s, n=n: content.__setitem__(("B", c, s), n)),
                           ("fn", lambda s=s, k=n // ST: bars[("bfull", s)].complete_tx(BY, k, "token copy"))])

    def code_prod(c):
        for u in range(nunits):
            cs = u % CST
            if not (mistake == "code-skips-cempty" and c == 1):
                yield W(("cempty", c, cs), ((u // CST) & 1) ^ 1, u // CST - 1)
            scales = u % 4 == 0
            yield ("fn", lambda c=c, cs=cs, scales=scales: bars[("cfull", c, cs)].arrive(expect=CBY + (CBY if scales else 0)))
            fills = [("fn", lambda c=c, cs=cs, u=u: content.__setitem__(("code", c, cs), u)),
                     ("fn", lambda c=c, cs=cs, k=u // CST: bars[("cfull", c, cs)].complete_tx(CBY, k, "code copy"))]
            if scales:
                sb = (u // 4) & 1
                fills += [("fn", lambda c=c, sb=sb, u=u: content.__setitem__(("scale", c, sb), u // 4)),
                          ("fn", lambda c=c, cs=cs, k=u // CST: bars[("cfull", c, cs)].complete_tx(CBY, k, "scale copy"))]
            yield ("tma", fills)

    def conv(c, gi):
        for t in range(tiles):
            for kb in range(gi, nk, 2):
                n = t * nk + kb
                u, s = n >> 1, n % ST
                yield W(("cfull", c, u % CST), (u // CST) & 1, u // CST)
                if (kb & 7) < 2:
                    yield ("fn", lambda c=c, n=n: read(("scale", c, (n >> 3) & 1), ("conv", c, n), n >> 3))
                yield ("fn", lambda c=c, u=u, n=n: read(("code", c, u % CST), ("conv", c, n), u))
                yield ("fn", lambda c=c, u=u: arrive(("cempty", c, u % CST), u // CST))
                if mistake != "conv-skips-empty":
                    yield W(("empty", c, s), ((n // ST) & 1) ^ 1, n // ST - 1)
                yield ("fn", lambda c=c, s=s, n=n: write(("A", c, s), f"converters of CTA {c}"))
                yield ("fn", lambda c=c, s=s, n=n: content.__setitem__(("A", c, s), n))
                yield ("fn", lambda s=s, n=n: arrive(("afull", s), n // ST))
            yield W(("tfull", c), t & 1, t)
            yield ("fn", lambda c=c, t=t: read(("acc", c), ("epi", c, gi, t), t))
            yield ("fn", lambda c=c, gi=gi, t=t: readers.get(("acc", c), set()).discard(("epi", c, gi, t)))
            yield ("fn", lambda t=t: arrive(("tempty",), t))

    def mma():
        for t in range(tiles):
            yield W(("tempty",), (t & 1) ^ 1, t - 1)
            for c in (0, 1):
                yield ("fn", lambda c=c, t=t: write(("acc", c), f"MMAs of tile {t}"))
            for kb in range(nk):
                n = t * nk + kb
                s = n % ST
                yield W(("bfull", s), (n // ST) & 1, n // ST)
                yield W(("afull", s), (n // ST) & 1, n // ST)
                for c in (0, 1):
                    for op in ("A", "B"):
                        yield ("fn", lambda c=c, s=s, n=n, op=op: [read((op, c, s), ("mma", n), n),
                                                                    readers.setdefault((op, c, s), set()).add(("mma", n))])
                yield ("commit", [("fn", lambda s=s, n=n: [readers.get((op, c, s), set()).discard(("mma", n))
                                                           for c in (0, 1) for op in ("A", "B")])]
                       + [("arrive", ("empty", c, s)) for c in (0, 1)])
            yield ("commit", [("fn", lambda t=t: [content.__setitem__(("acc", c), t) for c in (0, 1)]),
                              ("fn", lambda t=t: [readers.setdefault(("acc", c), set()).add(("epi", c, g, t))
                                                  for c in (0, 1) for g in (0, 1)])]
                   + [("arrive", ("tfull", c)) for c in (0, 1)])

    roles = {("mma",): mma()}
    for c in (0, 1):
        roles[("tok", c)] = tok_prod(c)
        roles[("code", c)] = code_prod(c)
        for gi in (0, 1):
            roles[("conv", c, gi)] = conv(c, gi)
    return roles, bars


def run_mx(tiles, nk, seed, mistake=None):
    rng = random.Random(seed)
    roles, bars = build_mx(tiles, nk, mistake)
    cur = {k: next(g, None) for k, g in roles.items()}
    tma, commits = [], []
    speed = {k: rng.choice([0.02, 0.3, 1.0, 1.0, 3.0]) for k in list(roles) + ["tma", "commit"]}

    def ok(act):
        if act[0] != "wait":
            return True
        bar, parity, means = act[1:]
        b = bars[bar]
        if (b.done & 1) == parity:
            return False
        if b.done != means + 1:
            raise Violation(f"wait on {bar} for phase {means} passed after {b.done} phases")
        return True

    def do(act):
        if act[0] == "arrive":
            bars[act[1]].arrive()
        elif act[0] == "fn":
            act[1]()

    for _ in range(10 ** 6):
        cands = [k for k, a in cur.items() if a is not None and ok(a)]
        cands += ["tma"] if tma else []
        cands += ["commit"] if commits else []
        if not cands:
            break
        k = rng.choices(cands, weights=[speed[x] for x in cands])[0]
        if k == "tma":
            for act in tma.pop(rng.randrange(len(tma))):
                do(act)
            continue
        if k == "commit":
            for act in commits.pop(0):
                do(act)
            continue
        act = cur[k]
        if act[0] == "tma":
            tma.append(act[1])
        elif act[0] == "commit":
            commits.append(act[1])
        elif act[0] != "wait":
            do(act)
        cur[k] = next(roles[k], None)
    stuck = {k: a for k, a in cur.items() if a is not None}
    if stuck or tma or commits:
        raise Violation(f"deadlock: {stuck}, {len(tma)} copies and {len(commits)} commits pending")


@pytest.mark.parametrize("tiles,nk", [(1, 8), (2, 8), (3, 16), (5, 8)])
def test_mx_pair_gemm_protocol_random_interleavings(tiles, nk):
    for seed in range(60):
        run_mx(tiles, nk, seed)


@pytest.mark.parametrize("mistake", ["code-skips-cempty", "conv-skips-empty", "afull-one-cta"])
def test_mx_pair_gemm_checker_catches_mistakes(mistake):
    """The code producer overwriting a unit (and with it a scale buffer) the converters have not
    read, converters writing an A stage the MMAs still read, and an afull phase completing on
    one CTA's converters."""
    for seed in range(400):
        try:
            run_mx(2, 8, seed, mistake=mistake)
        except Violation:
            return
    raise AssertionError(f"{mistake} went unnoticed")
