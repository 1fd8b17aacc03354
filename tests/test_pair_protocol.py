"""The barrier protocol of the CTA-pair decode attention kernel
(csrc/sm100_attend_pair.cu, attend_pair_kernel), modelled on the CPU.

Two CTAs form one MMA unit: the even CTA's MMA warp issues every score and
value GEMM; each GEMM reads operands staged in both CTAs' shared memory and
accumulates into both CTAs' TMEM, and its commits arrive on the barrier at
the same offset in both CTAs.  Per CTA the model runs the key/query loader,
the value loader (request and relay sides), and the softmax/epilogue group
as coroutines interleaved at random, plus the even CTA's MMA warp; the pair's
tensor core completes GEMMs in issue order, the copy engine lands loads in
any order.  Each mbarrier is a completion counter with expect-tx bytes whose
parity waits behave as on the device (a wait passes on any phase other than
the one its parity names).

The model checks that every wait passes on the completion it names, that no
staged chunk, query row block, P buffer or score buffer is replaced before
its last reader is done, that each GEMM reads what it should (the same tile
and chunk in both CTAs), that value GEMMs accumulate in order within an item
and the first one of an item starts only after both epilogues have read O,
that each epilogue reads its item's complete O, and that everything
finishes.  Control runs with one ordering removed must find a hazard."""
import random

import pytest

# key-tile slots, value-unit slots, staged units per tile (one key tile;
# value: 2 latent halves)
KS, VS, QB, VC = 2, 4, 1, 2
LAG = 1                               # value units of tile g wait for key unit QB (g + 1) + LAG


class Barrier:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.completions, self.tx = name, count, 0, 0, 0

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending += 1
        self._check()

    def complete_tx(self, n):
        self.tx -= n
        self._check()

    def _check(self):
        if self.pending == self.count and self.tx == 0:
            self.pending = 0
            self.completions += 1

    def passes(self, parity):
        return (self.completions & 1) != parity


class Hazard(AssertionError):
    pass


def wait(bar, parity, nth):
    while not bar.passes(parity):
        yield "blocked"
    if bar.completions != nth:
        raise Hazard(f"{bar.name}: {bar.completions} completions, the wait names #{nth}")


def run(items, seed, drop=None, rescale_p=0.3):
    """items: key tiles per item of one pair's range.  drop: name of an
    ordering to leave out (control runs)."""
    rng = random.Random(seed)
    G = sum(items)
    item_of = [n for n, T in enumerate(items) for _ in range(T)]
    first_of, last_of = [], []
    acc = 0
    for T in items:
        first_of.append(acc)
        last_of.append(acc + T - 1)
        acc += T

    class CTA:
        pass

    ctas = [CTA(), CTA()]
    for r, c in enumerate(ctas):
        c.kfull = [Barrier(f"{r}kfull{i}") for i in range(KS)]
        c.kempty = [Barrier(f"{r}kempty{i}") for i in range(KS)]
        c.vready = [Barrier(f"{r}vready{i}", 2) for i in range(VS)]
        c.vempty = [Barrier(f"{r}vempty{i}") for i in range(VS)]
        c.vland = [Barrier(f"{r}vland{i}") for i in range(VS)]
        c.qfull, c.qempty = Barrier(f"{r}qfull"), Barrier(f"{r}qempty")
        c.sfree = [Barrier(f"{r}sfree{i}", 2) for i in range(2)]
        c.pfull = [Barrier(f"{r}pfull{i}", 2) for i in range(2)]
        c.sfull = [Barrier(f"{r}sfull{i}") for i in range(2)]
        c.pfree = [Barrier(f"{r}pfree{i}") for i in range(2)]
        c.o_done = [Barrier(f"{r}o_done{i}") for i in range(2)]
        c.item_done = Barrier(f"{r}item_done")
        c.ep_done = Barrier(f"{r}ep_done", 2)
        c.kslot = [None] * KS            # (tile, chunk) staged, or None
        c.kused = [True] * KS            # its score GEMM chunk has executed
        c.vslot = [None] * VS
        c.vused = [True] * VS
        c.Q = None                       # item whose query rows are staged
        c.q_busy = False                 # query rows still read by pending score GEMMs
        c.P = [None, None]               # tile whose P each buffer holds
        c.P_pending = [False, False]     # value GEMMs of that P not yet executed
        c.S = [None, None]
        c.S_reading = [False, False]     # softmax still reads the buffer
        c.O_item, c.O_last, c.O_chunks = None, -1, 0
        c.ep_reading = False
        c.kiss = 0                       # key chunks requested
    lead = ctas[0]
    tq = []                              # the pair's tensor core queue (in order)
    engine = []                          # loads, landing in any order

    def both(name, i=None):
        return [getattr(c, name) if i is None else getattr(c, name)[i] for c in ctas]

    # ---------------------------------------------------------------- key / query loader
    def kload(r):
        c = ctas[r]
        kc = 0
        for n, T in enumerate(items):
            if n > 0 and drop != "qempty":
                yield from wait(c.qempty, (n - 1) & 1, n)
            if r == 0:
                lead.qfull.arrive(expect_tx=2)
            engine.append(("q", r, n))
            yield "step"
            for k in range(T):
                g = first_of[n] + k
                for ch in range(QB):
                    s = kc % KS
                    if kc >= KS and drop != "kempty":
                        yield from wait(c.kempty[s], ((kc // KS) - 1) & 1, kc // KS)
                    if r == 0:
                        lead.kfull[s].arrive(expect_tx=2)
                    engine.append(("k", r, s, (g, ch)))
                    kc += 1
                    c.kiss = kc
                    yield "step"
        c.kiss = 1 << 30

    # ---------------------------------------------------------------- MMA warp (even CTA)
    def mma():
        haveS, haveO = G > 0, G > 0
        gS = gO = cS = cO = 0
        kc = vc = 0
        nS = nO = 0
        qS = False
        while gO < G:
            progressed = False
            if gO < gS:
                ready = True
                kO = gO - first_of[item_of[gO]]
                if cO == 0:
                    ready = lead.pfull[gO & 1].passes((gO >> 1) & 1)
                    if ready and lead.pfull[gO & 1].completions != (gO >> 1) + 1:
                        raise Hazard("pfull aliasing")
                    if ready and kO == 0 and nO > 0 and drop != "ep_done":
                        ready = lead.ep_done.passes((nO - 1) & 1)
                        if ready and lead.ep_done.completions != nO:
                            raise Hazard("ep_done aliasing")
                vs = vc % VS
                if ready and lead.vready[vs].passes((vc // VS) & 1):
                    if lead.vready[vs].completions != vc // VS + 1:
                        raise Hazard("vready aliasing")
                    tq.append(("PV", gO, cO, vs))
                    tq.append(("commit", both("vempty", vs)))
                    vc += 1
                    cO += 1
                    if cO == VC:
                        cO = 0
                        tq.append(("commit", both("pfree", gO & 1)))
                        tq.append(("commit", both("o_done", gO & 1)))
                        if gO == last_of[item_of[gO]]:
                            tq.append(("commit", both("item_done")))
                            nO += 1
                        gO += 1
                    progressed = True
            if gS < G:
                if not qS:
                    qS = lead.qfull.passes(nS & 1)
                    if qS and lead.qfull.completions != nS + 1:
                        raise Hazard("qfull aliasing")
                ready = qS
                if ready and cS == 0 and gS >= 2:
                    ready = lead.sfree[gS & 1].passes(((gS >> 1) - 1) & 1)
                    if ready and lead.sfree[gS & 1].completions != gS >> 1:
                        raise Hazard("sfree aliasing")
                s = kc % KS
                if ready and lead.kfull[s].passes((kc // KS) & 1):
                    if lead.kfull[s].completions != kc // KS + 1:
                        raise Hazard("kfull aliasing")
                    tq.append(("QK", gS, cS, s))
                    tq.append(("commit", both("kempty", s)))
                    kc += 1
                    cS += 1
                    if cS == QB:
                        cS = 0
                        tq.append(("commit", both("sfull", gS & 1)))
                        if gS == last_of[item_of[gS]]:
                            tq.append(("commit", both("qempty")))
                            qS = False
                            nS += 1
                        gS += 1
                    progressed = True
            yield "step" if progressed else "blocked"

    # ---------------------------------------------------------------- value loader
    def vload(r):
        c = ctas[r]
        req = [(g, ch) for g in range(G) for ch in range(VC)]
        vq = vr = 0
        while vr < len(req):
            progressed = False
            if vq < len(req) and vq < vr + VS:
                g, ch = req[vq]
                vs = vq % VS
                lagged = drop == "lag" or c.kiss >= QB * (g + 1) + LAG
                free = vq < VS or c.vempty[vs].passes(((vq // VS) - 1) & 1)
                if lagged and free:
                    if vq >= VS and c.vempty[vs].completions != vq // VS:
                        raise Hazard("vempty aliasing")
                    c.vland[vs].arrive(expect_tx=1)
                    engine.append(("v", r, vs, (g, ch)))
                    vq += 1
                    progressed = True
            if vr < vq and c.vland[vr % VS].passes((vr // VS) & 1):
                vs = vr % VS
                if c.vland[vs].completions != vr // VS + 1:
                    raise Hazard("vland aliasing")
                if c.vslot[vs] != req[vr]:
                    raise Hazard(f"cta {r}: value slot {vs} holds {c.vslot[vs]}, relay wants {req[vr]}")
                lead.vready[vs].arrive()
                vr += 1
                progressed = True
            yield "step" if progressed else "blocked"

    # ---------------------------------------------------------------- softmax / epilogue
    def softmax(r):
        c = ctas[r]
        g = 0
        for n, T in enumerate(items):
            for k in range(T):
                sb = g & 1
                yield from wait(c.sfull[sb], (g >> 1) & 1, (g >> 1) + 1)
                if c.S[sb] != g:
                    raise Hazard(f"cta {r}: softmax reads score buffer {sb} = {c.S[sb]}, wants {g}")
                c.S_reading[sb] = True
                if drop == "sfree":                      # control: released before the read
                    lead.sfree[sb].arrive()
                yield "step"
                c.S_reading[sb] = False
                if drop != "sfree":
                    lead.sfree[sb].arrive()
                if g >= 2 and drop != "pfree":
                    yield from wait(c.pfree[sb], ((g >> 1) - 1) & 1, g >> 1)
                if k > 0 and rng.random() < rescale_p:
                    yield from wait(c.o_done[(g - 1) & 1], ((g - 1) >> 1) & 1, ((g - 1) >> 1) + 1)
                    if c.O_last != g - 1 or c.O_chunks != VC:
                        raise Hazard(f"cta {r}: rescale at {g} with O through {c.O_last}")
                    yield "step"
                if c.P_pending[sb]:
                    raise Hazard(f"cta {r}: P({g}) overwrites P({c.P[sb]}) before its value GEMMs")
                c.P[sb] = g
                c.P_pending[sb] = True
                yield "step"
                lead.pfull[sb].arrive()
                g += 1
            # epilogue
            yield from wait(c.item_done, n & 1, n + 1)
            c.ep_reading = True
            for _ in range(2):
                if c.O_item != n or c.O_last != last_of[n] or c.O_chunks != VC:
                    raise Hazard(f"cta {r}: epilogue of item {n} finds O of item {c.O_item} through "
                                 f"tile {c.O_last}")
                yield "step"
            c.ep_reading = False
            lead.ep_done.arrive()

    roles = {"mma": mma()}
    for r in range(2):
        roles[f"k{r}"] = kload(r)
        roles[f"v{r}"] = vload(r)
        roles[f"s{r}"] = softmax(r)
    finished, idle = set(), 0
    while len(finished) < len(roles):
        who = rng.choice([x for x in roles if x not in finished] + ["tc", "engine", "engine"])
        progressed = False
        if who == "tc":
            if tq:
                op = tq.pop(0)
                progressed = True
                if op[0] == "QK":
                    _, g, ch, s = op
                    for r, c in enumerate(ctas):
                        if c.kslot[s] != (g, ch):
                            raise Hazard(f"cta {r}: QK({g},{ch}) reads key slot {s} = {c.kslot[s]}")
                        if c.Q != item_of[g]:
                            raise Hazard(f"cta {r}: QK({g}) reads the query rows of item {c.Q}")
                        if c.S_reading[g & 1]:
                            raise Hazard(f"cta {r}: QK({g}) overwrites score buffer {g & 1} under the softmax")
                        c.kused[s] = True
                        if ch == QB - 1:
                            c.S[g & 1] = g
                elif op[0] == "PV":
                    _, g, ch, vs = op
                    for r, c in enumerate(ctas):
                        if c.vslot[vs] != (g, ch):
                            raise Hazard(f"cta {r}: PV({g},{ch}) reads value slot {vs} = {c.vslot[vs]}")
                        if c.P[g & 1] != g:
                            raise Hazard(f"cta {r}: PV({g}) reads P buffer holding {c.P[g & 1]}")
                        c.vused[vs] = True
                        if g == first_of[item_of[g]] and ch == 0:
                            if any(x.ep_reading for x in ctas):
                                raise Hazard(f"PV({g}) overwrites O while an epilogue reads it")
                            c.O_item, c.O_chunks = item_of[g], 0
                        elif ch == 0 and (c.O_last != g - 1 or c.O_chunks != VC):
                            raise Hazard(f"cta {r}: PV({g}) out of order")
                        elif ch > 0 and c.O_chunks != ch:
                            raise Hazard(f"cta {r}: PV({g},{ch}) out of order")
                        c.O_last, c.O_chunks = g, ch + 1
                        if ch == VC - 1:
                            c.P_pending[g & 1] = False
                else:
                    for b in op[1]:
                        b.arrive()
        elif who == "engine":
            if engine:
                ev = engine.pop(rng.randrange(len(engine)))
                progressed = True
                kind, r = ev[0], ev[1]
                c = ctas[r]
                if kind == "q":
                    if c.Q is not None and c.Q != ev[2] - 1:
                        raise Hazard(f"cta {r}: query rows of item {ev[2]} land over item {c.Q}")
                    c.Q = ev[2]
                    lead.qfull.complete_tx(1)
                elif kind == "k":
                    _, _, s, tag = ev
                    if not c.kused[s]:
                        raise Hazard(f"cta {r}: key slot {s} ({c.kslot[s]}) replaced before its GEMM")
                    c.kslot[s], c.kused[s] = tag, False
                    lead.kfull[s].complete_tx(1)
                else:
                    _, _, vs, tag = ev
                    if not c.vused[vs]:
                        raise Hazard(f"cta {r}: value slot {vs} ({c.vslot[vs]}) replaced before its GEMM")
                    c.vslot[vs], c.vused[vs] = tag, False
                    c.vland[vs].complete_tx(1)
        else:
            try:
                progressed = next(roles[who]) != "blocked"
            except StopIteration:
                finished.add(who)
                progressed = True
        idle = 0 if progressed else idle + 1
        if idle > 100000:
            raise Hazard("deadlock")
    # the query rows of the last item are consumed: the check above ran at each load


SHAPES = [(1,), (2,), (1, 1, 1), (3, 1, 2), (5,), (1, 4, 1, 1), (2, 2, 2), (7, 1)]


@pytest.mark.parametrize("items", SHAPES, ids=[str(s) for s in SHAPES])
def test_pair_protocol(items):
    for seed in range(12):
        run(list(items), seed * 17 + len(items))


@pytest.mark.parametrize("drop", ["pfree", "sfree", "qempty", "kempty"])
def test_pair_model_finds_a_missing_ordering(drop):
    """Control: removing one ordering makes the search find a hazard."""
    found = False
    for items in SHAPES:
        for seed in range(12):
            try:
                run(list(items), seed * 17 + len(items), drop=drop)
            except Hazard:
                found = True
                break
        if found:
            break
    assert found, drop


def test_ep_done_is_a_second_guard():
    """With one softmax group per CTA, the P tile of an item's first key tile
    is written after that CTA's epilogue of the previous item, so the value
    GEMM that restarts O already waits for both epilogues through pfull; the
    kernel's ep_done barrier repeats that ordering explicitly."""
    for items in SHAPES:
        for seed in range(6):
            run(list(items), seed * 17 + len(items), drop="ep_done")
