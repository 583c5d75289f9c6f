"""Barrier protocols of the decode kernels, modelled on the CPU.

Every warp role of the GQA/GTA kernel (group_decode.cu: box loads or gathered tiles), of the
GLA kernel (latent_decode.cu) and of the MLA CTA-pair kernel (latent_pair.cu) is a coroutine that waits on and arrives at its mbarriers in the order the
kernel does; TMA copies, bulk copies to the peer CTA and tcgen05.commit arrivals complete later,
in random order.  Random schedules over several segment patterns and stage counts must all
finish (no stall), and no wait may find its barrier two or more phases past the phase it waits
for: the kernels wait on a phase's parity, which cannot tell those apart.  (The kernels' waits
are bounded as well; this shows that the bound is never what ends them.)"""
import random

import pytest

ALIAS = []


class Bar:
    """An mbarrier: `count` arrivals plus a transaction count complete a phase."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.done = name, count, count, 0, 0

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def arrive(self):
        assert self.pending >= 1, (self.name, "more arrivals than the count")
        self.pending -= 1
        self._check()

    def expect_tx(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        self._check()

    def ready(self, k):
        """Phase k has completed (the kernel tests the parity k & 1)."""
        if self.done >= k + 2:
            ALIAS.append((self.name, k, self.done))
        return self.done > k


def wait(cond):
    while not cond():
        yield


def schedule(gens, events, rnd, limit=300000):
    alive = list(gens)
    for _ in range(limit):
        if not alive and not events:
            return "ok"
        if events and (not alive or rnd.random() < 0.5):
            events.pop(rnd.randrange(len(events)))()
            continue
        i = rnd.randrange(len(alive))
        try:
            next(alive[i])
        except StopIteration:
            alive.pop(i)
    return "stuck"


def mma_issuer(c, segs, nstage, events):
    """The MMA warp (both kernels): S(j + 1) is issued before P.V(j); qempty after the last S."""
    t = 0
    for si, n in enumerate(segs):
        yield from wait(lambda: c["qfull"].ready(si))
        yield from wait(lambda: c["qtm"].ready(si))

        def issue_s(gt):
            yield from wait(lambda: c["full"][gt % nstage].ready(gt // nstage))
            events.append(lambda: c["sfull"][gt % 2].arrive())

        yield from issue_s(t)
        if n == 1:
            events.append(lambda: c["qempty"].arrive())
        for j in range(n):
            if j + 1 < n:
                yield from issue_s(t + j + 1)
                if j + 1 == n - 1:
                    events.append(lambda: c["qempty"].arrive())
            yield from wait(lambda: c["pfull"][(t + j) % 2].ready((t + j) // 2))
            st = (t + j) % nstage
            events.append(lambda st=st: c["empty"][st].arrive())
        t += n


def producer(c, segs, nstage, events):
    it = 0
    for si, n in enumerate(segs):
        yield from wait(lambda: si == 0 or c["qempty"].ready(si - 1))
        c["qfull"].expect_tx(1)
        events.append(lambda: c["qfull"].complete_tx(1))
        for _ in range(n):
            st = it % nstage
            yield from wait(lambda: it < nstage or c["empty"][st].ready(it // nstage - 1))
            c["full"][st].expect_tx(1)
            events.append(lambda st=st: c["full"][st].complete_tx(1))
            it += 1


def common_bars(k, nstage, pfull_count):
    return {"full": [Bar(f"full{k}{s}", 1) for s in range(nstage)],
            "empty": [Bar(f"empty{k}{s}", 1) for s in range(nstage)],
            "sfull": [Bar(f"sfull{k}{s}", 1) for s in range(2)],
            "pfull": [Bar(f"pfull{k}{s}", pfull_count) for s in range(2)],
            "qfull": Bar(f"qfull{k}", 1), "qtm": Bar(f"qtm{k}", 4), "qempty": Bar(f"qempty{k}", 1)}


def gla_model(seed, segs, nstage):
    """latent_decode_kernel: warps 4..7 write q, run the softmax and write P over S."""
    rnd = random.Random(seed)
    events = []
    c = common_bars(0, nstage, 4)

    def softmax():
        x = 0
        for si, n in enumerate(segs):
            yield from wait(lambda: si == 0 or c["qempty"].ready(si - 1))
            c["qtm"].arrive()
            for _ in range(n):
                yield from wait(lambda: c["sfull"][x % 2].ready(x // 2))
                if x > 0 and rnd.random() < 0.3:  # lazy rescale: O settled after P.V(x - 1)
                    yield from wait(lambda: c["empty"][(x - 1) % nstage].ready((x - 1) // nstage))
                c["pfull"][x % 2].arrive()
                x += 1
            yield from wait(lambda: c["empty"][(x - 1) % nstage].ready((x - 1) // nstage))  # epilogue

    gens = [producer(c, segs, nstage, events), mma_issuer(c, segs, nstage, events)] + [softmax() for _ in range(4)]
    return schedule(gens, events, rnd)


def mla_pair_model(seed, segs, nstage):
    """mla_pair_kernel: per CTA warps 0..3 write q and send the partial S (two 32-token halves,
    one bulk copy per warp each), warps 4..7 add the peer's halves, run the softmax and write P
    over S once the send warps have read it."""
    rnd = random.Random(seed)
    events = []
    C = []
    for k in range(2):
        c = common_bars(k, nstage, 4)
        c["sread"] = [Bar(f"sread{k}{s}", 4) for s in range(2)]
        c["xfull"] = [Bar(f"xfull{k}{h}", 1) for h in range(2)]
        c["xfree"] = [Bar(f"xfree{k}{h}", 4) for h in range(2)]
        for h in range(2):
            c["xfull"][h].expect_tx(4)  # armed for the first tile: four 4 KB copies
        C.append(c)

    def send(k):
        c, p = C[k], C[k ^ 1]
        e = 0
        for si, n in enumerate(segs):
            yield from wait(lambda: si == 0 or c["qempty"].ready(si - 1))
            c["qtm"].arrive()
            for _ in range(n):
                yield from wait(lambda: c["sfull"][e % 2].ready(e // 2))
                c["sread"][e % 2].arrive()
                for h in range(2):
                    yield from wait(lambda: e == 0 or c["xfree"][h].ready(e - 1))
                    events.append(lambda h=h: p["xfull"][h].complete_tx(1))
                e += 1

    def softmax(k, first):
        c, p = C[k], C[k ^ 1]
        x = 0
        for si, n in enumerate(segs):
            for _ in range(n):
                yield from wait(lambda: c["sfull"][x % 2].ready(x // 2))
                for h in range(2):
                    yield from wait(lambda: c["xfull"][h].ready(x))
                    if first:
                        c["xfull"][h].expect_tx(4)
                    p["xfree"][h].arrive()
                if x > 0 and rnd.random() < 0.3:
                    yield from wait(lambda: c["empty"][(x - 1) % nstage].ready((x - 1) // nstage))
                yield from wait(lambda: c["sread"][x % 2].ready(x // 2))
                c["pfull"][x % 2].arrive()
                x += 1
            yield from wait(lambda: c["empty"][(x - 1) % nstage].ready((x - 1) // nstage))

    gens = []
    for k in range(2):
        gens += [producer(C[k], segs, nstage, events), mma_issuer(C[k], segs, nstage, events)]
        gens += [send(k) for _ in range(4)] + [softmax(k, w == 0) for w in range(4)]
    return schedule(gens, events, rnd)


def group_model(seed, segs, nstage, gpc=8, gather_warps=0):
    """group_decode_kernel: one producer warp (or `gather_warps` warps whose every lane arrives
    once its copies land) fills an n-stage ring; each of the gpc consumer warps frees a stage
    after its MMAs on it."""
    rnd = random.Random(seed)
    events = []
    full_count = 32 * gather_warps if gather_warps else 1
    full = [Bar(f"full{s}", full_count) for s in range(nstage)]
    empty = [Bar(f"empty{s}", gpc) for s in range(nstage)]
    ntiles = sum(segs)

    def box_producer():
        for it in range(ntiles):
            st = it % nstage
            yield from wait(lambda: it < nstage or empty[st].ready(it // nstage - 1))
            full[st].expect_tx(1)
            events.append(lambda st=st: full[st].complete_tx(1))

    def gather_producer():
        for it in range(ntiles):
            st = it % nstage
            yield from wait(lambda: it < nstage or empty[st].ready(it // nstage - 1))
            for _ in range(32):  # every lane's cp.async arrive fires when its copies land
                events.append(lambda st=st: full[st].arrive())

    def consumer():
        for it in range(ntiles):
            yield from wait(lambda: full[it % nstage].ready(it // nstage))
            empty[it % nstage].arrive()

    prods = [gather_producer() for _ in range(gather_warps)] if gather_warps else [box_producer()]
    return schedule(prods + [consumer() for _ in range(gpc)], events, rnd)


SEGS = [(3, 1, 4), (1, 1, 1, 1), (7,), (2, 5), (1, 9, 1)]


@pytest.mark.parametrize("gather_warps", [0, 4])
@pytest.mark.parametrize("nstage", [2, 3])
def test_group_protocol_finishes_without_parity_aliasing(gather_warps, nstage):
    ALIAS.clear()
    for seed in range(25):
        assert group_model(seed, (5, 2, 6), nstage, gather_warps=gather_warps) == "ok", seed
    assert not ALIAS, ALIAS[:5]


@pytest.mark.parametrize("model", [gla_model, mla_pair_model], ids=["gla", "mla_pair"])
@pytest.mark.parametrize("segs", SEGS)
@pytest.mark.parametrize("nstage", [2, 4])
def test_protocol_finishes_without_parity_aliasing(model, segs, nstage):
    ALIAS.clear()
    for seed in range(25):
        assert model(seed, segs, nstage) == "ok", seed
    assert not ALIAS, ALIAS[:5]


def test_model_detects_a_missing_arrival():
    """The model itself is not vacuous: with one softmax warp fewer than the P barrier counts,
    the GLA pipeline must stall."""
    def short(seed, segs, nstage):
        rnd = random.Random(seed)
        events = []
        c = common_bars(0, nstage, 5)  # five arrivals expected, four softmax warps

        def softmax():
            x = 0
            for si, n in enumerate(segs):
                yield from wait(lambda: si == 0 or c["qempty"].ready(si - 1))
                c["qtm"].arrive()
                for _ in range(n):
                    yield from wait(lambda: c["sfull"][x % 2].ready(x // 2))
                    c["pfull"][x % 2].arrive()
                    x += 1

        gens = [producer(c, segs, nstage, events), mma_issuer(c, segs, nstage, events)] + [softmax() for _ in range(4)]
        return schedule(gens, events, rnd, limit=20000)

    assert short(0, (3,), 2) == "stuck"
