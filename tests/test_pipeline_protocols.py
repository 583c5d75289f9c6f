"""Barrier protocols of the decode kernels, modelled on the CPU.

Every warp role of the GQA/GTA kernel (group_decode.cu: box loads or gathered tiles), of the
latent kernels (latent_decode.cu: the GTA shared-prefix pass; latent_narrow.cu and latent_m128.cu: GLA) and of the MLA CTA-pair kernel
(latent_pair.cu) is a coroutine that waits on and arrives at its mbarriers in the order the
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


def q_in_cta_model(seed, segs, nstage, pair, skip_exchange=False, log=None, no_exchange=False):
    """gla_narrow_kernel (pair=False: four softmax warps) and gla_m128_kernel (pair=True: eight,
    two per TMEM lane quadrant).  The softmax warps write each segment's q themselves: for the
    first segment at its start, for every later one as soon as the previous segment's last score
    product is done; their copies land later (an event) and, with `pair`, each warp also arrives
    once its tensor-memory writes are out.  The MMA warp waits for q before a segment's first
    score product.  With `pair` the two warps of a quadrant exchange their row maxima every tile
    and their row sums at each segment end through two mbarriers of two arrivals, used
    alternately.  With `log`, every softmax warp appends ("read", quadrant, half, tile) when it
    has loaded its scores and ("write", quadrant, half, tile) when it stores P over the S
    buffer."""
    rnd = random.Random(seed)
    events = []
    nsmx = 8 if pair else 4
    c = {"full": [Bar(f"full{s}", 1) for s in range(nstage)],
         "empty": [Bar(f"empty{s}", 1) for s in range(nstage)],
         "sfull": [Bar(f"sfull{s}", 1) for s in range(2)],
         "pfull": [Bar(f"pfull{s}", nsmx) for s in range(2)],
         "qfull": Bar("qfull", 2 * nsmx if pair else nsmx)}
    xbar = [[Bar(f"x{q}{b}", 2) for b in range(2)] for q in range(4)]

    def mma():
        t = 0
        for si, n in enumerate(segs):
            yield from wait(lambda: c["qfull"].ready(si))

            def issue_s(gt):
                yield from wait(lambda: c["full"][gt % nstage].ready(gt // nstage))
                events.append(lambda: c["sfull"][gt % 2].arrive())

            yield from issue_s(t)
            for j in range(n):
                if j + 1 < n:
                    yield from issue_s(t + j + 1)
                yield from wait(lambda: c["pfull"][(t + j) % 2].ready((t + j) // 2))
                st = (t + j) % nstage
                events.append(lambda st=st: c["empty"][st].arrive())
            t += n

    def prod():
        it = 0
        for n in segs:
            for _ in range(n):
                st = it % nstage
                yield from wait(lambda: it < nstage or c["empty"][st].ready(it // nstage - 1))
                c["full"][st].expect_tx(1)
                events.append(lambda st=st: c["full"][st].complete_tx(1))
                it += 1

    def softmax(w):
        q = w % 4
        x = 0
        xx = [0]

        def load_q():
            events.append(lambda: c["qfull"].arrive())  # the copies land
            if pair:
                c["qfull"].arrive()  # the warp's tensor-memory writes are out

        def exchange():
            if no_exchange or (skip_exchange and w == 4 and xx[0] == 1):
                return
            b = xx[0] % 2
            xbar[q][b].arrive()
            k = xx[0] // 2
            yield from wait(lambda: xbar[q][b].ready(k))
            xx[0] += 1

        load_q()
        for si, n in enumerate(segs):
            for j in range(n):
                yield from wait(lambda: c["sfull"][x % 2].ready(x // 2))
                if j == n - 1 and si + 1 < len(segs):
                    load_q()
                if log is not None:
                    log.append(("read", q, w // 4, x))
                    yield
                if pair:
                    yield from exchange() or ()
                if x > 0 and rnd.random() < 0.3:  # lazy rescale: O settled after P.V(x - 1)
                    yield from wait(lambda: c["empty"][(x - 1) % nstage].ready((x - 1) // nstage))
                if log is not None:
                    log.append(("write", q, w // 4, x))
                c["pfull"][x % 2].arrive()
                x += 1
            yield from wait(lambda: c["empty"][(x - 1) % nstage].ready((x - 1) // nstage))  # epilogue
            if pair:
                yield from exchange() or ()

    gens = [prod(), mma()] + [softmax(w) for w in range(nsmx)]
    return schedule(gens, events, rnd, limit=60000 if skip_exchange else 300000)


@pytest.mark.parametrize("pair", [False, True], ids=["narrow", "m128"])
@pytest.mark.parametrize("segs", SEGS)
@pytest.mark.parametrize("nstage", [3, 5])
def test_q_in_cta_protocols_finish_without_parity_aliasing(pair, segs, nstage):
    ALIAS.clear()
    for seed in range(25):
        assert q_in_cta_model(seed, segs, nstage, pair) == "ok", seed
    assert not ALIAS, ALIAS[:5]


def test_m128_p_over_s_follows_the_partners_score_read():
    """In the 128-row kernel the warp of a pair that holds the last 32 scores of a row writes its
    P over S columns [16, 32), which hold scores of the other warp's half: the exchange has to
    order the other warp's read of tile x before this write, in every schedule."""
    for seed in range(40):
        log = []
        assert q_in_cta_model(seed, (3, 1, 4), 3, True, log=log) == "ok", seed
        pos = {e: i for i, e in enumerate(log)}
        for (kind, q, h, x), i in pos.items():
            if kind == "write":
                assert pos[("read", q, 1 - h, x)] < i, (seed, q, h, x)


def test_m128_ordering_check_bites_without_the_exchange():
    """Without the exchange some schedule lets a warp write its P before its partner read."""
    def violated(seed):
        log = []
        assert q_in_cta_model(seed, (3, 1, 4), 3, True, log=log, no_exchange=True) == "ok"
        pos = {e: i for i, e in enumerate(log)}
        return any(kind == "write" and pos[("read", q, 1 - h, x)] > i for (kind, q, h, x), i in pos.items())
    assert any(violated(seed) for seed in range(40))


def test_pair_exchange_model_detects_a_skipped_exchange():
    """One warp of a pair that skips an exchange leaves its partner waiting: the model stalls."""
    assert q_in_cta_model(0, (3, 2), 3, True, skip_exchange=True) == "stuck"


def mla_exchange_abort_model(seed, ntiles, abort_cta, abort_tiles, drain=True):
    """The partial-score exchange of mla_pair_kernel when one CTA gives up early.

    Per CTA, four send warps copy each tile's two halves into the peer (a copy lands later, in
    random order) once the peer has freed the previous tile's half; four softmax warps wait for
    a half, the first of them arms the next phase and records it (xseen), and all free the half.
    In CTA `abort_cta` softmax warp w stops before tile abort_tiles[w] (a bounded wait that ran
    out).  Every wait is bounded: when nothing can move, all waiting warps give up.  Once every
    warp has stopped, copies still in flight stay in flight; then (with `drain`) the teardown
    runs as in the kernel: each CTA completes the bytes of the copies the peer never issued for
    tile xseen[h] and waits for the issued ones, landing copies only while it waits.  Returns the
    copies still in flight when the CTAs would exit and whether a drain wait would have run out."""
    rnd = random.Random(seed)
    events = []
    C = []
    for k in range(2):
        c = {"xfull": [Bar(f"xfull{k}{h}", 1) for h in range(2)],
             "xfree": [Bar(f"xfree{k}{h}", 4) for h in range(2)],
             "sent": [[0, 0] for _ in range(4)], "xseen": [0, 0], "inflight": [0, 0]}
        for h in range(2):
            c["xfull"][h].expect_tx(4)
        C.append(c)
    stop = [False]

    def land(k, h):
        C[k]["inflight"][h] -= 1
        C[k]["xfull"][h].complete_tx(1)

    def send(k, w):
        c, p = C[k], C[k ^ 1]
        for e in range(ntiles):
            for h in range(2):
                while not (e == 0 or c["xfree"][h].ready(e - 1)):
                    if stop[0]:
                        return
                    yield
                p["inflight"][h] += 1
                events.append(lambda h=h: land(k ^ 1, h))
                c["sent"][w][h] += 1

    def softmax(k, w):
        c, p = C[k], C[k ^ 1]
        for x in range(min(abort_tiles[w] if k == abort_cta else ntiles, ntiles)):
            for h in range(2):
                while not c["xfull"][h].ready(x):
                    if stop[0]:
                        return
                    yield
                if w == 0:
                    c["xfull"][h].expect_tx(4)
                    c["xseen"][h] = x + 1
                p["xfree"][h].arrive()

    alive = []
    for k in range(2):
        alive += [send(k, w) for w in range(4)] + [softmax(k, w) for w in range(4)]
    idle = 0
    while alive:
        if events and rnd.random() < 0.4:
            events.pop(rnd.randrange(len(events)))()
            idle = 0
            continue
        i = rnd.randrange(len(alive))
        try:
            next(alive[i])
            idle += 1
        except StopIteration:
            alive.pop(i)
            idle = 0
        if idle > 40 * (len(alive) + 1) and not events:
            stop[0] = True  # nothing can move: every bounded wait runs out
    timed_out = False
    if drain:
        for k in range(2):
            c, p = C[k], C[k ^ 1]
            for h in range(2):
                f = c["xseen"][h]
                n = sum(1 for w in range(4) if p["sent"][w][h] > f)
                if n:
                    if n < 4:
                        c["xfull"][h].complete_tx(4 - n)
                    while not c["xfull"][h].ready(f):
                        if not events:
                            timed_out = True
                            break
                        events.pop(rnd.randrange(len(events)))()
    return [c["inflight"][h] for c in C for h in range(2)], timed_out


def _abort_cases():
    for seed in range(300):
        rnd = random.Random(1000 + seed)
        ntiles = rnd.randint(1, 6)
        base = rnd.randint(0, ntiles)
        yield seed, ntiles, [max(0, min(ntiles, base + rnd.randint(-1, 1))) for _ in range(4)]


@pytest.mark.parametrize("abort_cta", [0, 1])
def test_pair_teardown_drains_the_peers_copies(abort_cta):
    """One CTA of the pair gives up mid-stream (its softmax warps at different tiles); after the
    teardown drain no bulk copy into either CTA's shared memory is still in flight, and no drain
    wait runs out."""
    for seed, ntiles, tiles in _abort_cases():
        inflight, timed_out = mla_exchange_abort_model(seed, ntiles, abort_cta, tiles)
        assert inflight == [0, 0, 0, 0], (seed, ntiles, tiles, inflight)
        assert not timed_out, (seed, ntiles, tiles)


def test_pair_teardown_without_the_drain_can_exit_under_a_copy():
    """The check is not vacuous: without the drain some of the same schedules reach the exit with
    a copy into a CTA's shared memory still in flight."""
    hits = sum(any(mla_exchange_abort_model(seed, ntiles, 0, tiles, drain=False)[0])
               for seed, ntiles, tiles in _abort_cases())
    assert hits > 0
