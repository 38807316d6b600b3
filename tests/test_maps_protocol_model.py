"""Discrete-event model of the barrier protocol of attn_maps_kernel (CPU only).

The roles of the averaged-maps kernel are re-enacted with its loop structure, barrier
counts and phase counters: the TMA producer (one Q block + K chunk per tile into NS
stages), the MMA issuer (four S buffers in tensor memory), and sixteen softmax warps
in four column parts of four warps.  A persistent CTA walks a random list of items
(row blocks of 1 to 4 chunks, 1 to 4 samples), with random latencies for the copies,
the MMAs, the softmax work and the map stores.

Checked in every run:
  * no deadlock, and every parity wait within one phase (protocol_sim);
  * a stage is refilled only after the MMA reading it has completed, and each MMA
    reads the tile it expects;
  * an S buffer is overwritten only after all sixteen warps have loaded it, and every
    warp loads the tile it expects;
  * at each sample's exchange part 0 reads the slots of that sample from every warp
    (none stale, none already overwritten by a later sample);
  * pass 2 reads the (m_b, 1 / l_b) part 0 wrote for the same item and sample;
  * a part's staging buffer is written only when no store is reading it, and each
    store sends one chunk written by all four warps of the part.
The model also shows that each of these protocol mistakes is caught: a single exchange
buffer (not double-buffered by sample parity) lets a part overwrite its slot before
part 0 has read it; without the stat_ready wait pass 2 reads statistics part 0 has not
written; without the stg_free wait a part rewrites its staging buffer while the store
reads it; an s_empty barrier that completes one warp early lets the issuer overwrite an
S buffer that a warp has not loaded.
"""

import random

import pytest

from protocol_sim import Engine, ProtocolError

NSB, PARTS, WPP = 4, 4, 4  # S buffers, column parts, warps per part
NWARP = PARTS * WPP


def tile(t, nc, B):
    """(pass2, b, c) of tile t of an item, as the kernel's m_tile."""
    n1 = nc * B
    if t < n1:
        return False, t // nc, t % nc
    u = t - n1
    return True, u % B, u // B


class MapsSim(Engine):
    def __init__(self, seed, items, B, nrb, NS, single_xch=False, broken=""):
        super().__init__(seed)
        self.items, self.B, self.nrb, self.NS = items, B, nrb, NS
        self.single_xch = single_xch
        self.broken = broken  # a planted protocol mistake (tests only), or ""
        b_ = self.barrier
        self.full = [b_(f"full{i}", 1) for i in range(NS)]
        self.empty = [b_(f"empty{i}", 1) for i in range(NS)]
        self.s_full = [b_(f"s_full{i}", 1) for i in range(NSB)]
        self.s_empty = [b_(f"s_empty{i}", NWARP - (broken == "short_s_empty")) for i in range(NSB)]
        self.xch = [b_(f"xch{i}", NWARP) for i in range(2)]
        self.stat_ready = b_("stat_ready", WPP)
        self.stg_full = [b_(f"stg_full{h}", WPP) for h in range(PARTS)]
        self.stg_free = [b_(f"stg_free{h}", 1) for h in range(PARTS)]
        self.stage = [None] * NS        # tile number staged in each stage
        self.sbuf = [None] * NSB        # tile number in each S buffer
        self.sbuf_loaded = [NWARP] * NSB
        self.xslot = {}                 # (parity, warp) -> (item, b)
        self.stat = {}                  # (b, quarter) -> item
        self.staging = {}               # (part, quarter) -> chunk id
        self.stg_reading = [False] * PARTS
        self.stores = []

    def tiles(self):
        return sum(2 * (rb + 1) * self.B for rb in self.items)

    def run(self, limit=10 ** 9):
        agents = {"prod": producer(self), "mma": issuer(self)}
        for w in range(NWARP):
            agents[f"sm{w}"] = softmax_warp(self, w)
        super().run(agents, limit)


def producer(sim):
    g = 0
    for rb in sim.items:
        for t in range(2 * (rb + 1) * sim.B):
            st = g % sim.NS
            if g >= sim.NS:
                yield ("wait", sim.empty[st], g // sim.NS - 1)
            sim.stage[st] = g
            sim.tma(sim.full[st], f"stage{st}")
            g += 1
            yield ("delay", sim.rng.randint(1, 60))


def issuer(sim):
    for g in range(sim.tiles()):
        st, sb = g % sim.NS, g % NSB
        yield ("wait", sim.full[st], g // sim.NS)
        if g >= NSB:
            yield ("wait", sim.s_empty[sb], g // NSB - 1)
        if sim.sbuf_loaded[sb] != NWARP:
            raise ProtocolError(f"S buffer {sb} overwritten by tile {g} after {sim.sbuf_loaded[sb]} loads")
        if sim.stage[st] != g:
            raise ProtocolError(f"tile {g} reads stage {st} holding tile {sim.stage[st]}")
        sim.mma(sim.rng.randint(100, 400), [f"stage{st}"])
        sim.sbuf[sb], sim.sbuf_loaded[sb] = g, 0
        sim.commit(sim.s_full[sb])
        sim.commit(sim.empty[st])
        yield ("delay", sim.rng.randint(1, 40))


def softmax_warp(sim, w):
    h, q = divmod(w, WPP)  # part and quarter (rows 32 q .. 32 q + 31)
    leader = q == 0
    B = sim.B
    g = gb = ne = 0

    def put_chunk(chunk):
        nonlocal ne
        if ne >= 1 and sim.broken != "no_stg_free_wait":
            yield ("wait", sim.stg_free[h], ne - 1)
        if sim.stg_reading[h]:
            raise ProtocolError(f"part {h}: staging written while a store reads it")
        sim.staging[(h, q)] = chunk
        sim.stg_full[h].arrive()
        if leader:
            yield ("wait", sim.stg_full[h], ne)
            got = {sim.staging.get((h, k)) for k in range(WPP)}
            if got != {chunk}:
                raise ProtocolError(f"part {h}: store of {chunk} sends {got}")
            sim.stg_reading[h] = True
            sim.stores.append((h, chunk))
            yield ("delay", sim.rng.randint(50, 800))  # the store reads shared memory
            sim.stg_reading[h] = False
            sim.stg_free[h].arrive()
        ne += 1

    for gi, rb in enumerate(sim.items):
        nc = rb + 1
        T = 2 * nc * B
        for t in range(T):
            pass2, b, c = tile(t, nc, B)
            sb = g % NSB
            if pass2 and t == nc * B and sim.broken != "no_stat_ready_wait":
                yield ("wait", sim.stat_ready, gi)
            yield ("wait", sim.s_full[sb], g // NSB)
            if sim.sbuf[sb] != g:
                raise ProtocolError(f"warp {w} loads tile {sim.sbuf[sb]} for tile {g}")
            sim.sbuf_loaded[sb] += 1
            sim.s_empty[sb].arrive()
            yield ("delay", sim.rng.randint(200, 1500))
            if not pass2 and c == nc - 1:
                par = 0 if sim.single_xch else gb & 1
                sim.xslot[(par, w)] = (gi, b)
                sim.xch[gb & 1].arrive()
                yield ("wait", sim.xch[gb & 1], gb // 2)
                if h == 0:
                    # part 0's warps may be scheduled late after the wait completes
                    yield ("delay", sim.rng.randint(0, 3000))
                    seen = {sim.xslot[(par, k)] for k in range(NWARP)}
                    if seen != {(gi, b)}:
                        raise ProtocolError(f"exchange of item {gi} sample {b} reads {seen}")
                    yield ("delay", sim.rng.randint(1, 100))
                    sim.stat[(b, q)] = gi
                    if b == B - 1:
                        sim.stat_ready.arrive()
                gb += 1
            if pass2:
                if sim.stat.get((b, q)) != gi:
                    raise ProtocolError(f"warp {w}: stat of sample {b} is from item {sim.stat.get((b, q))}, "
                                        f"not {gi}")
                if b == B - 1:
                    yield from put_chunk((gi, c))
            g += 1
        for cc in range(nc, sim.nrb):
            yield from put_chunk((gi, cc))


def _case(seed):
    rng = random.Random(seed)
    nrb = rng.randint(1, 4)
    B = rng.choice([1, 1, 2, 3, 4])
    items = [rng.randrange(nrb) for _ in range(rng.randint(1, 6))]
    NS = rng.choice([2, 3])
    return items, B, nrb, NS


@pytest.mark.parametrize("seed", range(40))
def test_maps_protocol_random_items(seed):
    items, B, nrb, NS = _case(seed)
    sim = MapsSim(seed, items, B, nrb, NS)
    sim.run()
    # every part stored every chunk of every item exactly once
    want = sorted((h, (gi, c)) for h in range(PARTS) for gi in range(len(items)) for c in range(nrb))
    assert sorted(sim.stores) == want


def test_single_exchange_buffer_breaks():
    broken = 0
    for seed in range(40):
        items, B, nrb, NS = _case(seed)
        try:
            MapsSim(seed, items, max(B, 2), nrb, NS, single_xch=True).run()
        except ProtocolError:
            broken += 1
    assert broken > 0


@pytest.mark.parametrize("broken", ["no_stat_ready_wait", "no_stg_free_wait", "short_s_empty"])
def test_planted_protocol_mistakes_are_caught(broken):
    caught = 0
    for seed in range(40):
        items, B, nrb, NS = _case(seed)
        try:
            MapsSim(seed, items, B, nrb, NS, broken=broken).run()
        except ProtocolError:
            caught += 1
    assert caught > 0
