"""Discrete-event model of the barrier protocol of sparse_attn_fwd_kernel (CPU only).

The attention kernel's roles (scheduler + K producer, Q/V producer, one MMA issuer per
slot, one softmax per slot) are re-enacted here with the same loop
structure, barrier counts and phase counters, over random work items (items without
tiles, items where one slot has no tile, windows shared by both slots, stripe tiles)
and random latencies for the copies, the MMAs, the softmax and the epilogue.  The
tensor pipe executes MMA groups in issue order; a commit completes when every group
issued before it has completed.  Each key tile is processed as two key regions (keys
0-63 and 64-127): per region an S-ready and a P-ready barrier, and one MMA bracket per
region (PV of that region of the previous tile, QK^T of that region of this tile), so
region a's MMAs run while the softmax works on region b.  Slot 1's issuer issues a bracket
only after slot 0's issuer has issued the same one (slot 0 never waits for slot 1).

Checked in every run:
  * no deadlock: every role finishes;
  * every parity wait targets the barrier's current or previous phase, never one that
    has already come round again (a waiter two phases behind would wait forever);
  * a K or V stage is refilled only after every MMA that reads its previous content
    has completed, and a Q buffer only after the last QK^T that reads it;
  * the first PV of an item (which overwrites O) is issued only after the epilogue of
    the slot's previous item has read O.  That epilogue runs after the softmax of the
    slot's first tile of the next item (it is deferred so the tensor pipe gets the next
    item's first P sooner); the issuer waits for it on o_empty;
  * every tile the producers stage is consumed by exactly the slots that list it;
  * when the softmax rescales O (a row max that grows past the lazy threshold), O holds
    exactly the PVs of the regions before the current one: region a waits for this
    tile's region-b QK^T (which follows the previous tile's region-b PV), region b for
    the PV of this tile's region a (pv_a).
The model also shows that releasing a V stage without first observing its fill (the
rule the issuers follow) breaks the phase invariant for runs of tile-less items, and
that each of these planted mistakes is caught: the first PV of an item without the
o_empty wait; a region-b rescale without the pv_a wait; a region-a rescale without
waiting for the tile's region-b QK^T; a K stage released by a plain arrival instead of
a commit after its QK^T; a Q tile loaded without the q_empty wait.
"""

import random

import pytest

from protocol_sim import Engine, ProtocolError

NK, NV, RING = 2, 3, 4


class Sim(Engine):
    def __init__(self, seed, items, release_without_fill=False, broken=""):
        super().__init__(seed)
        self.items = items
        self.release_without_fill = release_without_fill
        self.broken = broken  # a planted protocol mistake (tests only), or ""
        B = self.barrier
        self.item_full = [B(f"item_full{r}", 1) for r in range(RING)]
        self.item_empty = [B(f"item_empty{r}", 1 + 2) for r in range(RING)]  # Q/V producer + 2 softmax
        self.q_full = [B(f"q_full{s}", 1) for s in range(2)]
        self.q_empty = [B(f"q_empty{s}", 1) for s in range(2)]
        self.k_full = [B(f"k_full{i}", 1) for i in range(NK)]
        self.k_empty = [B(f"k_empty{i}", 2) for i in range(NK)]
        self.v_full = [B(f"v_full{i}", 1) for i in range(NV)]
        self.v_empty = [B(f"v_empty{i}", 2) for i in range(NV)]
        self.s_full = [[B(f"s_full{s}{h}", 1) for h in range(2)] for s in range(2)]
        self.p_full = [[B(f"p_full{s}{h}", 1) for h in range(2)] for s in range(2)]
        self.pv_a = [B(f"pv_a{s}", 1) for s in range(2)]
        self.pv_done = [[], []]
        self.lead = 0  # per slot: completion time of the PV of each region, in order
        self.o_full = [B(f"o_full{s}", 1) for s in range(2)]
        self.o_empty = [B(f"o_empty{s}", 1) for s in range(2)]
        self.ring = [None] * RING
        self.kflags = [None] * NK
        self.epi_done = [0, 0]   # epilogues that have read O, per slot
        self.first_pv = [0, 0]   # first PVs of items issued, per slot
        self.k_content, self.v_content = [None] * NK, [None] * NV
        self.consumed = []

    def run(self, limit=10 ** 9):
        super().run({"kprod": k_producer(self), "qvprod": qv_producer(self),
                     "mma0": mma_issuer(self, 0), "mma1": mma_issuer(self, 1),
                     "sm0": softmax(self, 0), "sm1": softmax(self, 1)}, limit)


# ---------------------------------------------------------------------------------------
# Work items and their merged step sequence (the rule of the kernel's steps_next)
# ---------------------------------------------------------------------------------------

def random_item(rng):
    kind = rng.random()
    if kind < 0.15:
        return ([], 0, [], 0)  # no tile at all
    keys = sorted(rng.sample(range(0, 40), rng.randint(0, 10)))
    k0 = [k for k in keys if rng.random() < 0.8]
    k1 = [k for k in keys if rng.random() < 0.8] + [k for k in range(41, 41 + rng.randint(0, 2))]
    ns0 = rng.randint(0, 2)
    ns1 = max(ns0, rng.randint(0, 2))
    if kind < 0.3:
        k0, ns0 = [], 0  # slot 0 without tiles
    return (k0, ns0, k1, ns1)


def steps(item):
    """Merged steps: (tile id or None, flags) with flags {slot: (first, last)}."""
    k0, ns0, k1, ns1 = item
    lists, ns = [list(k0), list(k1)], [ns0, ns1]
    out, started = [], [False, False]
    nb = [len(k0), len(k1)]
    idx = [0, 0]
    while idx[0] < nb[0] or idx[1] < nb[1]:
        key = min(lists[s][idx[s]] for s in range(2) if idx[s] < nb[s])
        fl = {}
        for s in range(2):
            if idx[s] < nb[s] and lists[s][idx[s]] == key:
                first = not started[s]
                started[s] = True
                idx[s] += 1
                fl[s] = (first, idx[s] == nb[s] and ns[s] == 0)
        out.append((("band", key), fl))
    for js in range(max(ns)):
        fl = {}
        for s in range(2):
            if js < ns[s]:
                first = not started[s]
                started[s] = True
                fl[s] = (first, js == ns[s] - 1)
        out.append((("stripe", js), fl))
    if not out:
        out.append((None, {}))  # no-op step
    return out


def tiles_of(item, s):
    k0, ns0, k1, ns1 = item
    keys, ns = (k0, ns0) if s == 0 else (k1, ns1)
    return [("band", k) for k in keys] + [("stripe", j) for j in range(ns)]


# ---------------------------------------------------------------------------------------
# Roles
# ---------------------------------------------------------------------------------------

def k_producer(sim):
    tk = 0
    for m, item in enumerate(sim.items + [None]):
        slot = m % RING
        if m >= RING:
            yield ("wait", sim.item_empty[slot], m // RING - 1)
        sim.ring[slot] = item
        sim.item_full[slot].arrive()
        if item is None:
            break
        for tile, fl in steps(item):
            si = tk % NK
            if tk >= NK:
                yield ("wait", sim.k_empty[si], tk // NK - 1)
            sim.kflags[si] = (tile, fl, False)
            if tile is None:
                sim.k_full[si].arrive()
            else:
                sim.k_content[si] = tile
                sim.tma(sim.k_full[si], f"K{si}")
            tk += 1
            yield ("delay", sim.rng.randint(1, 400))  # issue cost of a step
    si = tk % NK
    if tk >= NK:
        yield ("wait", sim.k_empty[si], tk // NK - 1)
    sim.kflags[si] = (None, {}, True)
    sim.k_full[si].arrive()


def qv_producer(sim):
    tv, qn = 0, [0, 0]
    m = 0
    while True:
        slot = m % RING
        yield ("wait", sim.item_full[slot], m // RING)
        item = sim.ring[slot]
        sim.item_empty[slot].arrive()
        m += 1
        if item is None:
            return
        for tile, fl in steps(item):
            # the Q tile of a slot is loaded at the slot's first step of the item, so
            # the V tiles of steps before it never wait on the slot's previous item
            for s in sorted(fl):
                if not fl[s][0]:
                    continue
                if qn[s] >= 1 and sim.broken != "no_q_empty_wait":
                    yield ("wait", sim.q_empty[s], qn[s] - 1)
                sim.tma(sim.q_full[s], f"Q{s}")
                qn[s] += 1
            si = tv % NV
            if tv >= NV:
                yield ("wait", sim.v_empty[si], tv // NV - 1)
            if tile is None:
                sim.v_full[si].arrive()
            else:
                sim.v_content[si] = tile
                sim.tma(sim.v_full[si], f"V{si}")
            tv += 1
            yield ("delay", sim.rng.randint(1, 400))  # issue cost of a step


def mma_issuer(sim, s):
    u, qcnt, pcnt, ocnt = 0, 0, 0, 0
    pend = pfirst = plast = False
    ptile = None
    while True:
        v = u - 1
        tile, fl, end, inn = None, {}, False, False
        for h in range(2):
            if h == 0 and u >= 1 and not (sim.release_without_fill and not pend):
                yield ("wait", sim.v_full[v % NV], v // NV)
            if pend:
                yield ("wait", sim.p_full[s][h], pcnt)
                if h == 0 and pfirst and ocnt >= 1 and sim.broken != "no_o_empty_wait":
                    yield ("wait", sim.o_empty[s], ocnt - 1)
            if h == 0:
                yield ("wait", sim.k_full[u % NK], u // NK)
                tile, fl, end = sim.kflags[u % NK]
                inn = (not end) and s in fl
                if inn and fl[s][0]:
                    yield ("wait", sim.q_full[s], qcnt)
            if s == 1:
                while sim.lead < 2 * u + h + 1:
                    yield ("delay", 5)
            if pend:
                if h == 0 and pfirst:
                    if sim.first_pv[s] > sim.epi_done[s]:
                        raise ProtocolError(f"slot {s}: first PV of an item before the epilogue read O")
                    sim.first_pv[s] += 1
                    ocnt += 1
                if sim.v_content[v % NV] != ptile:
                    raise ProtocolError(f"slot {s}: PV reads {sim.v_content[v % NV]}, wants {ptile}")
                sim.pv_done[s].append(sim.mma(256, [f"V{v % NV}"]))
                if h == 0:
                    sim.commit(sim.pv_a[s])
            if inn:
                if sim.k_content[u % NK] != tile:
                    raise ProtocolError(f"slot {s}: QK reads {sim.k_content[u % NK]}, wants {tile}")
                if h == 0:
                    sim.consumed.append((s, tile))
                sim.mma(400, [f"K{u % NK}", f"Q{s}"])
            if s == 0:
                sim.lead = 2 * u + h + 1
            if inn:
                sim.commit(sim.s_full[s][h])
            if h == 1:
                if pend:
                    if plast:
                        sim.commit(sim.o_full[s])
                    sim.commit(sim.v_empty[v % NV])
                    pcnt += 1
                elif u >= 1:
                    sim.v_empty[v % NV].arrive()
                if inn:
                    if fl[s][1]:
                        sim.commit(sim.q_empty[s])
                    if sim.broken == "k_release_by_arrival":
                        sim.k_empty[u % NK].arrive()
                    else:
                        sim.commit(sim.k_empty[u % NK])
                    if fl[s][0]:
                        qcnt += 1
                elif not end:
                    sim.k_empty[u % NK].arrive()
            yield ("delay", sim.rng.randint(1, 50))
        if end:
            return
        pend = inn
        if inn:
            pfirst, plast, ptile = fl[s][0], fl[s][1], tile
        u += 1


def softmax(sim, s):
    m, tcnt, icnt = 0, 0, 0
    owed = False  # the epilogue of the slot's last item with tiles is still to do

    def epilogue():
        nonlocal icnt
        yield ("wait", sim.o_full[s], icnt)
        icnt += 1
        yield ("delay", sim.rng.randint(100, 600))  # O read from tensor memory
        sim.epi_done[s] += 1
        sim.o_empty[s].arrive()
        yield ("delay", sim.rng.randint(100, 1500))  # normalise and store

    while True:
        slot = m % RING
        yield ("wait", sim.item_full[slot], m // RING)
        item = sim.ring[slot]
        sim.item_empty[slot].arrive()
        m += 1
        if item is None:
            break
        n = len(tiles_of(item, s))
        if n == 0:
            continue
        for j in range(n):
            for h in range(2):
                yield ("wait", sim.s_full[s][h], tcnt)
                yield ("delay", sim.rng.randint(400, 1500))
                if j > 0 and sim.rng.random() < 0.2:
                    # O rescale: O must hold exactly the PVs of the regions before this one
                    if h == 0:
                        if sim.broken != "no_region_b_wait":
                            yield ("wait", sim.s_full[s][1], tcnt)
                    elif sim.broken != "no_pv_a_wait":
                        yield ("wait", sim.pv_a[s], tcnt)
                    region = 2 * tcnt + h
                    done = sim.pv_done[s]
                    if len(done) != region or (done and done[-1] > sim.t):
                        raise ProtocolError(f"slot {s}: O rescaled at region {region} with "
                                            f"{len(done)} PVs issued")
                    yield ("delay", sim.rng.randint(100, 400))
                sim.p_full[s][h].arrive()
                if j == 0 and h == 0 and owed:
                    yield from epilogue()
                    owed = False
            tcnt += 1
        owed = True
    if owed:
        yield from epilogue()


def _items(seed, n):
    rng = random.Random(seed)
    items = [random_item(rng) for _ in range(n)]
    if seed % 3 == 0:  # long runs of items without tiles, as at the end of a schedule
        items += [([], 0, [], 0)] * rng.randint(5, 20)
    return items


@pytest.mark.parametrize("seed", range(40))
def test_protocol_random_schedules(seed):
    items = _items(seed, 30)
    sim = Sim(seed, items)
    sim.run()
    # every tile was consumed by exactly the slots that list it, in order
    want = [(s, t) for it in items for t, fl in steps(it) for s in sorted(fl)]
    assert sorted(sim.consumed, key=str) == sorted(want, key=str)


def test_release_without_observed_fill_breaks_phases():
    # Releasing a V stage that no slot reads without first observing its fill lets the
    # releases of a run of no-op steps race ahead of the producer.
    broken = 0
    for seed in range(40):
        items = [([], 0, [], 0)] * 12 + [([1, 2], 0, [1, 2, 3], 1)] + [([], 0, [], 0)] * 12
        sim = Sim(seed, items, release_without_fill=True)
        try:
            sim.run()
        except ProtocolError:
            broken += 1
    assert broken > 0


@pytest.mark.parametrize("broken", ["no_o_empty_wait", "no_pv_a_wait", "no_region_b_wait",
                                    "k_release_by_arrival", "no_q_empty_wait"])
def test_planted_protocol_mistakes_are_caught(broken):
    caught = 0
    for seed in range(40):
        try:
            Sim(seed, _items(seed, 30), broken=broken).run()
        except ProtocolError:
            caught += 1
    assert caught > 0
