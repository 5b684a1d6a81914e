"""Models of the backward kernels' mbarrier protocols, run under random schedules.

They mirror the hand-offs of the persistent `fa_bwd_dkdv_kernel` and
`fa_bwd_dq_kernel` (exact_attention_151_b200/csrc/fa_bwd_kernel.cuh), not their
arithmetic. A CTA has a loader warp, an MMA warp issuing in the kernel's order,
and two compute warpgroups (one per 64-column half of every score tile) of four
warps; the kernels' 128-thread arrivals are four warp arrivals here (256-thread
ones eight). The CTA works through a sequence of items (the scheduler's choice
does not matter to the protocol), each with its own number of streamed tiles,
zero included (an item whose gradients are zero: no loads, no products).

Items: the loader publishes each into a two-slot ring (ItemFull / ItemEmpty,
read by the MMA warp and the eight compute warps) and ends with -1. Ring
stages, score buffers and the phases of every barrier are counted across
items. The fixed operands of an item (dK/dV: K and V; dQ: Q and dO) are
reloaded once the previous item's last products reading them have completed
(XEmpty); the accumulators are reused once the compute warps have read the
previous item's out (AccEmpty).

dK/dV: per item, the MMA warp issues S^T(0) and dP^T(0), then per tile t:
dV += P^T dO per half (after that half's phase A), S^T(t+1) over the P^T
columns, dK += dS^T Q per half (after phase B), the stage release, and dP^T(t+1)
over the dS^T columns (or the item's final commit). At D = 64 (TMEM has room)
two S^T buffers: S^T(0) and S^T(1) up front, and S^T(t+2) right after
dP^T(t+1), into the buffer dV(t) has just read, with a three-stage ring; the
phase-A barriers are then per buffer too (with one, a warpgroup can finish
phase A of two tiles before the MMA warp waits for the first: two phases
ahead, which a parity wait misreads; planted as "db_one_a").

dQ: K_t into a 3-stage ring, V_t into a 2-stage ring. Per item the MMA warp
issues S(0), dP(0), S(1), then per tile t: after both warpgroups' phase B,
releases V_t, issues dP(t+1), dQ += dS(t) K_t, releases K_t, and issues S(t+2)
into the buffer of S(t).

Checked: no waiter more than one phase behind; nothing in TMEM or shared memory
(stages, fixed operands, item slots, accumulators) overwritten before its last
reader has finished; readers find what they expect; no deadlock. Planted bugs
must fail, or the models would prove nothing.
"""

import random

import pytest

from tests.protocol_sim import Model, ProtocolError

STAGES_DKDV = 2
K_STAGES_DQ, V_STAGES_DQ = 3, 2
ITEM_READERS = 9  # the MMA warp and the eight compute warps


class ItemRing:
    """The two-slot work-item ring: the loader publishes, nine warps read."""

    def __init__(self, m, seq, plant):
        self.m, self.seq, self.plant = m, seq, plant
        self.slots = [None, None]
        self.unread = [0, 0]
        for s in range(2):
            m.bar(f"IF{s}")
            m.bar(f"IE{s}", ITEM_READERS)

    def publish(self, i):
        slot = i & 1
        if i >= 2 and self.plant != "slot_early":
            yield from self.m.wait(f"IE{slot}", (i >> 1) - 1)
        if self.unread[slot]:
            raise ProtocolError(f"item slot {slot} overwritten before every warp read item {i - 2}")
        self.slots[slot] = (i, self.seq[i])
        self.unread[slot] = ITEM_READERS
        self.m.bars[f"IF{slot}"].arrive()

    def take(self, i):
        slot = i & 1
        yield from self.m.wait(f"IF{slot}", i >> 1)
        idx, n = self.slots[slot]
        if idx != i:
            raise ProtocolError(f"a warp expecting item {i} read item {idx}")
        self.unread[slot] -= 1
        self.m.bars[f"IE{slot}"].arrive()
        return n


def simulate_dkdv(items, seed, plant=None, db=False):
    """items: streamed-tile counts of the CTA's items, in order (0: no work).
    db: the D = 64 form, with two S^T buffers (one score barrier each) and a
    three-stage ring; S^T(t+2) is issued right after dP^T(t+1), into the buffer
    whose P^T dV(t) has just read."""
    m = Model(seed)
    seq = list(items) + [-1]
    ring = ItemRing(m, seq, plant)
    n_stages = 3 if db else STAGES_DKDV
    n_sbuf = 2 if db else 1
    for name in ("X", "XE", "DPF", "Done", "Drain"):
        m.bar(name)
    for b in range(n_sbuf):
        m.bar(f"SF{b}")
    m.bar("AccE", 8)
    for s in range(n_stages):
        m.bar(f"YF{s}")
        m.bar(f"YE{s}")
    for h in range(2):
        for b in range(n_sbuf):  # double-buffered: one phase-A barrier per S^T buffer
            m.bar(f"A{b}{h}", 4)
        m.bar(f"B{h}", 4)
    stage = [None] * n_stages   # global streamed tile held
    landed = [False] * n_stages
    xbuf = {"item": None, "landed": False}
    readers = {}     # ("Y", g) / ("X", xi) -> MMA ids reading it
    ws_users = {}    # g -> warps still reading the stage's -LSE / -D rows
    s_cols = [{"T": None} for _ in range(n_sbuf)]
    dp_cols = {"T": None}
    wrote_p, wrote_ds = {}, {}
    acc = {"item": None, "last": -1, "read": {}}  # item accumulating; last MMA id into it; warps that read item xi
    state = {}

    def busy(key):
        return any(i >= m.done for i in readers.get(key, []))

    def loader():
        yc = xi = 0
        for i, n in enumerate(seq):
            yield from ring.publish(i)
            yield
            if n < 0:
                return
            if n == 0:
                continue
            if xi > 0 and plant != "x_early":
                yield from m.wait("XE", xi - 1)
            if busy(("X", xi - 1)):
                raise ProtocolError(f"K, V of item {xi} loaded while item {xi - 1}'s products read theirs")
            xbuf["item"], xbuf["landed"] = xi, False

            def land_x(xi=xi):
                xbuf["landed"] = True
                m.bars["X"].arrive()
            m.later(land_x)
            xi += 1
            for _ in range(n):
                s = yc % n_stages
                if yc >= n_stages:
                    yield from m.wait(f"YE{s}", yc // n_stages - 1)
                    if busy(("Y", yc - n_stages)):
                        raise ProtocolError(f"stage {s} reloaded while an MMA reads tile {yc - n_stages}")
                    if ws_users.get(yc - n_stages):
                        raise ProtocolError(f"stage {s} reloaded while a warp reads tile {yc - n_stages}'s rows")
                stage[s], landed[s] = yc, False

                def land(s=s):
                    landed[s] = True
                    m.bars[f"YF{s}"].arrive()
                m.later(land)
                yc += 1
                yield

    def score(cols, g, T, xi, what):
        s = g % n_stages
        if stage[s] != g or not landed[s]:
            raise ProtocolError(f"{what}({T}) reads a stage without tile {g}")
        if xbuf["item"] != xi or not xbuf["landed"]:
            raise ProtocolError(f"{what}({T}) reads K, V without item {xi}'s")
        if cols["T"] is not None:
            prev = cols["T"]
            if not state.get((what, prev, "read")):
                raise ProtocolError(f"{what}({T}) overwrites {what}({prev}) before both warpgroups read it")
            # P^T (dS^T) of tile prev sits in these columns until the dV (dK)
            # MMAs that read it are issued; one thread's MMAs run in order
            reader = "dV" if what == "S" else "dK"
            if not (state.get((reader, prev, 0)) and state.get((reader, prev, 1))):
                raise ProtocolError(f"{what}({T}) overwrites the operand of {reader}({prev}) before it is issued")
        ids = [m.mma() for _ in range(8)]
        readers.setdefault(("Y", g), []).extend(ids)
        readers.setdefault(("X", xi), []).extend(ids)
        cols["T"] = T

    def issue_s(g, T, xi):
        b = T % n_sbuf
        score(s_cols[b], g, T, xi, "S")
        m.commit(f"SF{b}")

    def accumulate(g, T, h, kind, xi, first):
        if not (wrote_p if kind == "dV" else wrote_ds).get((T, h)):
            raise ProtocolError(f"{kind}({T}) half {h} before its operand was written")
        if first and xi > 0 and acc["read"].get(xi - 1, 0) < 8:
            raise ProtocolError(f"item {xi}'s first {kind} overwrites item {xi - 1}'s accumulators before they are read")
        ids = [m.mma() for _ in range(4)]
        readers.setdefault(("Y", g), []).extend(ids)
        acc["item"], acc["last"] = xi, ids[-1]
        state[(kind, T, h)] = True

    def mma_warp():
        yc = tc = xi = 0
        for i in range(len(seq)):
            n = yield from ring.take(i)
            if n < 0:
                return
            if n == 0:
                continue
            yield from m.wait("X", xi)
            yield from m.wait(f"YF{yc % n_stages}", yc // n_stages)
            issue_s(yc, tc, xi)
            score(dp_cols, yc, tc, xi, "dP")
            m.commit("DPF")
            if n == 1:
                m.commit("XE")
            if db and n > 1:
                yield from m.wait(f"YF{(yc + 1) % n_stages}", (yc + 1) // n_stages)
                issue_s(yc + 1, tc + 1, xi)
            yield
            for t in range(n):
                g, T = yc + t, tc + t
                s = g % n_stages
                more = t + 1 < n
                if db and plant == "db_s_early" and t + 2 < n:
                    yield from m.wait(f"YF{(g + 2) % n_stages}", (g + 2) // n_stages)
                    issue_s(g + 2, T + 2, xi)  # before dV(t) has read P^T(t) from that buffer
                for h in range(2):
                    a_k = T // n_sbuf if plant != "db_one_a" else T
                    yield from m.wait(f"A{T % n_sbuf if plant != 'db_one_a' else 0}{h}", a_k)
                    if t == 0 and h == 0 and xi > 0:
                        yield from m.wait("AccE", xi - 1)
                    accumulate(g, T, h, "dV", xi, t == 0 and h == 0)
                    yield
                if more and not db:
                    yield from m.wait(f"YF{(g + 1) % n_stages}", (g + 1) // n_stages)
                    issue_s(g + 1, T + 1, xi)
                for h in range(2):
                    yield from m.wait(f"B{h}", T)
                    accumulate(g, T, h, "dK", xi, False)
                    yield
                if plant != "early_release":
                    m.commit(f"YE{s}")
                if more:
                    score(dp_cols, g + 1, T + 1, xi, "dP")
                    m.commit("DPF")
                    if t + 1 == n - 1 or (plant == "xe_early" and t + 2 == n - 1):
                        m.commit("XE")
                    if db and plant != "db_s_early" and t + 2 < n:
                        yield from m.wait(f"YF{(g + 2) % n_stages}", (g + 2) // n_stages)
                        issue_s(g + 2, T + 2, xi)
                else:
                    m.commit("Done")
                if plant == "early_release" and t + 1 < n:
                    m.commit(f"YE{(g + 1) % n_stages}")
                yield
            yc += n
            tc += n
            xi += 1

    def warp(h, w):
        yc = tc = xi = 0
        i = 0
        n = yield from ring.take(0)
        while n >= 0:
            for t in range(n):
                g, T = yc + t, tc + t
                s = g % n_stages
                b = T % n_sbuf
                yield from m.wait(f"YF{s}", g // n_stages)
                ws_users[g] = ws_users.get(g, 0) + 1
                k = T // n_sbuf
                yield from m.wait(f"SF{b}", k if plant != "sf_parity" else k + 1)
                if stage[s] != g or s_cols[b]["T"] != T:
                    raise ProtocolError("warp reads a stage or S^T without its tile")
                state[(h, w, "S", T)] = True
                if all(state.get((hh, ww, "S", T)) for hh in range(2) for ww in range(4)):
                    state[("S", T, "read")] = True
                yield
                state[(h, w, "P", T)] = True
                wrote_p[(T, h)] = all(state.get((h, ww, "P", T)) for ww in range(4))
                m.bars[f"A{b if plant != 'db_one_a' else 0}{h}"].arrive()
                yield
                yield from m.wait("DPF", T)
                if dp_cols["T"] != T:
                    raise ProtocolError("warp reads dP^T without its tile")
                state[(h, w, "dP", T)] = True
                if all(state.get((hh, ww, "dP", T)) for hh in range(2) for ww in range(4)):
                    state[("dP", T, "read")] = True
                yield
                wrote_ds[(T, h)] = all(state.get((h, ww, "dP", T)) for ww in range(4))
                ws_users[g] -= 1
                m.bars[f"B{h}"].arrive()
                yield
            nxt = yield from ring.take(i + 1)
            if n > 0:
                yield from m.wait("Done", xi)
                if acc["item"] != xi or acc["last"] >= m.done:
                    raise ProtocolError(f"warp reads item {xi}'s accumulators before its last product finished")
                acc["read"][xi] = acc["read"].get(xi, 0) + 1
                m.bars["AccE"].arrive()
                xi += 1
                yield
            yc += n
            tc += n
            n = nxt
            i += 1

    actors = {"loader": loader(), "mma": mma_warp()}
    for h in range(2):
        for w in range(4):
            actors[f"wg{h}.{w}"] = warp(h, w)
    m.run(actors)


def simulate_dq(items, seed, plant=None):
    """items: key-tile counts of the CTA's items, in order (0: no work)."""
    m = Model(seed)
    seq = list(items) + [-1]
    ring = ItemRing(m, seq, plant)
    for name in ("X", "XE", "SF0", "SF1", "DPF", "Done"):
        m.bar(name)
    m.bar("AccE", 8)
    for s in range(K_STAGES_DQ):
        m.bar(f"KF{s}")
        m.bar(f"KE{s}")
    for s in range(V_STAGES_DQ):
        m.bar(f"VF{s}")
        m.bar(f"VE{s}")
    for h in range(2):
        m.bar(f"B{h}", 4)
    rings = {"K": [None] * K_STAGES_DQ, "V": [None] * V_STAGES_DQ}
    landed = {"K": [False] * K_STAGES_DQ, "V": [False] * V_STAGES_DQ}
    xbuf = {"item": None, "landed": False}
    readers = {}
    sbuf = [None, None]  # global score tile held by S buffer 0 / 1
    dp = {"T": None}
    acc = {"item": None, "last": -1, "read": {}}
    state = {}

    def busy(key):
        return any(i >= m.done for i in readers.get(key, []))

    def loader():
        cnt = {"K": 0, "V": 0}
        xi = 0
        for i, n in enumerate(seq):
            yield from ring.publish(i)
            yield
            if n < 0:
                return
            if n == 0:
                continue
            if xi > 0 and plant != "x_early":
                yield from m.wait("XE", xi - 1)
            if busy(("X", xi - 1)):
                raise ProtocolError(f"Q, dO of item {xi} loaded while item {xi - 1}'s products read theirs")
            xbuf["item"], xbuf["landed"] = xi, False

            def land_x():
                xbuf["landed"] = True
                m.bars["X"].arrive()
            m.later(land_x)
            xi += 1
            for _ in range(n):
                for kind, ns in (("K", K_STAGES_DQ), ("V", V_STAGES_DQ)):
                    g = cnt[kind]
                    s = g % ns
                    if g >= ns:
                        yield from m.wait(f"{kind}E{s}", g // ns - 1)
                        if busy((kind, g - ns)):
                            raise ProtocolError(f"{kind} stage {s} reloaded while tile {g - ns} is read")
                    rings[kind][s], landed[kind][s] = g, False

                    def land(kind=kind, s=s):
                        landed[kind][s] = True
                        m.bars[f"{kind}F{s}"].arrive()
                    m.later(land)
                    cnt[kind] += 1
                    yield

    def use(kind, g, ns, xi=None):
        s = g % ns
        if rings[kind][s] != g or not landed[kind][s]:
            raise ProtocolError(f"MMA reads {kind} stage {s} without tile {g}")
        ids = [m.mma() for _ in range(8)]
        readers.setdefault((kind, g), []).extend(ids)
        if xi is not None:
            if xbuf["item"] != xi or not xbuf["landed"]:
                raise ProtocolError(f"MMA reads Q, dO without item {xi}'s")
            readers.setdefault(("X", xi), []).extend(ids)
        return ids

    def mma_warp():
        kc = vc = tc = xi = 0

        def issue_s(t):
            T = tc + t
            b = T & 1
            if sbuf[b] is not None:
                prev = sbuf[b]
                if not state.get(("dS", prev, "written")) or not state.get(("dQ", prev)):
                    raise ProtocolError(f"S({T}) overwrites buffer {b} before dQ({prev}) is issued")
            use("K", kc + t, K_STAGES_DQ, xi)
            sbuf[b] = T
            m.commit(f"SF{b}")

        def issue_dp(t):
            T = tc + t
            if dp["T"] is not None and not state.get(("dS", dp["T"], "written")):
                raise ProtocolError(f"dP({T}) overwrites dP({dp['T']}) before both warpgroups read it")
            use("V", vc + t, V_STAGES_DQ, xi)
            dp["T"] = T
            m.commit("DPF")

        for i in range(len(seq)):
            n = yield from ring.take(i)
            if n < 0:
                return
            if n == 0:
                continue
            yield from m.wait("X", xi)
            yield from m.wait(f"KF{kc % K_STAGES_DQ}", kc // K_STAGES_DQ)
            issue_s(0)
            yield from m.wait(f"VF{vc % V_STAGES_DQ}", vc // V_STAGES_DQ)
            issue_dp(0)
            if n == 1:
                m.commit("XE")
            if n > 1:
                yield from m.wait(f"KF{(kc + 1) % K_STAGES_DQ}", (kc + 1) // K_STAGES_DQ)
                issue_s(1)
            yield
            for t in range(n):
                T = tc + t
                for h in range(2):
                    yield from m.wait(f"B{h}", T)
                state[("dS", T, "written")] = True
                m.commit(f"VE{(vc + t) % V_STAGES_DQ}")
                if t + 1 < n:
                    u = vc + t + 1
                    yield from m.wait(f"VF{u % V_STAGES_DQ}", u // V_STAGES_DQ)
                    issue_dp(t + 1)
                    if t + 1 == n - 1 and plant != "xe_early":
                        m.commit("XE")
                if t == 0 and xi > 0:
                    yield from m.wait("AccE", xi - 1)
                if t == 0 and xi > 0 and acc["read"].get(xi - 1, 0) < 8:
                    raise ProtocolError(f"item {xi}'s first dQ overwrites item {xi - 1}'s before it is read")
                if plant != "s_before_dq":
                    ids = use("K", kc + t, K_STAGES_DQ)  # dQ += dS(t) K_t
                    acc["item"], acc["last"] = xi, ids[-1]
                    state[("dQ", T)] = True
                    m.commit(f"KE{(kc + t) % K_STAGES_DQ}")
                if t + 2 < n:
                    u = kc + t + 2
                    yield from m.wait(f"KF{u % K_STAGES_DQ}", u // K_STAGES_DQ)
                    issue_s(t + 2)
                if plant == "s_before_dq":
                    ids = use("K", kc + t, K_STAGES_DQ)
                    acc["item"], acc["last"] = xi, ids[-1]
                    state[("dQ", T)] = True
                    m.commit(f"KE{(kc + t) % K_STAGES_DQ}")
                if plant == "xe_early" and t + 2 == n - 1:
                    m.commit("XE")  # before S(n-1) and dP(n-1) are issued
                if t == n - 1:
                    m.commit("Done")
                yield
            kc += n
            vc += n
            tc += n
            xi += 1

    def warp(h, w):
        tc = xi = 0
        i = 0
        n = yield from ring.take(0)
        while n >= 0:
            for t in range(n):
                T = tc + t
                b = T & 1
                yield from m.wait(f"SF{b}", T >> 1)
                if sbuf[b] != T:
                    raise ProtocolError("warp reads an S buffer without its tile")
                yield
                yield from m.wait("DPF", T if plant != "dp_parity" else T + 1)
                if dp["T"] != T:
                    raise ProtocolError("warp reads dP without its tile")
                yield
                m.bars[f"B{h}"].arrive()
                yield
            nxt = yield from ring.take(i + 1)
            if n > 0:
                yield from m.wait("Done", xi)
                if acc["item"] != xi or acc["last"] >= m.done:
                    raise ProtocolError(f"warp reads item {xi}'s dQ before its last product finished")
                acc["read"][xi] = acc["read"].get(xi, 0) + 1
                m.bars["AccE"].arrive()
                xi += 1
                yield
            tc += n
            n = nxt
            i += 1

    actors = {"loader": loader(), "mma": mma_warp()}
    for h in range(2):
        for w in range(4):
            actors[f"wg{h}.{w}"] = warp(h, w)
    m.run(actors)


def _item_lists(n, seed0, max_items=6, max_tiles=7, zero_frac=0.2):
    r = random.Random(seed0)
    out = []
    for i in range(n):
        k = r.randint(1, max_items)
        out.append(([0 if r.random() < zero_frac else r.randint(1, max_tiles) for _ in range(k)], seed0 + i))
    return out


def _planted_lists(plant, seed0):
    """Item sequences that give a planted bug room to show: the item ring can
    only run ahead through items without work; the rest need several tiles."""
    if plant == "slot_early":
        return [([0] * 4 + items, seed) for items, seed in _item_lists(300, seed0, zero_frac=0.6)]
    return [([max(n, 3) for n in items] + [3], seed) for items, seed in _item_lists(300, seed0, zero_frac=0.0)]


def test_dkdv_protocol_model_random_schedules():
    for items, seed in _item_lists(400, 0):
        simulate_dkdv(items, seed)


def test_dkdv_double_buffered_protocol_model_random_schedules():
    for items, seed in _item_lists(400, 500):
        simulate_dkdv(items, seed, db=True)


def test_dq_protocol_model_random_schedules():
    for items, seed in _item_lists(400, 1000):
        simulate_dq(items, seed)


def test_single_items_and_edge_sequences():
    for items in ([1], [2], [0], [0, 0], [1, 1, 1, 1], [0, 3, 0, 1], [9], [1, 9, 1], [2, 2, 3]):
        for seed in range(20):
            simulate_dkdv(items, seed)
            simulate_dkdv(items, seed, db=True)
            simulate_dq(items, seed)


@pytest.mark.parametrize("plant", ["early_release", "x_early", "xe_early", "slot_early", "sf_parity"])
def test_dkdv_protocol_model_catches_planted_bugs(plant):
    with pytest.raises(ProtocolError):
        for items, seed in _planted_lists(plant, 0):
            simulate_dkdv(items, seed, plant=plant)


@pytest.mark.parametrize("plant", ["early_release", "x_early", "xe_early", "slot_early", "sf_parity", "db_s_early",
                                   "db_one_a"])
def test_dkdv_double_buffered_protocol_model_catches_planted_bugs(plant):
    with pytest.raises(ProtocolError):
        for items, seed in _planted_lists(plant, 700):
            simulate_dkdv(items, seed, plant=plant, db=True)


@pytest.mark.parametrize("plant", ["s_before_dq", "dp_parity", "x_early", "xe_early", "slot_early"])
def test_dq_protocol_model_catches_planted_bugs(plant):
    with pytest.raises(ProtocolError):
        for items, seed in _planted_lists(plant, 1000):
            simulate_dq(items, seed, plant=plant)
