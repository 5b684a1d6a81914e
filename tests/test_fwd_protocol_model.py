"""A model of the forward kernel's mbarrier protocol, run under random schedules.

The model mirrors the hand-offs of `fa_fwd_kernel` (exact_attention_151_b200/csrc/
fa_fwd_kernel.cuh), not its arithmetic:
  * the loader warp: Q once, then for every ring item u the K tile and the V tile,
    each into stage u % S after the stage's previous item has been released;
  * the MMA warp, in the order S0(j), PV1(j-1), S1(j), PV0(j), with the commits
    that release K/V stages, publish S_i and mark the last PV_i; each PV waits
    for V before P, and unpaired the warp waits for V item j and polls K item
    j+1 before PV0(j)'s P wait, then skips the waits those already satisfied;
  * two softmax warpgroups of four warps, each warp arriving on the two halves of
    P_i (the kernel's barriers count 128 thread arrivals; here, 4 warp arrivals).
Items are one key tile shared by both query tiles (unpaired), or, paired (packed
heads with split-KV), alternating tile 0 / tile 1 items while both have tiles.

Checked at every step: a waiter is never more than one phase behind the barrier
it polls (a parity wait would misread it); a stage is reloaded only after every
MMA reading its previous item has completed; an MMA reads the item it expects,
and only after the MMA warp itself has seen that item's full barrier complete;
S_i(j) is issued only after PV_i(j-1) and after all four warps read S_i(j-1);
PV reads P only once all four warps wrote it; and the run ends (no deadlock).
Completions (TMA, commits) arrive at random times, commits in issue order.
A model that missed protocol bugs would prove nothing, so planted bugs must fail.
"""

import random

import pytest


class ProtocolError(Exception):
    pass


class _Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1


def simulate(last0, last1, pair, stages, seed, split0=False, split1=False, plant=None):
    # stages: K and V ring depths, (kstages, vstages), or one int for both
    ks, vs = stages if isinstance(stages, tuple) else (stages, stages)
    depth = {"K": ks, "V": vs}
    rng = random.Random(seed)
    n_kv = max(last0, last1) + 1
    n_items = (last0 + 1) + (last1 + 1) if pair else n_kv

    def item_of(i, j):
        if not pair:
            return j
        if plant == "item_order":
            return 2 * j + i if j < last1 else last1 + 1 + j
        return 2 * j + i if j <= last1 else last1 + 1 + j

    bars = {"Q": _Bar(1)}
    for kind in "KV":
        for s in range(depth[kind]):
            for name in ("F", "E"):
                bars[f"{kind}{name}{s}"] = _Bar(1)
    for i in range(2):
        bars[f"SF{i}"], bars[f"OF{i}"] = _Bar(1), _Bar(1)
        for h in range(2):
            bars[f"PF{i}{h}"] = _Bar(4)
    slot = {"K": [None] * ks, "V": [None] * vs}
    landed = {"K": [False] * ks, "V": [False] * vs}
    events, mmas, done, readers = [], [], set(), {}
    s_read, p_written, pv_issued = {}, {}, set()

    def ready(name, k):
        b = bars[name]
        if b.phase not in (k, k + 1):
            raise ProtocolError(f"{name}: waiting for phase {k} while at {b.phase}")
        return b.phase > k

    def mma(kind, u):
        mid = len(mmas)
        mmas.append(mid)
        readers.setdefault((kind, u), []).append(mid)

    def commit(name):
        events.append(("commit", name, len(mmas)))

    def loader():
        events.append(("q",))
        for u in range(n_items):
            for kind in "KV":
                n = depth[kind]
                s = u % n
                if u >= n:
                    while not ready(f"{kind}E{s}", u // n - 1):
                        yield
                    if any(m not in done for m in readers.get((kind, u - n), [])):
                        raise ProtocolError(f"{kind} stage {s} reloaded while item {u - n} is read")
                slot[kind][s], landed[kind][s] = u, False
                events.append(("tma", kind, s))
                yield

    def mma_warp():
        while not ready("Q", 0):
            yield
        seen = set()  # (kind, item) whose full barrier this warp has seen complete

        def observe(kind, u):
            ok = ready(f"{kind}F{u % depth[kind]}", u // depth[kind])
            if ok:
                seen.add((kind, u))
            return ok

        def wait_k(u):
            while not observe("K", u):
                yield

        def issue_s(i, j):
            u = item_of(i, j)
            s = u % ks
            if slot["K"][s] != u or not landed["K"][s] or ("K", u) not in seen:
                raise ProtocolError(f"S{i}({j}) reads K stage {s} without having seen item {u} land")
            if j > 0 and ((i, j - 1) not in pv_issued or not s_read.get((i, j - 1))):
                raise ProtocolError(f"S{i}({j}) overwrites S/P of tile {j - 1} too early")
            for _ in range(8):
                mma("K", u)
            commit(f"SF{i}")

        def issue_pv(i, j, split, need_v):
            u = item_of(i, j)
            s = u % vs
            if need_v:  # V first, then the halves of P
                while not observe("V", u):
                    yield
            for h in range(2):
                while not ready(f"PF{i}{h}", j):
                    yield
                if not p_written.get((i, j, h)):
                    raise ProtocolError(f"PV{i}({j}) half {h} before P was written")
                if slot["V"][s] != u or not landed["V"][s] or ("V", u) not in seen:
                    raise ProtocolError(f"PV{i}({j}) reads V stage {s} without having seen item {u} land")
                for _ in range(8 if split else 4):
                    mma("V", u)
                yield
            pv_issued.add((i, j))

        k_seen = False  # unpaired: K item j+1 polled ready before PV0(j)'s P wait
        for j in range(n_kv + 1):
            if j < n_kv and (j <= last0 or not pair):
                u = item_of(0, j)
                if not k_seen:
                    yield from wait_k(u)
                k_seen = False
                if j <= last0:
                    issue_s(0, j)
                if pair and u + ks < n_items:
                    commit(f"KE{u % ks}")
                yield
            if 1 <= j and j - 1 <= last1:
                u = item_of(1, j - 1)
                # unpaired: PV0(j-1) observed V item j-1 unless j-1 > last0
                need_v = pair or j - 1 > last0 or plant == "always_skip_v"
                if plant == "always_skip_v" and not pair:
                    need_v = False
                yield from issue_pv(1, j - 1, split1 and j == 1, need_v)
                if j - 1 == last1:
                    commit("OF1")
                if u + vs < n_items:
                    commit(f"VE{u % vs}")
            if j < n_kv:
                if j <= last1:
                    u = item_of(1, j)
                    if pair and plant != "skip_k_wait":
                        yield from wait_k(u)
                    issue_s(1, j)
                    if pair and u + ks < n_items:
                        commit(f"KE{u % ks}")
                if not pair and j + ks < n_kv:
                    commit(f"KE{j % ks}")
                if j <= last0:
                    u = item_of(0, j)
                    if not pair:
                        # V item j, then one poll of K item j+1, before the P wait
                        while not observe("V", u):
                            yield
                        if j + 1 < n_kv:
                            k_seen = observe("K", j + 1)
                            if plant == "k_probe_stage":
                                k_seen = True  # a poll taken as satisfied without looking
                        yield
                    yield from issue_pv(0, j, split0 and j == 0, pair)
                    if j == last0:
                        commit("OF0")
                    if (pair or j > last1) and u + vs < n_items and plant != "late_v_release":
                        commit(f"VE{u % vs}")
                    elif plant == "late_v_release" and j > last1 and u + vs < n_items:
                        commit(f"VE{u % vs}")
            yield

    def softmax_warp(i, w):
        last = last0 if i == 0 else last1
        for j in range(last + 1):
            while not ready(f"SF{i}", j):
                yield
            s_read[(i, j, w)] = True
            s_read[(i, j)] = all(s_read.get((i, j, x)) for x in range(4))
            yield
            for h in range(2):
                p_written[(i, j, h, w)] = True
                p_written[(i, j, h)] = all(p_written.get((i, j, h, x)) for x in range(4))
                bars[f"PF{i}{h}"].arrive()
                yield
        if last >= 0:
            while not ready(f"OF{i}", 0):
                yield

    actors = {"loader": loader(), "mma": mma_warp()}
    for i in range(2):
        for w in range(4):
            actors[f"softmax{i}.{w}"] = softmax_warp(i, w)
    for _ in range(400000):
        if not actors and not events:
            return
        names = list(actors) + (["event"] if events else [])
        pick = rng.choice(names)
        if pick == "event":
            ev = rng.choice(events)
            if ev[0] == "commit":  # a thread's commits complete in issue order
                ev = next(e for e in events if e[0] == "commit")
            events.remove(ev)
            if ev[0] == "commit":
                done.update(range(ev[2]))
                bars[ev[1]].arrive()
            elif ev[0] == "tma":
                landed[ev[1]][ev[2]] = True
                bars[f"{ev[1]}F{ev[2]}"].arrive()
            else:
                bars["Q"].arrive()
            continue
        try:
            next(actors[pick])
        except StopIteration:
            del actors[pick]
    raise ProtocolError("no progress: deadlock")


def _cases(n, seed0):
    out = []
    for seed in range(seed0, seed0 + n):
        r = random.Random(seed)
        # K / V ring depths: the kernel's at D = 128 and D = 64, and asymmetric rings
        stages = r.choice([(2, 2), (2, 3), (3, 2), (4, 4), (6, 6)])
        if r.random() < 0.5:
            t = r.randint(1, 8)  # tiles per key range
            out.append((t - 1, r.choice([-1, r.randint(0, t - 1), t - 1]), True, stages, seed, False, False))
        else:
            n_kt = r.randint(1, 9)
            last0, last1 = r.choice([(n_kt - 1, n_kt - 1), (n_kt - 2, n_kt - 1), (n_kt - 1, -1)])
            out.append((last0, last1, False, stages, seed, r.random() < 0.3, r.random() < 0.3))
    return out


def test_protocol_model_random_schedules():
    for case in _cases(600, 0):
        simulate(*case)


@pytest.mark.parametrize("plant", ["item_order", "skip_k_wait", "late_v_release"])
def test_protocol_model_catches_planted_bugs(plant):
    with pytest.raises(ProtocolError):
        for case in _cases(600, 0):
            if case[2]:  # paired cases exercise all three plants
                simulate(*case, plant=plant)


@pytest.mark.parametrize("plant", ["always_skip_v", "k_probe_stage"])
def test_protocol_model_catches_planted_unpaired_bugs(plant):
    """Unpaired plants: PV1 skipping its V wait also where PV0 did not observe
    that item (query tile 0 ends a tile earlier), and the K poll's result taken
    as ready without looking."""
    with pytest.raises(ProtocolError):
        for case in _cases(600, 0):
            if not case[2]:
                simulate(*case, plant=plant)
