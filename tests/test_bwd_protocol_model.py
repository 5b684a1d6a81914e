"""Models of the backward kernels' mbarrier protocols, run under random schedules.

They mirror the hand-offs of `fa_bwd_dkdv_kernel` and `fa_bwd_dq_kernel`
(exact_attention_151_b200/csrc/fa_bwd_kernel.cuh), not their arithmetic. Each has
a loader warp, an MMA warp issuing in the kernel's order, and two compute
warpgroups (one per 64-column half of every score tile) of four warps; the
kernels' 128-thread arrivals are four warp arrivals here.

dK/dV (one key tile, n query tiles t): the loader brings K, V once and, per t,
Q_t, dO_t and the -LSE / -D rows into stage t % 2. The MMA warp issues S^T(0) and
dP^T(0), then per t: dV += P^T dO per half (after that half's phase A), S^T(t+1)
over the P^T columns, dK += dS^T Q per half (after phase B), the stage release,
and dP^T(t+1) over the dS^T columns (or the final commit). A warpgroup waits for
the stage and S^T(t), runs phase A (P^T in place), then waits for dP^T(t) and
runs phase B (dS^T in place, reading the stage's -D row).

dQ (one query tile, n key tiles t): K_t into a 3-stage ring, V_t into a 2-stage
ring. The MMA warp issues S(0) (buffer 0), dP(0), S(1) (buffer 1), then per t:
after both warpgroups' phase B, releases V_t, issues dP(t+1), dQ += dS(t) K_t
(A = dS in S buffer t % 2), releases K_t, and issues S(t+2) into buffer t % 2.

Checked: no waiter more than one phase behind; nothing in TMEM or shared memory
overwritten before its last reader has finished; readers find what they expect;
no deadlock. Planted bugs must fail, or the models would prove nothing.
"""

import random

import pytest

from tests.protocol_sim import Model, ProtocolError

STAGES_DKDV = 2
K_STAGES_DQ, V_STAGES_DQ = 3, 2


def simulate_dkdv(n_t, seed, plant=None):
    m = Model(seed)
    m.bar("X")
    for s in range(STAGES_DKDV):
        m.bar(f"YF{s}")
        m.bar(f"YE{s}")
    for name in ("SF", "DPF", "Done"):
        m.bar(name)
    for h in range(2):
        m.bar(f"A{h}", 4)
        m.bar(f"B{h}", 4)
    stage = [None] * STAGES_DKDV
    landed = [False] * STAGES_DKDV
    readers = {}  # stage item t -> MMA ids reading it
    ws_users = {}  # stage item t -> warps still reading its -LSE / -D rows
    s_cols, dp_cols = {"t": None}, {"t": None}
    wrote_p, wrote_ds = {}, {}
    state = {}

    def loader():
        m.later(lambda: m.bars["X"].arrive())
        for t in range(n_t):
            s = t % STAGES_DKDV
            if t >= STAGES_DKDV:
                yield from m.wait(f"YE{s}", t // STAGES_DKDV - 1)
                if any(i >= m.done for i in readers.get(t - STAGES_DKDV, [])):
                    raise ProtocolError(f"stage {s} reloaded while an MMA reads tile {t - STAGES_DKDV}")
                if ws_users.get(t - STAGES_DKDV):
                    raise ProtocolError(f"stage {s} reloaded while a warp reads tile {t - STAGES_DKDV}'s rows")
            stage[s], landed[s] = t, False

            def land(s=s):
                landed[s] = True
                m.bars[f"YF{s}"].arrive()
            m.later(land)
            yield

    def score(cols, t, what):
        s = t % STAGES_DKDV
        if stage[s] != t or not landed[s]:
            raise ProtocolError(f"{what}({t}) reads a stage without tile {t}")
        if cols["t"] is not None:
            prev = cols["t"]
            if not state.get((what, prev, "read")):
                raise ProtocolError(f"{what}({t}) overwrites {what}({prev}) before both warpgroups read it")
            # P^T (dS^T) of tile prev sits in these columns until the dV (dK) MMAs
            # that read it are issued; one thread's MMAs run in order
            reader = "dV" if what == "S" else "dK"
            if not (state.get((reader, prev, 0)) and state.get((reader, prev, 1))):
                raise ProtocolError(f"{what}({t}) overwrites the operand of {reader}({prev}) before it is issued")
        ids = [m.mma() for _ in range(8)]
        readers.setdefault(t, []).extend(ids)
        cols["t"] = t

    def acc(t, h, kind):
        if not (wrote_p if kind == "dV" else wrote_ds).get((t, h)):
            raise ProtocolError(f"{kind}({t}) half {h} before its operand was written")
        ids = [m.mma() for _ in range(4)]
        readers.setdefault(t, []).extend(ids)
        state[(kind, t, h)] = True

    def mma_warp():
        yield from m.wait("X", 0)
        yield from m.wait("YF0", 0)
        score(s_cols, 0, "S")
        m.commit("SF")
        score(dp_cols, 0, "dP")
        m.commit("DPF")
        yield
        for t in range(n_t):
            s = t % STAGES_DKDV
            more = t + 1 < n_t
            if more and plant == "s_over_p":
                yield from m.wait(f"YF{(t + 1) % STAGES_DKDV}", (t + 1) // STAGES_DKDV)
                score(s_cols, t + 1, "S")
                m.commit("SF")
            for h in range(2):
                yield from m.wait(f"A{h}", t)
                acc(t, h, "dV")
                yield
            if more and plant != "s_over_p":
                yield from m.wait(f"YF{(t + 1) % STAGES_DKDV}", (t + 1) // STAGES_DKDV)
                score(s_cols, t + 1, "S")
                m.commit("SF")
            for h in range(2):
                yield from m.wait(f"B{h}", t)
                acc(t, h, "dK")
                yield
            if t + STAGES_DKDV < n_t and plant != "early_release":
                m.commit(f"YE{s}")
            if more:
                score(dp_cols, t + 1, "dP")
                m.commit("DPF")
            else:
                m.commit("Done")
            if plant == "early_release" and t + 1 + STAGES_DKDV < n_t:
                m.commit(f"YE{(t + 1) % STAGES_DKDV}")
            yield

    def warp(h, w):
        for t in range(n_t):
            s = t % STAGES_DKDV
            yield from m.wait(f"YF{s}", t // STAGES_DKDV)
            ws_users[t] = ws_users.get(t, 0) + 1
            yield from m.wait("SF", t)
            if stage[s] != t:
                raise ProtocolError("warp reads a stage without its tile")
            state[(h, w, "S", t)] = True
            if all(state.get((hh, ww, "S", t)) for hh in range(2) for ww in range(4)):
                state[("S", t, "read")] = True
            yield
            state[(h, w, "P", t)] = True
            wrote_p[(t, h)] = all(state.get((h, ww, "P", t)) for ww in range(4))
            m.bars[f"A{h}"].arrive()
            yield
            yield from m.wait("DPF", t)
            state[(h, w, "dP", t)] = True
            if all(state.get((hh, ww, "dP", t)) for hh in range(2) for ww in range(4)):
                state[("dP", t, "read")] = True
            yield
            wrote_ds[(t, h)] = all(state.get((h, ww, "dP", t)) for ww in range(4))
            ws_users[t] -= 1
            m.bars[f"B{h}"].arrive()
            yield
        yield from m.wait("Done", 0)

    actors = {"loader": loader(), "mma": mma_warp()}
    for h in range(2):
        for w in range(4):
            actors[f"wg{h}.{w}"] = warp(h, w)
    m.run(actors)


def simulate_dq(n_t, seed, plant=None):
    m = Model(seed)
    m.bar("X")
    for s in range(K_STAGES_DQ):
        m.bar(f"KF{s}")
        m.bar(f"KE{s}")
    for s in range(V_STAGES_DQ):
        m.bar(f"VF{s}")
        m.bar(f"VE{s}")
    for name in ("SF0", "SF1", "DPF", "Done"):
        m.bar(name)
    for h in range(2):
        m.bar(f"B{h}", 4)
    ring = {"K": [None] * K_STAGES_DQ, "V": [None] * V_STAGES_DQ}
    landed = {"K": [False] * K_STAGES_DQ, "V": [False] * V_STAGES_DQ}
    readers = {}
    sbuf = [None, None]  # tile held by S buffer 0 / 1
    state = {}

    def loader():
        m.later(lambda: m.bars["X"].arrive())
        for t in range(n_t):
            for kind, n in (("K", K_STAGES_DQ), ("V", V_STAGES_DQ)):
                s = t % n
                if t >= n:
                    yield from m.wait(f"{kind}E{s}", t // n - 1)
                    if any(i >= m.done for i in readers.get((kind, t - n), [])):
                        raise ProtocolError(f"{kind} stage {s} reloaded while tile {t - n} is read")
                ring[kind][s], landed[kind][s] = t, False

                def land(kind=kind, s=s):
                    landed[kind][s] = True
                    m.bars[f"{kind}F{s}"].arrive()
                m.later(land)
                yield

    def use(kind, t, n):
        s = t % n
        if ring[kind][s] != t or not landed[kind][s]:
            raise ProtocolError(f"MMA reads {kind} stage {s} without tile {t}")
        ids = [m.mma() for _ in range(8)]
        readers.setdefault((kind, t), []).extend(ids)
        return ids

    def issue_s(t):
        b = t & 1
        if sbuf[b] is not None:
            prev = sbuf[b]
            if not state.get(("dS", prev, "written")) or not state.get(("dQ", prev)):
                raise ProtocolError(f"S({t}) overwrites buffer {b} before dQ({prev}) is issued")
        use("K", t, K_STAGES_DQ)
        sbuf[b] = t
        m.commit(f"SF{b}")

    def mma_warp():
        yield from m.wait("X", 0)
        yield from m.wait("KF0", 0)
        issue_s(0)
        yield from m.wait("VF0", 0)
        use("V", 0, V_STAGES_DQ)
        state[("dP", 0)] = True
        m.commit("DPF")
        if n_t > 1:
            yield from m.wait("KF1", 0)
            issue_s(1)
        yield
        for t in range(n_t):
            for h in range(2):
                yield from m.wait(f"B{h}", t)
            state[("dS", t, "written")] = True
            m.commit(f"VE{t % V_STAGES_DQ}")
            if t + 1 < n_t:
                u = t + 1
                yield from m.wait(f"VF{u % V_STAGES_DQ}", u // V_STAGES_DQ)
                use("V", u, V_STAGES_DQ)
                state[("dP", u)] = True
                m.commit("DPF")
            if plant != "s_before_dq":
                use("K", t, K_STAGES_DQ)  # dQ += dS(t) K_t
                state[("dQ", t)] = True
                m.commit(f"KE{t % K_STAGES_DQ}")
            if t + 2 < n_t:
                u = t + 2
                yield from m.wait(f"KF{u % K_STAGES_DQ}", u // K_STAGES_DQ)
                issue_s(u)
            if plant == "s_before_dq":
                use("K", t, K_STAGES_DQ)
                state[("dQ", t)] = True
                m.commit(f"KE{t % K_STAGES_DQ}")
            if t == n_t - 1:
                m.commit("Done")
            yield

    def warp(h, w):
        for t in range(n_t):
            b = t & 1
            yield from m.wait(f"SF{b}", t >> 1)
            if sbuf[b] != t:
                raise ProtocolError("warp reads an S buffer without its tile")
            yield
            yield from m.wait("DPF", t if plant != "dp_parity" else t + 1)
            yield
            m.bars[f"B{h}"].arrive()
            yield
        yield from m.wait("Done", 0)

    actors = {"loader": loader(), "mma": mma_warp()}
    for h in range(2):
        for w in range(4):
            actors[f"wg{h}.{w}"] = warp(h, w)
    m.run(actors)


def _lengths(n, seed0):
    r = random.Random(seed0)
    return [(r.randint(1, 9), seed0 + i) for i in range(n)]


def test_dkdv_protocol_model_random_schedules():
    for n_t, seed in _lengths(500, 0):
        simulate_dkdv(n_t, seed)


def test_dq_protocol_model_random_schedules():
    for n_t, seed in _lengths(500, 1000):
        simulate_dq(n_t, seed)


@pytest.mark.parametrize("plant", ["s_over_p", "early_release"])
def test_dkdv_protocol_model_catches_planted_bugs(plant):
    with pytest.raises(ProtocolError):
        for n_t, seed in _lengths(300, 0):
            simulate_dkdv(max(n_t, 3), seed, plant=plant)


@pytest.mark.parametrize("plant", ["s_before_dq", "dp_parity"])
def test_dq_protocol_model_catches_planted_bugs(plant):
    with pytest.raises(ProtocolError):
        for n_t, seed in _lengths(300, 1000):
            simulate_dq(max(n_t, 3), seed, plant=plant)
