"""A model check of the attention kernels' mbarrier protocols (CPU).

attn_tc_kernel coordinates two TMA producer lanes (K ring, V ring), an MMA issuer and two
softmax groups of four warps through mbarriers with phase parities.  This module restates
those waits, arrivals, expected byte counts and MMA-completion commits (in attn.cu's order),
runs them under random interleavings and random completion orders of the asynchronous copies
and MMAs, and checks that every role finishes, that no barrier phase receives more arrivals
than it expects, and that every wait really orders what it is meant to order (an S read after
its product, a P written after the product that read the buffer before, the merge after every
product) — a parity that aliases an older phase fails here.  The planted case below shows that
a missing wait is caught, without a GPU.  Keep it in step with attn.cu."""
import random

import pytest

Q_BYTES, K_BYTES, V_BYTES = 100, 10, 10   # any positive sizes: only the bookkeeping matters


class Bar:
    """An mbarrier: expected arrivals, pending transaction bytes and the phase bit; a wait on
    parity p is satisfied once the phase with parity p has completed."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase ^= 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "over-arrival"
        self._maybe_complete()

    def expect_tx(self, nbytes):       # arrive.expect_tx
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):     # a copy's bytes landing
        self.tx -= nbytes
        self._maybe_complete()

    def done(self, parity):
        return self.phase != parity


class Sim:
    def __init__(self):
        self.bars = {}
        self.events = []               # asynchronous completions not yet delivered

    def bar(self, key, count=1):
        if key not in self.bars:
            self.bars[key] = Bar(count)
        return self.bars[key]


def run(actors, sim, seed):
    """Actors are generators that yield wait conditions.  Returns "ok", or "deadlock ..." when
    no actor can move and no asynchronous completion is outstanding."""
    rnd = random.Random(seed)
    cond = {k: None for k in actors}
    live = dict(actors)
    for _ in range(500000):
        if not live:
            break
        ready = [k for k in live if cond[k] is None or cond[k]()]
        if sim.events and (not ready or rnd.random() < 0.4):
            sim.events.pop(rnd.randrange(len(sim.events)))()
            continue
        if not ready:
            return "deadlock " + ",".join(sorted(live))
        k = rnd.choice(ready)
        try:
            cond[k] = next(live[k])
        except StopIteration:
            del live[k]
    else:
        return "timeout"
    while sim.events:
        sim.events.pop()()
    return "ok"


def mma_issuer(nkv, NS, sim, q_full, k_full, v_full, s_free, p_full, on_s, on_pv, st):
    """S(0) and S(1), then per tile j in order: O_{j&1} += P(j) V(j) once P(j) and V(j) are
    there, then S(j + 2) into buffer j & 1 once K(j + 2) landed and the buffer is free.
    on_s / on_pv deliver the commits' arrivals."""
    yield lambda: q_full.done(0)
    ring = {"stage": 0, "phase": 0}

    def issue_s(j):
        b = j & 1
        yield lambda s=ring["stage"], p=ring["phase"]: k_full[s].done(p)
        yield lambda b=b, j=j: s_free[b].done(((j >> 1) & 1) ^ 1)
        # the buffer's previous tile (j - 2) was read and its P V product issued before
        assert j < 2 or (st["reads"][j - 2] == 4 and (j - 2) in st["pv_issued"])
        sim.events.append(lambda b=b, s=ring["stage"], j=j: on_s(j, b, s))
        ring["stage"] += 1
        if ring["stage"] == NS:
            ring["stage"], ring["phase"] = 0, ring["phase"] ^ 1

    yield from issue_s(0)
    if nkv > 1:
        yield from issue_s(1)
    pstage = pphase = 0
    for j in range(nkv):
        pb = j & 1
        yield lambda pb=pb, j=j: p_full[pb].done((j >> 1) & 1)
        assert st["writes"][j] == 4, "P V issued before all of P(j) was written"
        yield lambda s=pstage, p=pphase: v_full[s].done(p)
        st["pv_issued"].add(j)
        sim.events.append(lambda s=pstage, pb=pb, j=j: on_pv(j, s, pb))
        pstage += 1
        if pstage == NS:
            pstage, pphase = 0, pphase ^ 1
        if j + 2 < nkv:
            yield from issue_s(j + 2)


def softmax_warp(g, nkv, s_full, pv_done, s_free, p_full, st, final_wait=True):
    """One warp of softmax group g (tiles g, g + 2, ...): wait for S of its tile, then for the
    group's previous P V product (its P buffer and O accumulator), release S and publish P.  At
    the end wait for the group's last product, then meet the other group at a named barrier,
    after which every product of the CTA must have completed (the merge reads both O)."""
    n_mine = (nkv - g + 1) // 2
    for it in range(n_mine):
        j = g + 2 * it
        yield lambda it=it: s_full[g].done(it & 1)
        assert j in st["s_done"], "S(j) read before its product completed"
        if it >= 1:
            yield lambda it=it: pv_done[g].done((it - 1) & 1)
            assert (j - 2) in st["pv_done"], "P(j) written over a P still being read"
        st["reads"][j] += 1
        st["writes"][j] += 1
        s_free[g].arrive()
        p_full[g].arrive()
    if n_mine and final_wait:
        yield lambda: pv_done[g].done((n_mine - 1) & 1)
    st["at_bar"] += 1
    yield lambda: st["at_bar"] == 8
    assert len(st["pv_done"]) == nkv, "merge before every product completed"


def single(nkv, NS, sim, final_wait=True):
    """attn_tc_kernel: separate K and V rings, each filled by its own producer lane; a K stage
    is released by the commit after S = Q K^T, a V stage by the commit after P V; two softmax
    groups of four warps take the key tiles in turn."""
    q_full = sim.bar("q_full")
    k_full = [sim.bar(("k", s)) for s in range(NS)]
    v_full = [sim.bar(("v", s)) for s in range(NS)]
    k_empty = [sim.bar(("k_empty", s)) for s in range(NS)]
    v_empty = [sim.bar(("v_empty", s)) for s in range(NS)]
    s_full = [sim.bar(("s_full", b)) for b in range(2)]
    s_free = [sim.bar(("s_free", b), 4) for b in range(2)]
    p_full = [sim.bar(("p_full", b), 4) for b in range(2)]
    pv_done = [sim.bar(("pv_done", b)) for b in range(2)]
    st = {"s_done": set(), "pv_done": set(), "pv_issued": set(), "at_bar": 0,
          "reads": [0] * nkv, "writes": [0] * nkv}

    def producer(full, empty, nbytes, with_q):
        if with_q:
            q_full.expect_tx(Q_BYTES)
            sim.events.append(lambda: q_full.complete_tx(Q_BYTES))
        stage = phase = 0
        for _ in range(nkv):
            yield lambda s=stage, p=phase ^ 1: empty[s].done(p)
            full[stage].expect_tx(nbytes)
            sim.events.append(lambda s=stage: full[s].complete_tx(nbytes))
            stage += 1
            if stage == NS:
                stage, phase = 0, phase ^ 1

    def on_s(j, b, s):
        st["s_done"].add(j)
        s_full[b].arrive()
        k_empty[s].arrive()

    def on_pv(jj, s, pb):
        st["pv_done"].add(jj)
        v_empty[s].arrive()
        pv_done[pb].arrive()

    actors = {"producer_k": producer(k_full, k_empty, K_BYTES, True),
              "producer_v": producer(v_full, v_empty, V_BYTES, False),
              "mma": mma_issuer(nkv, NS, sim, q_full, k_full, v_full, s_free, p_full,
                                on_s, on_pv, st)}
    for g in range(2):
        for w in range(4):
            actors[f"softmax{g}{w}"] = softmax_warp(g, nkv, s_full, pv_done, s_free, p_full, st,
                                                    final_wait)
    return actors


@pytest.mark.parametrize("NS", [2, 3, 4])
def test_protocol_completes(NS):
    for nkv in (1, 2, 3, 4, 5, 7, 9, 16):
        for seed in range(20):
            sim = Sim()
            assert run(single(nkv, NS, sim), sim, seed) == "ok", (nkv, NS, seed)


def test_planted_missing_final_wait_is_caught():
    """Both groups meeting at the merge barrier without first waiting for their last product:
    the merge then reads an accumulator that is still being written."""
    fails = 0
    for seed in range(20):
        sim = Sim()
        try:
            fails += run(single(5, 2, sim, final_wait=False), sim, seed) != "ok"
        except AssertionError:
            fails += 1
    assert fails > 0
