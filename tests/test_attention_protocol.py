"""A model check of the attention kernels' mbarrier protocols (CPU).

attn_tc_kernel (one CTA) and attn_pair_kernel (a CTA pair) coordinate a TMA producer, an MMA
issuer and four softmax warps per CTA through mbarriers with phase parities.  This module
restates those waits, arrivals, expected byte counts and MMA-completion commits (in attn.cu's
order, with the pair's collecting barriers in the first CTA and multicast commits to both),
runs them under random interleavings and random completion orders of the asynchronous copies
and MMAs, and checks that every role finishes and that no barrier phase receives more arrivals
than it expects.  A wrong parity or arrival count deadlocks or over-arrives here (the planted
case below), without a GPU.  Keep it in step with attn.cu."""
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


def softmax_warp(nkv, s_full, pv_done, s_free, p_full, rescale, rnd):
    """One softmax warp: per key tile wait S(j); before writing P(j) wait for the product of
    tile j-2 (its P buffer) and, when the reference maximum moves, of tile j-1; then release
    S(j) and publish P(j).  At the end wait for the last product."""
    for j in range(nkv):
        b = j & 1
        yield lambda b=b, j=j: s_full[b].done((j >> 1) & 1)
        if j >= 2:
            yield lambda j=j: pv_done[j & 1].done(((j - 2) >> 1) & 1)
        if j >= 1 and rnd.random() < rescale:
            yield lambda j=j: pv_done[(j - 1) & 1].done(((j - 1) >> 1) & 1)
        s_free[b].arrive()
        p_full[j & 1].arrive()
    yield lambda: pv_done[(nkv - 1) & 1].done(((nkv - 1) >> 1) & 1)


def mma_issuer(nkv, NS, sim, q_full, k_full, v_full, s_free, p_full, on_s, on_pv):
    """S(j) = Q K(j)^T once K(j) landed and S buffer j & 1 is free; then O += P(j-1) V(j-1)
    once P(j-1) and V(j-1) are there.  on_s / on_pv deliver the commits' arrivals."""
    yield lambda: q_full.done(0)
    stage = phase = pstage = pphase = 0
    for j in range(nkv + 1):
        if j < nkv:
            b = j & 1
            yield lambda s=stage, p=phase: k_full[s].done(p)
            yield lambda b=b, j=j: s_free[b].done(((j >> 1) & 1) ^ 1)
            sim.events.append(lambda b=b, s=stage: on_s(b, s))
            stage += 1
            if stage == NS:
                stage, phase = 0, phase ^ 1
        if j >= 1:
            jj = j - 1
            pb = jj & 1
            yield lambda pb=pb, jj=jj: p_full[pb].done((jj >> 1) & 1)
            yield lambda s=pstage, p=pphase: v_full[s].done(p)
            sim.events.append(lambda s=pstage, pb=pb: on_pv(s, pb))
            pstage += 1
            if pstage == NS:
                pstage, pphase = 0, pphase ^ 1


def single(nkv, NS, rescale, sim, rnd):
    """attn_tc_kernel: separate K and V rings, each filled by its own producer lane; a K stage
    is released by the commit after S = Q K^T, a V stage by the commit after P V."""
    q_full = sim.bar("q_full")
    k_full = [sim.bar(("k", s)) for s in range(NS)]
    v_full = [sim.bar(("v", s)) for s in range(NS)]
    k_empty = [sim.bar(("k_empty", s)) for s in range(NS)]
    v_empty = [sim.bar(("v_empty", s)) for s in range(NS)]
    s_full = [sim.bar(("s_full", b)) for b in range(2)]
    s_free = [sim.bar(("s_free", b), 4) for b in range(2)]
    p_full = [sim.bar(("p_full", b), 4) for b in range(2)]
    pv_done = [sim.bar(("pv_done", b)) for b in range(2)]

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

    def on_s(b, s):
        s_full[b].arrive()
        k_empty[s].arrive()

    def on_pv(s, pb):
        v_empty[s].arrive()
        pv_done[pb].arrive()

    actors = {"producer_k": producer(k_full, k_empty, K_BYTES, True),
              "producer_v": producer(v_full, v_empty, V_BYTES, False),
              "mma": mma_issuer(nkv, NS, sim, q_full, k_full, v_full, s_free, p_full,
                                on_s, on_pv)}
    for w in range(4):
        actors[f"softmax{w}"] = softmax_warp(nkv, s_full, pv_done, s_free, p_full, rescale, rnd)
    return actors


def pair(nkv, NS, rescale, sim, rnd, s_free_count=8):
    # barriers that collect both CTAs live in CTA 0; MMA commits are multicast to both CTAs
    q_full = sim.bar((0, "q_full"))
    k_full = [sim.bar((0, "k", s)) for s in range(NS)]
    v_full = [sim.bar((0, "v", s)) for s in range(NS)]
    s_free = [sim.bar((0, "s_free", b), s_free_count) for b in range(2)]
    p_full = [sim.bar((0, "p_full", b), 8) for b in range(2)]
    kv_empty = {r: [sim.bar((r, "empty", s)) for s in range(NS)] for r in (0, 1)}
    s_full = {r: [sim.bar((r, "s_full", b)) for b in range(2)] for r in (0, 1)}
    pv_done = {r: [sim.bar((r, "pv_done", b)) for b in range(2)] for r in (0, 1)}

    def producer(rank):
        if rank == 0:
            q_full.expect_tx(2 * Q_BYTES)
        sim.events.append(lambda: q_full.complete_tx(Q_BYTES))
        stage = phase = 0
        for _ in range(nkv):
            yield lambda s=stage, p=phase ^ 1: kv_empty[rank][s].done(p)
            if rank == 0:
                k_full[stage].expect_tx(2 * K_BYTES)
            sim.events.append(lambda s=stage: k_full[s].complete_tx(K_BYTES))
            if rank == 0:
                v_full[stage].expect_tx(2 * V_BYTES)
            sim.events.append(lambda s=stage: v_full[s].complete_tx(V_BYTES))
            stage += 1
            if stage == NS:
                stage, phase = 0, phase ^ 1
        # the last commits land in this CTA's barriers before it may exit
        for i in range(nkv, nkv + NS):
            yield lambda i=i: kv_empty[rank][i % NS].done(((i // NS) & 1) ^ 1)

    def on_s(b, s):
        for r in (0, 1):
            s_full[r][b].arrive()

    def on_pv(s, pb):
        for r in (0, 1):
            kv_empty[r][s].arrive()
        for r in (0, 1):
            pv_done[r][pb].arrive()

    actors = {"producer0": producer(0), "producer1": producer(1),
              "mma": mma_issuer(nkv, NS, sim, q_full, k_full, v_full, s_free, p_full, on_s,
                                on_pv)}
    for r in (0, 1):
        for w in range(4):
            actors[f"softmax{r}{w}"] = softmax_warp(nkv, s_full[r], pv_done[r], s_free, p_full,
                                                    rescale, rnd)
    return actors


@pytest.mark.parametrize("kind", ["single", "pair"])
@pytest.mark.parametrize("NS", [2, 3, 4])
def test_protocol_completes(kind, NS):
    for nkv in (1, 2, 3, 4, 5, 7, 9, 16):
        for seed in range(20):
            sim = Sim()
            rnd = random.Random(seed * 7 + nkv)
            actors = (single if kind == "single" else pair)(nkv, NS, 0.3, sim, rnd)
            assert run(actors, sim, seed) == "ok", (kind, nkv, NS, seed)


def test_planted_wrong_arrival_count_is_caught():
    """The pair's S-free barrier expecting one CTA's softmax warps only (4 instead of 8)."""
    fails = 0
    for seed in range(10):
        sim = Sim()
        try:
            fails += run(pair(5, 2, 0.3, sim, random.Random(seed), s_free_count=4), sim,
                         seed) != "ok"
        except AssertionError:
            fails += 1
    assert fails == 10
