"""The key layout of smdm_step_switched, checked against the step-causal predicate (CPU).

The library runs the Table-6 switch settings with prefix attention only: the sequence's KV
cache holds the prompt at slots [0, P) and the decoded tokens in decode order after it; the
step's masks and tail rows follow.  Each row then sees exactly the key prefix [0, kvlen) that
the library assigns it.  This test rebuilds that layout and those prefix lengths from the rules
stated in include/smdm.h and checks, for every switch setting and every step of a small run,
that the step-causal predicate allows exactly the prefix for every row, and that the rows are,
as a set, the ones the oracle's Switched state feeds to the network."""
import itertools

import numpy as np
import pytest

import oracle
import synth

PROMPT, CLEAN, MASK, REG = oracle.PROMPT, oracle.CLEAN, oracle.MASK, oracle.REG


def library_layout(P, L, k, dec, dec_lab, n_new, qp, extra, n_tail, cp, cr):
    """(key types, key labels, rows) with rows as (type, label, pos, kvlen): the layout the
    library's switched pack builds at step k.  dec / dec_lab: decoded positions in decode order
    and their steps, the last n_new of them committed at step k-1."""
    n_dec = len(dec)
    base = P + n_dec
    keys_t = [PROMPT] * P + [CLEAN] * n_dec + [MASK] * (len(qp) + len(extra)) + [REG] * n_tail
    keys_l = [0] * P + list(dec_lab) + [k] * (len(qp) + len(extra) + n_tail)
    all_keys = len(keys_t)
    rows = []
    if not cp:
        rows += [(PROMPT, 0, i + 1, P) for i in range(P)]
    if cr:
        rows += [(CLEAN, k - 1, int(p), base) for p in dec[n_dec - n_new:]]
    else:
        for j, p in enumerate(dec):
            hi = int(np.searchsorted(dec_lab, dec_lab[j], side="right"))
            rows += [(CLEAN, int(dec_lab[j]), int(p), P + hi)]
    rows += [(MASK, k, int(p), all_keys) for p in qp]
    rows += [(MASK, k, int(p), all_keys) for p in extra]
    rows += [(REG, k, L + 1 + t, all_keys) for t in range(n_tail)]
    return np.array(keys_t), np.array(keys_l), rows


@pytest.mark.parametrize("switches", list(itertools.product([True, False], repeat=3)))
def test_every_row_sees_a_key_prefix(switches):
    cp, cr, tr = switches
    shape = synth.ModelShape(1, 16, 1, 16, 16, 20, n_reg=3, dtype=synth.F32)
    m = oracle.Model(synth.make_weights(shape, 5, std=0.3))
    P, Lg = 5, 18
    prompt = np.arange(P) % shape.vocab
    order = np.random.Generator(np.random.PCG64(9)).permutation(Lg) + P + 1
    n_steps = synth.cosine_schedule(Lg, 5)
    st = oracle.Switched(m, prompt, Lg, cache_prompt=cp, cache_res=cr, truncate=tr)
    dec, dec_lab, off, prev = [], [], 0, 0
    for k in range(1, len(n_steps) + 1):
        qp = order[off:off + n_steps[k - 1]]
        off += n_steps[k - 1]
        masked = [p for p in range(P + 1, P + Lg + 1) if st.grid[p - P - 1] < 0]
        extra = [] if tr else [p for p in masked if p not in set(qp.tolist())]
        keys_t, keys_l, rows = library_layout(P, P + Lg, k, np.array(dec, dtype=np.int64),
                                              np.array(dec_lab, dtype=np.int64), prev, qp,
                                              extra, shape.n_reg, cp, cr)
        for (t, lab, pos, kvlen) in rows:
            vis = oracle.cross_mask([t], [lab], keys_t, keys_l)[0]
            assert np.array_equal(np.flatnonzero(vis), np.arange(kvlen)), (switches, k, t, lab)
        ref, c0, keep = st.rows(qp)
        mine = sorted((t, lab, pos) for (t, lab, pos, _) in rows)
        theirs = sorted(zip(ref.types.tolist(), ref.labels.tolist(), ref.pos.tolist()))
        assert mine == theirs, (switches, k)
        # commit the decode set (its tokens do not matter to the layout)
        st.step_k += 1
        st.commit(qp, np.zeros(len(qp), dtype=np.int64))
        dec += qp.tolist()
        dec_lab += [k] * len(qp)
        prev = len(qp)
