"""Per-row key bounds of the training form (CPU).

For bf16 models the library gives every row of a step-labelled forward the bound
kvlen = 1 + the last key index it may see, from per-label last indices and their prefix maximum
(misc.cu, label bounds).  This restates that rule and checks it against the step-causal
predicate of the oracle for random row sets in any order, and shows that a trajectory's rows,
grouped by step, get triangular bounds."""
import numpy as np

import oracle
import synth

CLEAN_TYPES = (oracle.PROMPT, oracle.CLEAN)


def library_bounds(types, labels):
    n = len(types)
    if any(l < 0 or l > n for l in labels):
        return np.full(n, n)
    lastc = np.full(n + 1, -1)
    lastm = np.full(n + 1, -1)
    for j, (t, l) in enumerate(zip(types, labels)):
        if t in CLEAN_TYPES:
            lastc[l] = max(lastc[l], j)
        else:
            lastm[l] = max(lastm[l], j)
    prefix = np.maximum.accumulate(lastc)
    out = np.empty(n, dtype=np.int64)
    for r, (t, l) in enumerate(zip(types, labels)):
        hi = prefix[l] if t in CLEAN_TYPES else max(prefix[l - 1] if l > 0 else -1, lastm[l])
        out[r] = min(n, max(hi + 1, r + 1))
    return out


def test_bounds_are_one_past_the_last_visible_key():
    g = np.random.Generator(np.random.PCG64(17))
    for trial in range(40):
        n = int(g.integers(1, 60))
        types = g.integers(0, 4, n)
        labels = g.integers(0, min(6, n + 1), n)     # labels within [0, n]: exact bounds
        # prompt rows carry label 0, as in every form the library builds
        labels[types == oracle.PROMPT] = 0
        vis = oracle.cross_mask(types, labels, types, labels)
        expect = np.array([np.flatnonzero(vis[r]).max() + 1 for r in range(n)])
        assert np.array_equal(library_bounds(types, labels), expect), trial


def test_out_of_range_labels_leave_every_bound_at_n():
    """A label outside [0, n] turns the bounds off (n for every row), which is never tighter
    than the predicate allows."""
    types = np.array([oracle.PROMPT, oracle.MASK, oracle.CLEAN])
    labels = np.array([0, 7, 1])
    assert list(library_bounds(types, labels)) == [3, 3, 3]


def test_trajectory_rows_get_triangular_bounds():
    shape = synth.ModelShape(1, 16, 1, 16, 16, 20, n_reg=3, dtype=synth.F32)
    m = oracle.Model(synth.make_weights(shape, 5, std=0.3))
    P, Lg = 6, 40
    prompt = np.arange(P) % shape.vocab
    order = (np.random.Generator(np.random.PCG64(4)).permutation(Lg) + P + 1).astype(np.int32)
    plan = synth.Plan("order", 8, order, synth.cosine_schedule(Lg, 8))
    st, recs = oracle.generate(m, prompt, Lg, plan)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, shape, Lg, recs)
    # group the rows by step: prompt, then for each step its clean tokens and its masks/registers
    cls = np.where(np.isin(types, CLEAN_TYPES), 0, 1)
    order_rows = np.lexsort((cls, labels))
    t, l = types[order_rows], labels[order_rows]
    kv = library_bounds(t, l)
    n = len(t)
    vis = oracle.cross_mask(t, l, t, l)
    assert np.array_equal(kv, [np.flatnonzero(vis[r]).max() + 1 for r in range(n)])
    assert np.all(np.diff(kv) >= 0)
    assert kv.sum() < 0.6 * n * n          # about half of the full n x n scan


# ------------------------------------------------------------------------------------------
# Key-tile lists: per 128-row query tile, the key tiles that may hold a visible key.
# ------------------------------------------------------------------------------------------

BIG, SMALL = 2 ** 31 - 1, -2 ** 31


def tile_summary(types, labels, tile):
    """Per tile: label ranges of its clean rows and of its mask/register rows (empty: BIG/SMALL)."""
    out = []
    for t0 in range(0, len(types), tile):
        ty, lb = types[t0:t0 + tile], labels[t0:t0 + tile]
        c = [l for t, l in zip(ty, lb) if t in CLEAN_TYPES]
        m = [l for t, l in zip(ty, lb) if t not in CLEAN_TYPES]
        out.append((min(c, default=BIG), max(c, default=SMALL),
                    min(m, default=BIG), max(m, default=SMALL)))
    return out


def library_tile_lists(types, labels, tile=128):
    s = tile_summary(types, labels, tile)
    lists = []
    for q in s:
        lists.append([t for t, k in enumerate(s)
                      if k[0] <= q[1] or k[0] < q[3] or max(k[2], q[2]) <= min(k[3], q[3])])
    return lists


def test_tile_lists_cover_every_visible_key():
    g = np.random.Generator(np.random.PCG64(23))
    tile = 8   # small tiles, the same rule as the library's 128
    for trial in range(30):
        n = int(g.integers(1, 90))
        types = g.integers(0, 4, n)
        labels = g.integers(0, 7, n)
        labels[types == oracle.PROMPT] = 0
        vis = oracle.cross_mask(types, labels, types, labels)
        lists = library_tile_lists(types, labels, tile)
        for qt, lst in enumerate(lists):
            need = {j // tile for r in range(qt * tile, min(n, qt * tile + tile))
                    for j in np.flatnonzero(vis[r])}
            assert need <= set(lst), (trial, qt)
            assert lst == sorted(lst)


def test_tile_lists_skip_most_of_a_trajectory():
    """Rows laid out as the oracle's trajectory and bench.py --form training lay them out
    (the prompt, every step's clean tokens by step, then every step's masks and registers by
    step): a query tile's list holds the clean prefix it may see and its own mask block, so the
    lists cover a small part of the full scan and of the triangular bound, and still every
    tile a visible key needs."""
    P, Lg, K, nreg, tile = 16, 256, 16, 8, 16
    n = synth.cosine_schedule(Lg, K)
    types, labels = [oracle.PROMPT] * P, [0] * P
    for k in range(1, K + 1):
        types += [oracle.CLEAN] * n[k - 1]
        labels += [k] * n[k - 1]
    for k in range(1, K + 1):
        types += [oracle.MASK] * n[k - 1] + [oracle.REG] * nreg
        labels += [k] * (n[k - 1] + nreg)
    types, labels = np.array(types), np.array(labels)
    vis = oracle.cross_mask(types, labels, types, labels)
    lists = library_tile_lists(types, labels, tile)
    kv = library_bounds(types, labels)
    T = len(lists)
    rows_of = lambda q: range(q * tile, min(len(kv), q * tile + tile))
    listed = sum(len(x) for x in lists)
    bounded = sum((max(kv[r] for r in rows_of(q)) + tile - 1) // tile for q in range(T))
    for q in range(T):
        assert {j // tile for r in rows_of(q) for j in np.flatnonzero(vis[r])} <= set(lists[q])
    assert listed < 0.6 * bounded and listed < 0.3 * T * T
