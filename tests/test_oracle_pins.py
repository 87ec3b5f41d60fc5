"""Pins for the fp64 oracle: values and statements the Sparse-LaViDa pages fix, closed forms,
library routines and the method's exactness invariants.  CPU only."""
import dataclasses
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TYPES = {"PROMPT": oracle.PROMPT, "CLEAN": oracle.CLEAN, "MASK": oracle.MASK, "REG": oracle.REG}


def tiny_shape(n_reg=4, **kw):
    args = dict(n_layers=2, d_model=32, n_heads=2, d_head=16, d_ffn=48, vocab=40, n_reg=n_reg,
                dtype=synth.F32)
    args.update(kw)
    return synth.ModelShape(**args)


def tiny_model(seed=7, n_reg=4, std=0.25, **kw):
    return oracle.Model(synth.make_weights(tiny_shape(n_reg, **kw), seed, gain_std=0.1, std=std))


def tiny_plan(P, Lg, steps, seed=3):
    g = np.random.Generator(np.random.PCG64(seed))
    order = (g.permutation(Lg) + P + 1).astype(np.int32)
    n = synth.cosine_schedule(Lg, steps)
    return synth.Plan("order", steps, order, n)


# ------------------------------------------------------------------------------------------
# Worked example (sparse parameterization, Sec. 3.1)
# ------------------------------------------------------------------------------------------

def test_worked_example_roundtrip():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    toks, pos, L = oracle.sparse_encode(g["dense"], g["mask"])
    assert toks == g["clean"] and pos == g["positions"] and L == g["length"]
    assert oracle.sparse_decode(toks, pos, L, g["mask"]) == g["dense"]


def test_worked_example_packed_rows():
    """The same example as packed rows: 3 clean + 4 masks + 64 registers at 8..71."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    vocab = {w: i for i, w in enumerate(["I", "have", "dog"])}
    shape = synth.ModelShape(1, 8, 1, 8, 8, 3, n_reg=g["n_registers"], dtype=synth.F32)
    L = g["length"]
    grid = np.full(L, -1)
    for t, p in zip(g["clean"], g["positions"]):
        grid[p - 1] = vocab[t]
    masked = [p for p in range(1, L + 1) if p not in g["positions"]]
    rows = oracle.pack_step(shape, 0, L, grid, g["positions"], masked, k=2)
    # |A| + |C| + m rows (Appendix 7.2)
    assert rows.n == len(g["positions"]) + len(masked) + g["n_registers"]
    assert list(rows.pos[:3]) == g["positions"]
    assert list(rows.ids[:3]) == [vocab[t] for t in g["clean"]]
    assert (rows.ids[3:7] == shape.mask_id).all()
    regs = rows.pos[rows.types == oracle.REG]
    assert [regs[0], regs[-1]] == g["register_positions_first_last"]
    assert (np.diff(regs) == 1).all()
    assert list(rows.ids[rows.types == oracle.REG]) == [shape.vocab + 2 + j for j in range(64)]
    # decode back from the clean rows + L
    dense = oracle.sparse_decode([g["clean"][i] for i in range(3)], list(rows.pos[:3]), L, "[m]")
    assert dense == g["dense"]


def test_sparse_decode_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.sparse_decode(["a", "b"], [1, 1], 3, "[m]")
    with pytest.raises(ValueError):
        oracle.sparse_decode(["a"], [4], 3, "[m]")


# ------------------------------------------------------------------------------------------
# Step-causal mask: the Figure-3 example and the two-path training example
# ------------------------------------------------------------------------------------------

def _read_fig3():
    lines = [l for l in open(os.path.join(GOLDEN, "fig3_visibility.txt")) if not l.startswith("#")]
    spec = lines[0].split(":", 1)[1].split("|")
    rows = [s.split() for s in spec]
    names = [r[0] for r in rows]
    types = [TYPES[r[2]] for r in rows]
    labels = [int(r[3]) for r in rows]
    mat = np.array([[int(v) for v in l.split()[1:]] for l in lines[1:] if l.strip()], dtype=bool)
    return names, types, labels, mat


def test_fig3_mask_matches_page_statements():
    names, types, labels, expect = _read_fig3()
    got = oracle.mask_matrix(types, labels)
    np.testing.assert_array_equal(got, expect)
    np.testing.assert_array_equal(oracle.cross_mask(types, labels, types, labels), expect)


def test_two_path_block_rule():
    lines = [l.split() for l in open(os.path.join(GOLDEN, "two_path_blocks.txt"))
             if l.strip() and not l.startswith("#")]
    M = int(lines[0][1])
    N = int(lines[1][1])
    expect = np.array([[int(v) for v in l[1:]] for l in lines[2:]], dtype=bool)
    types = [oracle.PROMPT] + [oracle.CLEAN] * M + [oracle.MASK] * N
    labels = list(range(M + N + 1))
    np.testing.assert_array_equal(oracle.mask_matrix(types, labels), expect)
    # registers share their masked block's number and obey the same rule
    t2 = types + [oracle.REG]
    l2 = labels + [M + 1]
    m2 = oracle.mask_matrix(t2, l2)
    np.testing.assert_array_equal(m2[-1, :-1], expect[M + 1])          # reg row == block M+1 row
    np.testing.assert_array_equal(m2[:-1, -1], expect[:, M + 1])       # seen like block M+1


def test_incremental_mask_is_prefix_shaped():
    """At a sampling step the rule reduces to per-row prefixes of [cache | new | queries | regs]:
    new-cache rows see cache + new rows, mask/register rows see everything."""
    ct = [oracle.PROMPT] * 5 + [oracle.CLEAN] * 6
    cl = [0] * 5 + [1] * 3 + [2] * 3
    k = 4
    rt = [oracle.CLEAN] * 2 + [oracle.MASK] * 3 + [oracle.REG] * 4
    rl = [k - 1] * 2 + [k] * 7
    vis = oracle.cross_mask(rt, rl, ct + rt, cl + rl)
    ctx, nn, R = len(ct), 2, len(rt)
    for r in range(R):
        kv = ctx + nn if r < nn else ctx + R
        assert vis[r, :kv].all() and not vis[r, kv:].any()


# ------------------------------------------------------------------------------------------
# Transformer primitives against independent formulations / library routines
# ------------------------------------------------------------------------------------------

def _rand_vis(g, nq, nk):
    vis = g.random((nq, nk)) < 0.6
    vis[np.arange(nq), g.integers(0, nk, nq)] = True
    return vis


def test_attention_bruteforce():
    g = np.random.Generator(np.random.PCG64(11))
    nq, nk, H, dh = 5, 7, 2, 4
    q, k, v = (g.standard_normal((n, H, dh)) for n in (nq, nk, nk))
    vis = _rand_vis(g, nq, nk)
    got = oracle.attention(q, k, v, vis)
    for h in range(H):
        for i in range(nq):
            w = {}
            for j in range(nk):
                if vis[i, j]:
                    w[j] = math.exp(sum(q[i, h, t] * k[j, h, t] for t in range(dh)) / math.sqrt(dh))
            z = sum(w.values())
            for t in range(dh):
                ref = sum(w[j] * v[j, h, t] for j in w) / z
                assert abs(got[i, h, t] - ref) < 1e-12


def test_attention_vs_torch_sdpa_fp64():
    g = np.random.Generator(np.random.PCG64(12))
    nq, nk, H, dh = 9, 13, 3, 8
    q, k, v = (g.standard_normal((n, H, dh)) for n in (nq, nk, nk))
    vis = _rand_vis(g, nq, nk)
    got = oracle.attention(q, k, v, vis)
    tq, tk, tv = (torch.from_numpy(a).permute(1, 0, 2) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv,
                                                           attn_mask=torch.from_numpy(vis))
    np.testing.assert_allclose(got, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    # all-visible case equals plain softmax attention
    full = np.ones((nq, nk), bool)
    ref2 = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    np.testing.assert_allclose(oracle.attention(q, k, v, full), ref2.permute(1, 0, 2).numpy(),
                               rtol=0, atol=1e-12)


def test_rmsnorm_vs_torch():
    g = np.random.Generator(np.random.PCG64(13))
    x = g.standard_normal((6, 32)) * 3
    w = 1 + 0.1 * g.standard_normal(32)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (32,), torch.from_numpy(w), eps=1e-6)
    np.testing.assert_allclose(oracle.rmsnorm(x, w, 1e-6), ref.numpy(), rtol=1e-13, atol=1e-13)


def test_silu_vs_torch():
    x = np.linspace(-30, 30, 101)
    np.testing.assert_allclose(oracle.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(),
                               rtol=1e-13, atol=1e-15)


def test_rope_is_complex_rotation():
    """Rotate-half RoPE == multiplying z_i = x_i + i x_{i+dh/2} by exp(i pos theta^(-2i/dh))."""
    g = np.random.Generator(np.random.PCG64(14))
    n, H, dh, theta = 5, 2, 16, 10000.0
    x = g.standard_normal((n, H, dh))
    pos = g.integers(1, 5000, n)
    z = x[..., :dh // 2] + 1j * x[..., dh // 2:]
    freq = np.array([theta ** (-(2 * i) / dh) for i in range(dh // 2)])
    rot = z * np.exp(1j * pos[:, None, None] * freq[None, None, :])
    expect = np.concatenate([rot.real, rot.imag], axis=-1)
    np.testing.assert_allclose(oracle.rope(x, pos, theta), expect, rtol=0, atol=1e-12)


def test_rope_relative_position():
    """<rope(q, p1), rope(k, p2)> depends only on p1 - p2."""
    g = np.random.Generator(np.random.PCG64(15))
    q = g.standard_normal((1, 1, 32))
    k = g.standard_normal((1, 1, 32))
    dots = []
    for p in (3, 100, 2000):
        a = oracle.rope(q, np.array([p + 7]), 10000.0)
        b = oracle.rope(k, np.array([p]), 10000.0)
        dots.append(float(np.sum(a * b)))
    assert max(dots) - min(dots) < 1e-10


def test_unmask_rules():
    lg = np.array([[0.0, 2.0, 2.0, 1.0],     # tie -> lowest id (1)
                   [5.0, 0.0, 0.0, 0.0],
                   [1.0, 1.0, 1.0, 1.0]])    # uniform -> id 0, conf 1/4
    tok, conf, rows = oracle.unmask(lg, oracle.POLICY_ALL)
    assert list(tok) == [1, 0, 0] and list(rows) == [0, 1, 2]
    ref = torch.softmax(torch.from_numpy(lg), dim=1).max(dim=1).values.numpy()
    np.testing.assert_allclose(conf, ref, rtol=1e-14)
    assert abs(conf[2] - 0.25) < 1e-15
    _, _, rows = oracle.unmask(lg, oracle.POLICY_TOPN, 1)
    assert list(rows) == [1]
    # equal confidence -> lowest row wins; committed rows come back in row order
    lg2 = np.array([[1.0, 0.0], [0.0, 1.0], [3.0, 0.0], [1.0, 0.0]])
    _, conf2, rows2 = oracle.unmask(lg2, oracle.POLICY_TOPN, 2)
    assert conf2[0] == conf2[1] == conf2[3]
    assert list(rows2) == [0, 2]


# ------------------------------------------------------------------------------------------
# Plans (inputs) — closed forms
# ------------------------------------------------------------------------------------------

def test_cosine_schedule_closed_form():
    for Lg, lo, hi, ones in ((1024, 1, 25, 3), (4096, 2, 101, 0)):
        n = synth.cosine_schedule(Lg, 64)
        assert n.sum() == Lg and n.min() == lo and n.max() == hi and (n == 1).sum() == ones
        assert n[0] < 100 and n[1] < 100          # "early steps sample fewer than 100 tokens"
        m = Lg - np.cumsum(n)
        for k in range(1, 64):
            assert m[k - 1] <= math.floor(Lg * math.cos(math.pi * k / 128))


def test_stratified_order_is_round_robin_permutation():
    g = np.random.Generator(np.random.PCG64(1))
    o = synth.stratified_order(16, g)
    assert sorted(o.tolist()) == list(range(256))
    tile = (o // 16 // 4) * 4 + (o % 16) // 4
    for j in range(16):                  # every tile appears once in each round of 16
        assert sorted(tile[16 * j:16 * (j + 1)].tolist()) == list(range(16))


# ------------------------------------------------------------------------------------------
# Exactness invariants of the method
# ------------------------------------------------------------------------------------------

def _tiny_run(m, P=6, Lg=24, steps=5, seed=3):
    prompt = np.random.Generator(np.random.PCG64(seed)).integers(0, m.shape.vocab, P)
    plan = tiny_plan(P, Lg, steps, seed)
    st, recs = oracle.generate(m, prompt, Lg, plan)
    return prompt, plan, st, recs


def check_training_equals_incremental(m):
    prompt, plan, st, recs = _tiny_run(m)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, m.shape, st.Lg, recs)
    rows = np.concatenate([qrows[r.k] for r in recs])
    lg = oracle.forward_stepcausal(m, ids, pos, types, labels, rows)
    inc = np.concatenate([r.logits for r in recs])
    return float(np.max(np.abs(lg - inc)))


def test_invariant_training_form_equals_incremental():
    """(b): the parallel training-form forward reproduces every cached sampling step exactly
    (the sparse parameterization is an exact re-parameterization, no approximation)."""
    m = tiny_model()
    assert check_training_equals_incremental(m) < 1e-10


def check_truncation(m):
    prompt, plan, st, recs = _tiny_run(m)
    k = 3
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, m.shape, st.Lg, recs, steps=[k])
    base = oracle.forward_stepcausal(m, ids, pos, types, labels, qrows[k])
    # masks outside C_k that are still masked at step k, materialised as their own masked block
    decoded_before = set(np.concatenate([r.committed_pos for r in recs[:k - 1]]).tolist())
    outside = [p for p in range(len(prompt) + 1, len(prompt) + st.Lg + 1)
               if p not in decoded_before and p not in set(recs[k - 1].query_pos.tolist())]
    n_out = len(outside)
    ids2 = np.concatenate([ids, np.full(n_out, m.shape.mask_id)])
    pos2 = np.concatenate([pos, outside])
    types2 = np.concatenate([types, np.full(n_out, oracle.MASK)])
    labels2 = np.concatenate([labels, np.full(n_out, 1000 + k)])
    trunc = oracle.forward_stepcausal(m, ids2, pos2, types2, labels2, qrows[k])
    return float(np.max(np.abs(trunc - base))), base, n_out


def test_invariant_truncated_and_dropped_masks():
    """(c): C-row predictions are unchanged whether the masks outside C are dropped entirely
    (base) or present but truncated from C's view (own masked block)."""
    m = tiny_model()
    err, base, n_out = check_truncation(m)
    assert n_out > 0
    assert err < 1e-12
    # and both equal the incremental run
    prompt, plan, st, recs = _tiny_run(m)
    np.testing.assert_allclose(base, recs[2].logits, rtol=0, atol=1e-10)


def test_two_masked_blocks_are_independent_paths():
    """One forward with masked blocks of two different steps gives each block the logits of a
    forward holding that block alone (paths 0->..->3->4 and 0->..->3->5)."""
    m = tiny_model()
    prompt, plan, st, recs = _tiny_run(m)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, m.shape, st.Lg, recs, steps=[3, 5])
    both = oracle.forward_stepcausal(m, ids, pos, types, labels,
                                     np.concatenate([qrows[3], qrows[5]]))
    for k, sl in ((3, slice(0, len(qrows[3]))), (5, slice(len(qrows[3]), None))):
        i2, p2, t2, l2, q2 = oracle.trajectory(prompt, m.shape, st.Lg, recs, steps=[k])
        alone = oracle.forward_stepcausal(m, i2, p2, t2, l2, q2[k])
        np.testing.assert_allclose(both[sl], alone, rtol=0, atol=1e-12)
        np.testing.assert_allclose(alone, recs[k - 1].logits, rtol=0, atol=1e-10)


def test_rope_shift_invariance():
    m = tiny_model()
    prompt, plan, st, recs = _tiny_run(m)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, m.shape, st.Lg, recs, steps=[4])
    a = oracle.forward_stepcausal(m, ids, pos, types, labels, qrows[4])
    b = oracle.forward_stepcausal(m, ids, pos + 123, types, labels, qrows[4])
    assert np.max(np.abs(a - b)) < 1e-10
    assert np.max(np.abs(a)) > 0.1


def test_row_permutation_equivariance():
    m = tiny_model()
    prompt, plan, st, recs = _tiny_run(m)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, m.shape, st.Lg, recs)
    rows = np.arange(len(ids))
    perm = np.random.Generator(np.random.PCG64(5)).permutation(len(ids))
    a = oracle.forward_stepcausal(m, ids, pos, types, labels, rows)
    inv = np.argsort(perm)
    b = oracle.forward_stepcausal(m, ids[perm], pos[perm], types[perm], labels[perm], rows)
    np.testing.assert_allclose(b[inv], a, rtol=0, atol=1e-11)


def test_reduces_to_standard_mdm_when_C_is_all_masks():
    """Appendix 7.2: with C = B (every masked position decoded in one step), no registers and
    nothing cached, the sparse step is the standard dense MDM step."""
    m = tiny_model(n_reg=0)
    Lg = 12
    plan = synth.Plan("order", 1, np.arange(1, Lg + 1, dtype=np.int32), np.array([Lg], np.int32))
    st = oracle.Incremental(m, np.zeros(0, np.int64), Lg)
    sparse = st.step_logits(plan.query_positions(1))
    dense = oracle.dense_step_logits(m, np.zeros(0, np.int64), np.full(Lg, -1))
    np.testing.assert_allclose(sparse, dense, rtol=0, atol=1e-11)


def test_dense_step_with_prompt_and_decoded_tokens():
    """The dense comparator at P > 0 with part of the grid decoded: every one of the P + Lg rows
    sees every other ("Key design 1": masks included, full attention), which is the training
    form with every row a clean row of block 0.  Both must give the same generated-row logits;
    dropping the prompt offset of the logit rows or the [MASK] ids of undecoded positions is
    caught."""
    m = tiny_model(n_reg=0)
    g = np.random.Generator(np.random.PCG64(17))
    P, Lg = 9, 14
    prompt = g.integers(0, m.shape.vocab, P)
    grid = np.full(Lg, -1, dtype=np.int64)
    done = g.permutation(Lg)[:6]
    grid[done] = g.integers(0, m.shape.vocab, len(done))
    dense = oracle.dense_step_logits(m, prompt, grid)
    assert dense.shape == (Lg, m.shape.vocab)
    ids = np.concatenate([prompt, np.where(grid < 0, m.shape.mask_id, grid)])
    n = P + Lg
    ref = oracle.forward_stepcausal(m, ids, np.arange(1, n + 1), np.full(n, oracle.CLEAN),
                                    np.zeros(n, dtype=np.int64), np.arange(P, n))
    np.testing.assert_allclose(dense, ref, rtol=0, atol=1e-11)
    # planted: logits of the first Lg rows instead of the generated rows
    wrong = oracle.forward_stepcausal(m, ids, np.arange(1, n + 1), np.full(n, oracle.CLEAN),
                                      np.zeros(n, dtype=np.int64), np.arange(Lg))
    assert np.abs(wrong - dense).max() > 1e-3
    # planted: undecoded positions carrying token 0 instead of [MASK]
    ids0 = np.concatenate([prompt, np.where(grid < 0, 0, grid)])
    wrong = oracle.forward_stepcausal(m, ids0, np.arange(1, n + 1), np.full(n, oracle.CLEAN),
                                      np.zeros(n, dtype=np.int64), np.arange(P, n))
    assert np.abs(wrong - dense).max() > 1e-3


def test_semiar_run_structure():
    wl = synth.WORKLOADS["tiny-bf16-semiar"]
    m = oracle.Model(synth.make_weights(wl.model, wl.seed))
    plan = synth.make_plan(wl)
    st, recs = oracle.generate(m, synth.make_prompt(wl), wl.gen_len, plan)
    assert (st.grid >= 0).all()
    for r in recs:
        lo, hi = synth.semiar_block(plan, wl.prompt_len, r.k)
        assert len(r.committed_pos) == wl.commit
        assert ((r.committed_pos >= lo) & (r.committed_pos < hi)).all()
        j = (r.k - 1) % plan.steps_per_block
        assert len(r.query_pos) == wl.block - j * wl.commit
        assert (np.diff(r.query_pos) > 0).all()          # the block's masks in position order


# ------------------------------------------------------------------------------------------
# Planted mistakes: each plausible error in the oracle must trip one of the pins above.
# ------------------------------------------------------------------------------------------

def test_planted_mask_leak_is_caught(monkeypatch):
    """New-cache rows allowed to see the current masks breaks the Figure-3 pin and (b)."""
    orig = oracle.cross_mask

    def leaky(tq, lq, tk, lk):
        v = orig(tq, lq, tk, lk)
        tq_ = np.asarray(tq)[:, None]
        tk_ = np.asarray(tk)[None, :]
        return v | ((tq_ == oracle.CLEAN) & (tk_ == oracle.MASK))

    monkeypatch.setattr(oracle, "cross_mask", leaky)
    names, types, labels, expect = _read_fig3()
    assert (oracle.cross_mask(types, labels, types, labels) != expect).any()


def test_planted_rope_sign_is_caught(monkeypatch):
    def bad_rope(x, pos, theta):
        dh = x.shape[-1]
        half = dh // 2
        inv = theta ** (-(2.0 * np.arange(half)) / dh)
        ang = pos[:, None] * inv[None, :]
        c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
        a, b = x[..., :half], x[..., half:]
        return np.concatenate([a * c + b * s, a * s + b * c], axis=-1)

    g = np.random.Generator(np.random.PCG64(14))
    x = g.standard_normal((3, 1, 8))
    pos = np.array([1, 5, 9])
    z = x[..., :4] + 1j * x[..., 4:]
    freq = np.array([10000.0 ** (-(2 * i) / 8) for i in range(4)])
    rot = z * np.exp(1j * pos[:, None, None] * freq)
    expect = np.concatenate([rot.real, rot.imag], axis=-1)
    assert np.max(np.abs(bad_rope(x, pos, 10000.0) - expect)) > 1e-3


def test_planted_mask_leak_breaks_invariant_b(monkeypatch):
    """The same leak (clean rows seeing masks), applied everywhere, breaks invariant (b): the
    trajectory's clean rows would see every step's masks, the cached rows only their own."""
    m = tiny_model()
    orig = oracle.cross_mask

    def leaky(tq, lq, tk, lk):
        v = orig(tq, lq, tk, lk)
        tq_ = np.asarray(tq)[:, None]
        tk_ = np.asarray(tk)[None, :]
        return v | ((tq_ == oracle.CLEAN) & (tk_ == oracle.MASK))

    monkeypatch.setattr(oracle, "cross_mask", leaky)
    assert check_training_equals_incremental(m) > 1e-6


def test_planted_register_offset_is_caught(monkeypatch):
    """Registers placed at L..L+63 instead of L+1..L+64 fail the worked-example pin."""
    orig = oracle.pack_step

    def shifted(*a, **kw):
        r = orig(*a, **kw)
        r.pos[r.types == oracle.REG] -= 1
        return r

    monkeypatch.setattr(oracle, "pack_step", shifted)
    with pytest.raises(AssertionError):
        test_worked_example_packed_rows()


def test_planted_missing_register_visibility_is_caught(monkeypatch):
    """Masks not seeing the registers of their own block changes C-row logits vs (b)."""
    m = tiny_model()
    orig = oracle.cross_mask

    def no_regs(tq, lq, tk, lk):
        v = orig(tq, lq, tk, lk)
        tq_ = np.asarray(tq)[:, None]
        tk_ = np.asarray(tk)[None, :]
        return v & ~((tq_ == oracle.MASK) & (tk_ == oracle.REG))

    # The training form uses the patched predicate; the reference incremental logits are taken
    # before patching.
    prompt, plan, st, recs = _tiny_run(m)
    monkeypatch.setattr(oracle, "cross_mask", no_regs)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, m.shape, st.Lg, recs, steps=[2])
    lg = oracle.forward_stepcausal(m, ids, pos, types, labels, qrows[2])
    assert np.max(np.abs(lg - recs[1].logits)) > 1e-6


# ------------------------------------------------------------------------------------------
# Bidirectional tasks: generation positions given from the start (inpainting, outpainting,
# infilling).  Given tokens are clean rows of block 0, cached with the prompt.
# ------------------------------------------------------------------------------------------

def _bidir_run(m, P=6, Lg=24, n_given=10, steps=4, seed=5):
    g = np.random.Generator(np.random.PCG64(seed))
    prompt = g.integers(0, m.shape.vocab, P)
    idx = g.permutation(Lg)
    given = np.sort(idx[:n_given]) + P + 1
    given_tok = g.integers(0, m.shape.vocab, n_given)
    rest = idx[n_given:] + P + 1
    plan = synth.Plan("order", steps, rest.astype(np.int32),
                      synth.cosine_schedule(Lg - n_given, steps))
    st, recs = oracle.generate(m, prompt, Lg, plan, preset_pos=given, preset_tok=given_tok)
    return prompt, given, given_tok, plan, st, recs


def test_bidir_training_form_equals_incremental():
    """(b) with given generation tokens: the one-forward training form (given tokens as
    label-0 clean rows) reproduces every cached step of the bidirectional run exactly."""
    m = tiny_model()
    prompt, given, given_tok, plan, st, recs = _bidir_run(m)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, m.shape, st.Lg, recs,
                                                       preset_pos=given, preset_tok=given_tok)
    rows = np.concatenate([qrows[r.k] for r in recs])
    lg = oracle.forward_stepcausal(m, ids, pos, types, labels, rows)
    inc = np.concatenate([r.logits for r in recs])
    assert float(np.max(np.abs(lg - inc))) < 1e-10


def test_bidir_given_tokens_stay_and_condition():
    m = tiny_model()
    prompt, given, given_tok, plan, st, recs = _bidir_run(m)
    P = len(prompt)
    # the given tokens are in the grid from the start and are never overwritten
    assert (st.grid[given - P - 1] == given_tok).all()
    assert (st.grid >= 0).all()
    with pytest.raises(ValueError):
        st.commit(given[:1], [0])
    # they condition the generation: another given token changes the first step's logits
    other = given_tok.copy()
    other[0] = (other[0] + 1) % m.shape.vocab
    st2 = oracle.Incremental(m, prompt, st.Lg, given, other)
    q = plan.query_positions(1)
    assert np.max(np.abs(st2.step_logits(q) - recs[0].logits)) > 1e-6
    # and an empty given set is the plain prompt-only run
    st3 = oracle.Incremental(m, prompt, st.Lg, [], [])
    st4 = oracle.Incremental(m, prompt, st.Lg)
    assert np.array_equal(st3.step_logits(q), st4.step_logits(q))


def test_bidir_tasks_split_the_generation_region():
    for name, kinds in (("tiny-bf16-cos", ("inpaint", "outpaint", "infill")),
                        ("tiny-bf16-semiar", ("infill",))):
        wl = synth.WORKLOADS[name]
        for kind in kinds:
            t = synth.make_bidir_task(wl, kind)
            gen = set(range(wl.prompt_len + 1, wl.prompt_len + wl.gen_len + 1))
            given = set(t.preset_pos.tolist())
            todo = set(t.plan.order.tolist())
            assert given | todo == gen and not (given & todo)
            assert int(t.plan.n_per_step.sum()) == len(todo)
            if kind == "inpaint":     # a centred hole: the masked positions form one square
                side = wl.grid_side
                hole = sorted(p - wl.prompt_len - 1 for p in todo)
                rows = {i // side for i in hole}
                cols = {i % side for i in hole}
                assert len(hole) == len(rows) * len(cols) == (side // 2) ** 2


# ------------------------------------------------------------------------------------------
# Table-6 speed switches (cache prompt / cache responses / truncate)
# ------------------------------------------------------------------------------------------

SWITCHES = [(cp, cr, tr) for cp in (True, False) for cr in (True, False) for tr in (True, False)]


def _replay_switched(m, prompt, Lg, recs, cp, cr, tr):
    st = oracle.Switched(m, prompt, Lg, cache_prompt=cp, cache_res=cr, truncate=tr)
    out = []
    for r in recs:
        out.append(st.step_logits(r.query_pos))
        st.commit(r.committed_pos, r.committed_tok)
    return st, out


def test_switches_cache_are_exact():
    """Caching the prompt and the decoded responses changes only the cost: with truncation on,
    all four cache settings give the sparse step's decode-set logits (fp64, 1e-10)."""
    m = tiny_model()
    prompt, plan, st, recs = _tiny_run(m)
    for cp, cr, tr in SWITCHES:
        if not tr:
            continue
        _, out = _replay_switched(m, prompt, st.Lg, recs, cp, cr, tr)
        err = max(float(np.max(np.abs(o - r.logits))) for o, r in zip(out, recs))
        assert err < 1e-10, (cp, cr, tr, err)


def test_switches_without_truncation_match_the_one_forward_form():
    """Without truncation the step's other masks are mask rows of the step (the decode set sees
    them), so the logits change; every cache setting still reproduces the one-forward
    step-labelled form of the same rows exactly."""
    m = tiny_model()
    prompt, plan, st, recs = _tiny_run(m)
    P, Lg = len(prompt), st.Lg
    ref = None
    for cp, cr, tr in SWITCHES:
        if tr:
            continue
        _, out = _replay_switched(m, prompt, Lg, recs, cp, cr, tr)
        if ref is None:
            ref = out
            # differs from the truncated step on some step (the other masks are visible)
            assert max(float(np.max(np.abs(o - r.logits))) for o, r in zip(out, recs)) > 1e-6
        assert max(float(np.max(np.abs(o - q))) for o, q in zip(out, ref)) < 1e-10
    # one forward per step: all clean rows so far + this step's masks (C first) + registers
    sw = oracle.Switched(m, prompt, Lg, cache_prompt=False, cache_res=False, truncate=False)
    for r, o in zip(recs, ref):
        rows, c0, _ = sw.rows(r.query_pos)
        lg = oracle.forward_stepcausal(m, rows.ids, rows.pos, rows.types, rows.labels,
                                       np.arange(c0, c0 + len(r.query_pos)))
        assert float(np.max(np.abs(lg - o))) < 1e-10
        sw.step_k += 1
        sw.commit(r.committed_pos, r.committed_tok)


def test_switches_visible_keys_are_one_range_per_row():
    """With the step rows ordered by label, every row's visible keys over [cache | step rows]
    form one contiguous range [lo, hi): lo = cache length for prompt rows recomputed next to a
    cache of decoded tokens, else 0; hi = cache length + (the step rows with label <= the row's
    label for clean rows, all step rows for mask and register rows).  Checked against the
    predicate for every switch setting and step."""
    m = tiny_model()
    prompt, plan, st, recs = _tiny_run(m)
    for cp, cr, tr in SWITCHES:
        sw = oracle.Switched(m, prompt, st.Lg, cache_prompt=cp, cache_res=cr, truncate=tr)
        for r in recs:
            rows, c0, keep = sw.rows(r.query_pos)
            ctx = sw.ctx
            kt = np.concatenate([sw.c_types, rows.types])
            kl = np.concatenate([sw.c_labels, rows.labels])
            vis = oracle.cross_mask(rows.types, rows.labels, kt, kl)
            clean = (rows.types == oracle.PROMPT) | (rows.types == oracle.CLEAN)
            for i in range(rows.n):
                idx = np.flatnonzero(vis[i])
                lo, hi = int(idx[0]), int(idx[-1]) + 1
                assert hi - lo == len(idx), (cp, cr, tr, i)          # contiguous
                exp_lo = ctx if (clean[i] and rows.labels[i] == 0 and not cp and ctx > 0) else 0
                if clean[i]:
                    exp_hi = ctx + int(np.sum(clean & (rows.labels <= rows.labels[i])))
                else:
                    exp_hi = ctx + rows.n
                assert (lo, hi) == (exp_lo, exp_hi), (cp, cr, tr, i, lo, hi, exp_lo, exp_hi)
            sw.step_logits(r.query_pos)
            sw.commit(r.committed_pos, r.committed_tok)


# ------------------------------------------------------------------------------------------
# Length-token variant (the 0-register row of the register-count ablation): one [LEN] row at
# L+1 instead of registers, under the masked block's attention rule.
# ------------------------------------------------------------------------------------------

def test_length_token_variant_rows():
    """The worked example with the length token: 3 clean + 4 masks + one [LEN] row at L+1 = 8
    (the sparse sequence carries the clean tokens, their positions and the length)."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    vocab = {w: i for i, w in enumerate(["I", "have", "dog"])}
    shape = synth.ModelShape(1, 8, 1, 8, 8, 3, n_reg=0, dtype=synth.F32, len_token=True)
    L = g["length"]
    grid = np.full(L, -1)
    for t, p in zip(g["clean"], g["positions"]):
        grid[p - 1] = vocab[t]
    masked = [p for p in range(1, L + 1) if p not in g["positions"]]
    rows = oracle.pack_step(shape, 0, L, grid, g["positions"], masked, k=2)
    assert rows.n == len(g["positions"]) + len(masked) + 1
    assert rows.ids[-1] == shape.len_id == shape.vocab + 1
    assert rows.pos[-1] == L + 1 and rows.types[-1] == oracle.REG and rows.labels[-1] == 2
    with pytest.raises(ValueError):
        synth.ModelShape(1, 8, 1, 8, 8, 3, n_reg=4, len_token=True)


def test_length_token_training_form_equals_incremental():
    """Invariant (b) with the length-token variant: the one-forward trajectory form reproduces
    every cached step, and the [LEN] row does condition the decode set (dropping it changes
    the logits)."""
    m = tiny_model(n_reg=0, len_token=True)
    assert check_training_equals_incremental(m) < 1e-10
    prompt, plan, st, recs = _tiny_run(m)
    bare = oracle.Model(synth.make_weights(tiny_shape(0), 7, gain_std=0.1, std=0.25))
    st0, recs0 = oracle.generate(bare, prompt, st.Lg, plan, max_steps=1)
    assert np.max(np.abs(recs0[0].logits - recs[0].logits)) > 1e-3


def test_semiar_blocks_in_any_order():
    """Semi-AR decoding with the blocks taken in a permuted order (a bidirectional task may
    decode a middle block first): every step commits inside its own block, the run fills the
    grid, the one-forward training form reproduces every step (invariant (b)), and a block
    decoded after its right neighbour is conditioned by it (the logits differ from the
    left-to-right run's)."""
    wl = synth.WORKLOADS["tiny-bf16-semiar"]
    m = oracle.Model(synth.make_weights(wl.model, wl.seed))
    prompt = synth.make_prompt(wl)
    base = synth.make_plan(wl)
    n_blocks = wl.gen_len // wl.block
    perm = dataclasses.replace(base, block_order=np.array([1, 2, 0][:n_blocks]))
    st, recs = oracle.generate(m, prompt, wl.gen_len, perm)
    assert (st.grid >= 0).all()
    for r in recs:
        lo, hi = synth.semiar_block(perm, wl.prompt_len, r.k)
        assert ((r.committed_pos >= lo) & (r.committed_pos < hi)).all()
    first = synth.semiar_block(perm, wl.prompt_len, 1)
    assert first[0] == wl.prompt_len + 1 + wl.block
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, wl.model, wl.gen_len, recs)
    rows = np.concatenate([qrows[r.k] for r in recs])
    lg = oracle.forward_stepcausal(m, ids, pos, types, labels, rows)
    assert np.max(np.abs(lg - np.concatenate([r.logits for r in recs]))) < 1e-10
    # block 0 is decoded last here, after blocks 1 and 2: its first step differs from the
    # left-to-right run's first step (which saw no generated tokens)
    _, recs_lr = oracle.generate(m, prompt, wl.gen_len, base, max_steps=1)
    k0 = 2 * wl.steps_per_block + 1
    assert np.array_equal(recs[k0 - 1].query_pos, recs_lr[0].query_pos)
    assert np.max(np.abs(recs[k0 - 1].logits - recs_lr[0].logits)) > 1e-3
