"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bar: packing, positions, labels, mask structure and the unmask scatter bit-exact; logits within
max-abs error tol * max(1, max|oracle logit|) with tol = 2e-2 for bf16 weights and 1e-4 for
fp32 weights; sampled tokens equal the oracle's argmax except where the oracle's top-2 gap is
below that tolerance.  Trajectories are teacher-forced: after every step the oracle adopts the
device's committed tokens when they are admissible.
"""
import dataclasses
import os

import numpy as np
import pytest
import torch

import masked_discrete_diffusion_sparse_b200 as smdm
import oracle
import synth
from smdm_testlib import Runner, i32, logit_err, run_teacher_forced

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from masked_discrete_diffusion_sparse_b200 import build
    build.build()


def _check_all(checks, tol):
    print(f"max logit error {max(c.err for c in checks):.3g} (tol {tol}) over {len(checks)} steps")
    for c in checks:
        assert c.rows_exact, f"step {c.k}: packed rows differ from the oracle"
        assert c.err <= tol, f"step {c.k}: logit error {c.err:.3g} > {tol}"
        assert c.tok_ok, f"step {c.k}: inadmissible token"
        assert c.commit_ok, f"step {c.k}: committed set / scatter wrong"


# ------------------------------------------------------------------------------------------
# mask structure
# ------------------------------------------------------------------------------------------

def _bitmap_to_bool(bm: np.ndarray, n: int) -> np.ndarray:
    words = (n + 31) // 32
    bm = bm.reshape(n, words).astype(np.uint64)
    out = np.zeros((n, n), dtype=bool)
    for j in range(n):
        out[:, j] = (bm[:, j // 32] >> np.uint64(j % 32)) & np.uint64(1)
    return out


def test_device_mask_predicate_matches_oracle():
    r = Runner(synth.WORKLOADS["tiny-f32-cos"])
    try:
        g = np.random.Generator(np.random.PCG64(3))
        for n in (9, 70, 133):
            types = g.integers(0, 4, n)
            labels = g.integers(0, 6, n)
            bm = torch.zeros(n * ((n + 31) // 32), dtype=torch.int32, device="cuda")
            r.model.smdm_debug_mask(i32(types), i32(labels), bm)
            got = _bitmap_to_bool(bm.cpu().numpy().view(np.uint32), n)
            np.testing.assert_array_equal(got, oracle.cross_mask(types, labels, types, labels))
        # the Figure-3 example
        lines = [l for l in open(os.path.join(GOLDEN, "fig3_visibility.txt")) if not l.startswith("#")]
        spec = [s.split() for s in lines[0].split(":", 1)[1].split("|")]
        tmap = {"PROMPT": 0, "CLEAN": 1, "MASK": 2, "REG": 3}
        types = [tmap[s[2]] for s in spec]
        labels = [int(s[3]) for s in spec]
        expect = np.array([[int(v) for v in l.split()[1:]] for l in lines[1:] if l.strip()], bool)
        n = len(types)
        bm = torch.zeros(n, dtype=torch.int32, device="cuda")
        r.model.smdm_debug_mask(i32(types), i32(labels), bm)
        np.testing.assert_array_equal(_bitmap_to_bool(bm.cpu().numpy().view(np.uint32), n), expect)
    finally:
        r.close()


# ------------------------------------------------------------------------------------------
# incremental sampling, teacher-forced
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny-f32-cos", "tiny-bf16-cos", "tiny-bf16-semiar"])
def test_sparse_run_tiny(name):
    wl = synth.WORKLOADS[name]
    r = Runner(wl)
    try:
        checks, grids, states = run_teacher_forced(r)
        _check_all(checks, r.tol)
        assert (grids.cpu().numpy() >= 0).all()
    finally:
        r.close()


@pytest.mark.parametrize("n_reg", [1, 32])
def test_sparse_run_register_count(n_reg):
    """Register-count variants of the sparse row set (the method uses 64 registers): n_reg
    register rows with ids REG_0.. at positions L+1..L+n_reg; same kernels, parity per step."""
    base = synth.WORKLOADS["tiny-bf16-cos"]
    wl = dataclasses.replace(base, name=f"{base.name}-reg{n_reg}",
                             model=dataclasses.replace(base.model, n_reg=n_reg))
    r = Runner(wl)
    try:
        checks, grids, states = run_teacher_forced(r)
        _check_all(checks, r.tol)
        assert (grids.cpu().numpy() >= 0).all()
    finally:
        r.close()


@pytest.mark.parametrize("kind", ["inpaint", "outpaint", "infill"])
def test_bidirectional_task_run(kind):
    """Bidirectional tasks (given generation tokens as block-0 clean rows, cached with the
    prompt): teacher-forced sampling of the remaining positions against the oracle."""
    wl = synth.WORKLOADS["tiny-bf16-cos"]
    task = synth.make_bidir_task(wl, kind)
    r = Runner(wl, tasks=[task])
    try:
        checks, grids, states = run_teacher_forced(r)
        _check_all(checks, r.tol)
        g = grids[0].cpu().numpy()
        assert (g >= 0).all()
        assert (g[task.preset_pos - wl.prompt_len - 1] == task.preset_tok).all()
    finally:
        r.close()


def test_sparse_run_batched_sequences():
    """Three sequences with different prompts and orders in one forward per step."""
    wl = synth.WORKLOADS["tiny-bf16-batch"]
    r = Runner(wl, batch=wl.batch)
    try:
        checks, grids, states = run_teacher_forced(r)
        _check_all(checks, r.tol)
    finally:
        r.close()


def test_sparse_run_config_A():
    """Tiny fp32 MDM (2 layers, d=256, vocab 1024, 8 steps of 32): every step at 1e-4."""
    wl = synth.WORKLOADS["A"]
    r = Runner(wl)
    try:
        checks, grids, states = run_teacher_forced(r)
        _check_all(checks, r.tol)
    finally:
        r.close()


# ------------------------------------------------------------------------------------------
# training (parallel) form
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny-f32-cos", "tiny-bf16-cos", "tiny-bf16-semiar"])
def test_forward_stepcausal_matches_oracle(name):
    wl = synth.WORKLOADS[name]
    w = synth.make_weights(wl.model, wl.seed, gain_std=0.02)
    om = oracle.Model(w)
    prompt = synth.make_prompt(wl)
    plan = synth.make_plan(wl)
    st, recs = oracle.generate(om, prompt, wl.gen_len, plan)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, wl.model, wl.gen_len, recs)
    rows = np.concatenate([qrows[r.k] for r in recs])
    ref = oracle.forward_stepcausal(om, ids, pos, types, labels, rows)
    r = Runner(wl, train_rows=len(ids), weights=w)
    try:
        out = torch.empty((len(rows), wl.model.vocab), dtype=torch.float32, device="cuda")
        r.model.smdm_forward_stepcausal(i32(ids), i32(pos), i32(types), i32(labels), i32(rows), out)
        torch.cuda.synchronize()
        assert r.model.smdm_device_status() == 0
        err = logit_err(out.cpu().numpy().astype(np.float64), ref)
        assert err <= r.tol, err
        # invariant (b) on the device: the same logits as the incremental oracle run
        inc = np.concatenate([rec.logits for rec in recs])
        assert logit_err(out.cpu().numpy().astype(np.float64), inc) <= r.tol
    finally:
        r.close()


# ------------------------------------------------------------------------------------------
# dense comparator
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny-f32-cos", "tiny-bf16-cos"])
def test_dense_step_matches_oracle(name):
    wl = synth.WORKLOADS[name]
    r = Runner(wl)
    try:
        P, Lg, V = wl.prompt_len, wl.gen_len, wl.model.vocab
        plan = r.plans[0]
        grid = torch.empty(Lg, dtype=torch.int32, device="cuda")
        r.model.smdm_prefill(0, i32(r.prompts[0]), Lg, grid)
        og = np.full(Lg, -1, dtype=np.int64)
        for k in range(1, 4):
            qp = plan.query_positions(k)
            logits = torch.empty((Lg, V), dtype=torch.float32, device="cuda")
            tok = torch.empty(len(qp), dtype=torch.int32, device="cuda")
            r.model.smdm_dense_step(dict(seq=0, query_pos=i32(qp), n_query=len(qp),
                                         policy=smdm.SMDM_POLICY_ALL), logits=logits, tok=tok)
            torch.cuda.synchronize()
            assert r.model.smdm_device_status() == 0
            ref = oracle.dense_step_logits(r.om, r.prompts[0], og)
            assert logit_err(logits.cpu().numpy().astype(np.float64), ref) <= r.tol
            g = grid.cpu().numpy()
            og[qp - P - 1] = g[qp - P - 1]   # adopt the device tokens
            assert (g[qp - P - 1] == tok.cpu().numpy()).all()
    finally:
        r.close()
