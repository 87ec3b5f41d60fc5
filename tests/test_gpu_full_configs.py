"""GPU parity at the full workload sizes (the same bar as test_gpu_parity.py).

The fp64 oracle is exact but slow at d=4096, so the large workloads compare logits on their
first sampling steps (prefill + steps, computed by the oracle's incremental form from scratch)
and check packing, the commit rule and the scatter bit-exactly over every step of the run.  The
late steps, where the step's rows (up to 265 per sequence, over 1000 for a batch of four) and
the KV cache (over 4000 keys, split over several key ranges) are largest, compare logits through
the oracle's training form: one forward over the teacher-forced trajectory gives every asked
step's logits (the two forms agree exactly, invariant (b)).
"""
import numpy as np
import pytest
import torch

import masked_discrete_diffusion_sparse_b200 as smdm
import oracle
import synth
from smdm_testlib import Runner, i32, logit_err, run_teacher_forced

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from masked_discrete_diffusion_sparse_b200 import build
    build.build()


def _check(checks, tol):
    print(f"max logit error {max(c.err for c in checks):.3g} (tol {tol}) over {len(checks)} steps")
    for c in checks:
        assert c.rows_exact, f"step {c.k}: packed rows differ from the oracle"
        assert c.err <= tol, f"step {c.k}: logit error {c.err:.3g} > {tol}"
        assert c.tok_ok, f"step {c.k}: inadmissible token"
        assert c.commit_ok, f"step {c.k}: committed set / scatter wrong"


def test_config_B_text_semiar_full_run():
    """8-layer d=1024 bf16, prompt 512 Zipf tokens, 4 blocks x 16 steps, top-8 confidence."""
    r = Runner(synth.WORKLOADS["B"])
    try:
        checks, grids, _ = run_teacher_forced(r)
        _check(checks, r.tol)
        assert (grids.cpu().numpy() >= 0).all()
    finally:
        r.close()


@pytest.mark.parametrize("name,logit_steps,late", [("C", 2, [32, 64]), ("D", 1, [32, 64])])
def test_config_t2i_full_run(name, logit_steps, late):
    """T2I 1024 / 4096 tokens, all 64 steps: logits on the first steps and on a middle and the
    last step (4096 tokens: 265 rows against a 4252-key cache at step 64), structure on all."""
    r = Runner(synth.WORKLOADS[name])
    try:
        checks, grids, _ = run_teacher_forced(r, logit_steps=logit_steps, late_steps=late)
        _check(checks, r.tol)
        for k in late:
            print(f"{name} step {k}: logit error {checks[k - 1].err:.3g}")
        assert (grids.cpu().numpy() >= 0).all()
    finally:
        r.close()


def test_config_D_batch4_full_run():
    """Four independent 4096-token sequences in one forward per step, all 64 steps: logits on
    step 1 for all four and on step 64 (1060 batched rows: the GEMMs' row dimension spans
    several row tiles) for the first and the last sequence."""
    wl = synth.WORKLOADS["D4"]
    r = Runner(wl, batch=4)
    try:
        checks, grids, _ = run_teacher_forced(r, logit_steps=1, late_steps=[64],
                                              late_seqs=[0, 3])
        _check(checks, r.tol)
        print(f"D x4 step 64: logit error {checks[63].err:.3g}")
        assert (grids.cpu().numpy() >= 0).all()
    finally:
        r.close()


def test_config_E_editing_to_step_32():
    """8 layers, prompt 256 text + 4096 reference-image tokens prefilled: logits on step 1 and
    on step 32 (a 5400-key cache), structure on steps 1-32."""
    r = Runner(synth.WORKLOADS["E"])
    try:
        checks, _, _ = run_teacher_forced(r, max_steps=32, logit_steps=1, late_steps=[32])
        _check(checks, r.tol)
        print(f"E step 32: logit error {checks[31].err:.3g}")
    finally:
        r.close()


def test_dense_step_config_C():
    """The dense comparator at T2I-1024 size: all 1152 rows, full attention, Lg x V logits."""
    wl = synth.WORKLOADS["C"]
    r = Runner(wl)
    try:
        P, Lg, V = wl.prompt_len, wl.gen_len, wl.model.vocab
        plan = r.plans[0]
        grid = torch.empty(Lg, dtype=torch.int32, device="cuda")
        r.model.smdm_prefill(0, i32(r.prompts[0]), Lg, grid)
        qp = plan.query_positions(1)
        logits = torch.empty((Lg, V), dtype=torch.float32, device="cuda")
        r.model.smdm_dense_step(dict(seq=0, query_pos=i32(qp), n_query=len(qp),
                                     policy=smdm.SMDM_POLICY_ALL), logits=logits)
        torch.cuda.synchronize()
        assert r.model.smdm_device_status() == 0
        ref = oracle.dense_step_logits(r.om, r.prompts[0], np.full(Lg, -1))
        err = logit_err(logits.cpu().numpy().astype(np.float64), ref)
        print(f"dense C logit error {err:.3g}")
        assert err <= r.tol
    finally:
        r.close()


def test_forward_stepcausal_config_B_first_block():
    """Training form over a step-labelled B trajectory (first block, 16 steps) in one forward."""
    wl = synth.WORKLOADS["B"]
    w = synth.make_weights(wl.model, wl.seed)
    om = oracle.Model(w)
    prompt = synth.make_prompt(wl)
    st, recs = oracle.generate(om, prompt, wl.gen_len, synth.make_plan(wl), max_steps=16)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, wl.model, wl.gen_len, recs)
    rows = np.concatenate([qrows[k] for k in sorted(qrows)])
    r = Runner(wl, train_rows=len(ids), weights=w)
    try:
        out = torch.empty((len(rows), wl.model.vocab), dtype=torch.float32, device="cuda")
        r.model.smdm_forward_stepcausal(i32(ids), i32(pos), i32(types), i32(labels), i32(rows), out)
        torch.cuda.synchronize()
        assert r.model.smdm_device_status() == 0
        inc = np.concatenate([rec.logits for rec in recs])
        err = logit_err(out.cpu().numpy().astype(np.float64), inc)
        print(f"training-form B logit error {err:.3g} over {len(ids)} rows")
        assert err <= r.tol
    finally:
        r.close()
