"""GPU parity of the step variants: the length-token variant (n_reg = SMDM_REG_LEN), semi-AR
plans with the blocks in a permuted order (stepwise and through smdm_generate), and the Table-6
speed switches (smdm_step_switched, five settings against oracle.Switched).  On a machine
without CUDA they skip."""
import dataclasses

import numpy as np
import pytest
import torch

import masked_discrete_diffusion_sparse_b200 as smdm
import synth
from smdm_testlib import Runner, i32, run_teacher_forced

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from masked_discrete_diffusion_sparse_b200 import build
    build.build()


def _check_all(checks, tol):
    for c in checks:
        assert c.rows_exact and c.tok_ok and c.commit_ok, f"step {c.k}"
        assert c.err <= tol, f"step {c.k}: logit error {c.err:.3g}"


def test_length_token_variant_run():
    """One [LEN] row (id V+1, position L+1) instead of registers, every step teacher-forced."""
    base = synth.WORKLOADS["tiny-bf16-cos"]
    wl = dataclasses.replace(base, name="tiny-bf16-cos-len",
                             model=dataclasses.replace(base.model, n_reg=0, len_token=True))
    r = Runner(wl)
    try:
        checks, grids, _ = run_teacher_forced(r)
        _check_all(checks, r.tol)
        assert (grids.cpu().numpy() >= 0).all()
    finally:
        r.close()


def _permuted_semiar(wl):
    plan = synth.make_plan(wl)
    n_blocks = wl.gen_len // wl.block
    order = np.roll(np.arange(n_blocks), -1)          # 1, 2, ..., 0
    return dataclasses.replace(plan, block_order=order)


def test_semiar_blocks_in_any_order_run():
    """Semi-AR with the first block decoded last, step by step through smdm_step."""
    wl = synth.WORKLOADS["tiny-bf16-semiar"]
    r = Runner(wl)
    r.plans = [_permuted_semiar(wl)]
    try:
        checks, grids, _ = run_teacher_forced(r)
        _check_all(checks, r.tol)
        assert (grids.cpu().numpy() >= 0).all()
    finally:
        r.close()


def test_generate_with_block_order_runs_the_plan():
    """smdm_generate with a SEMIAR block order: every position is decoded, and the rows of the
    run's last forward (its last step) are that of the plan's LAST block: new-cache rows and
    queries inside it, registers after L.  (The stepwise test above checks the same order's
    numerics against the oracle; two device runs are not compared bit for bit, because the
    residual GEMMs add K-split partial sums with fp32 atomics in no fixed order, so a near-tied
    argmax may go either way.)"""
    wl = synth.WORKLOADS["tiny-bf16-semiar"]
    plan = _permuted_semiar(wl)
    P, Lg = wl.prompt_len, wl.gen_len
    r = Runner(wl)
    r.plans = [plan]
    try:
        grids = torch.empty((1, Lg), dtype=torch.int32, device="cuda")
        prompts = i32(np.asarray(r.prompts[0])[None, :])
        r.model.smdm_generate(prompts, Lg,
                              [dict(kind=smdm.SMDM_PLAN_SEMIAR, n_steps=plan.n_steps,
                                    block=plan.block, steps_per_block=plan.steps_per_block,
                                    commit=plan.commit,
                                    block_order=[int(b) for b in plan.block_order])], grids)
        n = r.model.smdm_debug_rows()
        ids = torch.empty(n, dtype=torch.int32, device="cuda")
        pos, typ, lab = torch.empty_like(ids), torch.empty_like(ids), torch.empty_like(ids)
        r.model.smdm_debug_rows(ids, pos, typ, lab)
        torch.cuda.synchronize()
        assert r.model.smdm_device_status() == 0
        g = grids.cpu().numpy()[0]
        assert ((g >= 0) & (g < wl.model.vocab)).all()
        last = int(plan.block_order[-1])
        lo = P + 1 + last * plan.block
        pos, typ, lab = pos.cpu().numpy(), typ.cpu().numpy(), lab.cpu().numpy()
        gen_rows = typ != smdm.SMDM_TYPE_REG
        assert ((pos[gen_rows] >= lo) & (pos[gen_rows] < lo + plan.block)).all()
        assert (pos[~gen_rows] > P + Lg).all() and (lab == plan.n_steps).sum() >= 1
    finally:
        r.close()


@pytest.mark.parametrize("switches", [smdm.SMDM_SW_ALL,
                                      smdm.SMDM_SW_ALL & ~smdm.SMDM_SW_CACHE_PROMPT,
                                      smdm.SMDM_SW_ALL & ~smdm.SMDM_SW_CACHE_RES,
                                      smdm.SMDM_SW_ALL & ~smdm.SMDM_SW_TRUNCATE, 0])
def test_switched_steps_match_the_oracle(switches):
    """smdm_step_switched against oracle.Switched, step by step (teacher-forced): the rows as a
    set, the decode set's logits within tolerance, admissible tokens, the grid."""
    from smdm_testlib import config_for, logit_err, token_admissible, upload_weights, TOL
    import oracle
    wl = synth.WORKLOADS["tiny-bf16-cos"]
    P, Lg, V = wl.prompt_len, wl.gen_len, wl.model.vocab
    cp = bool(switches & smdm.SMDM_SW_CACHE_PROMPT)
    cr = bool(switches & smdm.SMDM_SW_CACHE_RES)
    tr = bool(switches & smdm.SMDM_SW_TRUNCATE)
    w = synth.make_weights(wl.model, wl.seed, gain_std=0.02)
    om = oracle.Model(w)
    plan = synth.make_plan(wl)
    prompt = synth.make_prompt(wl)
    cfg = config_for(wl)
    cfg.max_step_rows = cfg.max_rows = P + Lg + wl.model.n_tail
    model = smdm.Model(cfg, upload_weights(w))
    tol = TOL[wl.model.dtype]
    try:
        grid = torch.empty(Lg, dtype=torch.int32, device="cuda")
        model.smdm_prefill(0, i32(prompt), Lg, grid)
        st = oracle.Switched(om, prompt, Lg, cache_prompt=cp, cache_res=cr, truncate=tr)
        for k in range(1, plan.n_steps + 1):
            qp = np.asarray(plan.query_positions(k), dtype=np.int64)
            logits = torch.empty((len(qp), V), dtype=torch.float32, device="cuda")
            tok = torch.empty(len(qp), dtype=torch.int32, device="cuda")
            model.smdm_step_switched(dict(seq=0, query_pos=i32(qp), n_query=len(qp),
                                          policy=smdm.SMDM_POLICY_ALL), switches,
                                     logits=logits, tok=tok)
            R = model.smdm_debug_rows()
            ids = torch.empty(R, dtype=torch.int32, device="cuda")
            pos, typ, lab = torch.empty_like(ids), torch.empty_like(ids), torch.empty_like(ids)
            model.smdm_debug_rows(ids, pos, typ, lab)
            torch.cuda.synchronize()
            assert model.smdm_device_status() == 0
            rows, _, _ = st.rows(qp)
            got = sorted(zip(ids.cpu().tolist(), pos.cpu().tolist(), typ.cpu().tolist(),
                             lab.cpu().tolist()))
            ref_rows = sorted(zip(rows.ids.tolist(), rows.pos.tolist(), rows.types.tolist(),
                                  rows.labels.tolist()))
            assert got == ref_rows, f"step {k}: rows differ"
            ref = st.step_logits(qp)
            assert logit_err(logits.cpu().numpy().astype(np.float64), ref) <= tol, f"step {k}"
            tk = tok.cpu().numpy()
            assert token_admissible(tk, ref, tol).all(), f"step {k}"
            g = grid.cpu().numpy()
            assert (g[qp - P - 1] == tk).all()
            st.commit(qp, tk)          # teacher forcing
        assert np.array_equal(grid.cpu().numpy(), st.grid)
    finally:
        model.close()
