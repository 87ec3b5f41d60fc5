"""GPU parity cases for device modes that have not yet run on a B200: the length-token variant
(n_reg = SMDM_REG_LEN) and semi-AR plans with the blocks in a permuted order.  They carry the
`gpu_pending` marker instead of `gpu`, so the regular GPU suite does not select them; run them
with `pytest -m gpu_pending` on a B200, and move them to the `gpu` marker once green.  On a
machine without CUDA they skip."""
import dataclasses

import numpy as np
import pytest
import torch

import masked_discrete_diffusion_sparse_b200 as smdm
import synth
from smdm_testlib import Runner, i32, run_teacher_forced

pytestmark = pytest.mark.gpu_pending


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


def test_generate_with_block_order_equals_the_stepwise_run():
    """smdm_generate with a SEMIAR block order gives the same grid as the same plan driven step
    by step (both on the device; the kernels are deterministic)."""
    wl = synth.WORKLOADS["tiny-bf16-semiar"]
    plan = _permuted_semiar(wl)
    r = Runner(wl)
    r.plans = [plan]
    try:
        _, stepwise, _ = run_teacher_forced(r, logit_steps=0)
        grids = torch.empty((1, wl.gen_len), dtype=torch.int32, device="cuda")
        prompts = i32(np.asarray(r.prompts[0])[None, :])
        r.model.smdm_generate(prompts, wl.gen_len,
                              [dict(kind=smdm.SMDM_PLAN_SEMIAR, n_steps=plan.n_steps,
                                    block=plan.block, steps_per_block=plan.steps_per_block,
                                    commit=plan.commit,
                                    block_order=[int(b) for b in plan.block_order])], grids)
        torch.cuda.synchronize()
        assert r.model.smdm_device_status() == 0
        assert np.array_equal(grids.cpu().numpy()[0], stepwise.cpu().numpy()[0])
    finally:
        r.close()
