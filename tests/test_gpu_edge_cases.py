"""GPU parity on degenerate shapes of the sampling step: an empty prompt (nothing cached before
the first step) and one-token steps (a single query row, a single new-cache row), through the
C ABI against the fp64 oracle with the same bar as the other parity tests."""
import dataclasses

import pytest
import torch

import synth
from smdm_testlib import Runner, run_teacher_forced

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from masked_discrete_diffusion_sparse_b200 import build
    build.build()


def test_empty_prompt_one_token_steps():
    """P = 0 and 24 steps of one token: the first step attends over its own rows only (the
    cache is empty), every later step has one new-cache row and one query row."""
    base = synth.WORKLOADS["tiny-bf16-cos"]
    wl = dataclasses.replace(base, name="edge-p0-n1", prompt_len=0, gen_len=24, plan="perm",
                             n_steps=24, step_size=1, grid_side=0)
    r = Runner(wl)
    try:
        checks, grids, states = run_teacher_forced(r)
        for c in checks:
            assert c.rows_exact and c.tok_ok and c.commit_ok, f"step {c.k}"
            assert c.err <= r.tol, f"step {c.k}: logit error {c.err:.3g}"
        assert (grids.cpu().numpy() >= 0).all()
        assert len(checks) == 24
    finally:
        r.close()
