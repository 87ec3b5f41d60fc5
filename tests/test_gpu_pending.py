"""GPU parity cases for device modes that have not yet run on a B200: the length-token variant
(n_reg = SMDM_REG_LEN), semi-AR plans with the blocks in a permuted order, and the Table-6
speed switches (smdm_step_switched).  They carry the
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


def test_pair_attention_kernel_parity():
    """The CTA-pair attention kernel (SMDM_ATTN_PAIR=1, d_head 128): the d_head-128 parity cases
    — sparse runs, the training form, the dense step, bidirectional tasks, the T2I runs — in a
    child process with the switch on (it is read once per process)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SMDM_ATTN_PAIR="1")
    sel = ("tiny-bf16-cos or batched or bidirectional or register_count or config_t2i or "
           "config_D_batch4 or dense_step_config_C")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-k", sel,
                        os.path.join(root, "tests", "test_gpu_parity.py"),
                        os.path.join(root, "tests", "test_gpu_full_configs.py")],
                       env=env, cwd=root, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]


def test_training_form_key_bounds_parity():
    """The training form with per-row key bounds (SMDM_TRAIN_BOUND=1): its GPU parity cases —
    the tiny shapes, the text model's first block and the allocation-free entry point — in a
    child process with the switch on (it is read once per process)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SMDM_TRAIN_BOUND="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-k",
                        "forward_stepcausal or noalloc",
                        os.path.join(root, "tests", "test_gpu_parity.py"),
                        os.path.join(root, "tests", "test_gpu_full_configs.py"),
                        os.path.join(root, "tests", "test_zz_no_alloc.py")],
                       env=env, cwd=root, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]


def test_split_qkv_parity():
    """The split QKV path (SMDM_QKV_SPLIT=1: an additive fp32 QKV GEMM over all SMs and a
    finalize kernel for RoPE and the K/V append): the bf16 GPU parity cases — sparse runs of
    both head sizes, the batched step, the dense step and the training form — in a child
    process with the switch on (it is read once per process)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SMDM_QKV_SPLIT="1")
    sel = ("bf16 or batched or bidirectional or register_count or config_t2i or "
           "config_B_text or dense_step_config_C or forward_stepcausal_config_B or edge")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-k", sel,
                        os.path.join(root, "tests", "test_gpu_edge_cases.py"),
                        os.path.join(root, "tests", "test_gpu_parity.py"),
                        os.path.join(root, "tests", "test_gpu_full_configs.py")],
                       env=env, cwd=root, capture_output=True, text=True, timeout=2400)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
