"""The allocation-free training-form forward, checked against the handle-based one and the
oracle.

smdm_forward_stepcausal_noalloc is for callers that cannot allocate device memory when they
need a forward (a frozen allocator, a plug-in that is only handed pointers): it keeps all its
scratch in a static array inside the library.  This file is collected last so that a failure
here cannot hide any other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import masked_discrete_diffusion_sparse_b200 as smdm
import oracle
import synth
from smdm_testlib import config_for, i32, logit_err, token_admissible, upload_weights, TOL

pytestmark = pytest.mark.gpu


def test_noalloc_forward_matches_handle_forward_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from masked_discrete_diffusion_sparse_b200 import build
    build.build()
    wl = synth.WORKLOADS["tiny-bf16-cos"]
    w = synth.make_weights(wl.model, wl.seed)
    om = oracle.Model(w)
    prompt = synth.make_prompt(wl)
    st, recs = oracle.generate(om, prompt, wl.gen_len, synth.make_plan(wl), max_steps=2)
    ids, pos, types, labels, qrows = oracle.trajectory(prompt, wl.model, wl.gen_len, recs)
    rows = np.concatenate([qrows[k] for k in sorted(qrows)])
    dev_w = upload_weights(w)
    cfg = config_for(wl, train_rows=len(ids))
    args = [i32(ids), i32(pos), i32(types), i32(labels), i32(rows)]
    model = smdm.Model(cfg, dev_w)
    try:
        ref = torch.empty((len(rows), wl.model.vocab), dtype=torch.float32, device="cuda")
        model.smdm_forward_stepcausal(*args, ref)
        torch.cuda.synchronize()
        ref_np = ref.cpu().numpy().astype(np.float64)
    finally:
        model.close()
    tol = TOL[wl.model.dtype]
    for call in range(2):
        out = torch.full((len(rows), wl.model.vocab), float("nan"), dtype=torch.float32,
                         device="cuda")
        smdm.smdm_forward_stepcausal_noalloc(cfg, dev_w, *args, out)
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all(), f"call {call}: non-finite logits"
        err = logit_err(got, ref_np)
        assert err <= tol, f"call {call}: {err:.3g} > {tol}"
        # and against the oracle's incremental logits of the same two steps (invariant (b)),
        # with every row's argmax admissible under the lowest-id tie rule
        inc = np.concatenate([rec.logits for rec in recs])
        err_o = logit_err(got, inc)
        assert err_o <= tol, f"call {call}: {err_o:.3g} > {tol} against the oracle"
        assert token_admissible(np.argmax(got, axis=1), inc, tol).all()
