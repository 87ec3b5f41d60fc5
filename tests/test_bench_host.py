"""Host-side pieces of bench.py that shape the measured workloads (CPU)."""
import importlib.util
import os

import numpy as np

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_training_form_rows_match_the_oracle_trajectory():
    """bench --form training builds the whole-trajectory training-form rows itself; as a
    multiset of (position, type, label) rows they equal the oracle's trajectory of a finished
    run with the same plan (the order of rows does not matter to the predicate)."""
    b = _bench()
    wl = synth.WORKLOADS["tiny-f32-cos"]
    plan = synth.make_plan(wl, 0)
    prompt = synth.make_prompt(wl, 0)
    ids, pos, types, labels, lrows = b.trajectory_rows(wl, plan, prompt, 0)
    om = oracle.Model(synth.make_weights(wl.model, wl.seed))
    st, recs = oracle.generate(om, prompt, wl.gen_len, plan)
    o_ids, o_pos, o_types, o_labels, o_q = oracle.trajectory(prompt, wl.model, wl.gen_len, recs)
    mine = sorted(zip(pos.tolist(), types.tolist(), labels.tolist()))
    ref = sorted(zip(o_pos.tolist(), o_types.tolist(), o_labels.tolist()))
    assert mine == ref
    # logit rows are exactly the mask copies, one per generated position
    assert (types[lrows] == 2).all() and len(lrows) == wl.gen_len
    assert sorted(pos[lrows].tolist()) == list(range(wl.prompt_len + 1,
                                                     wl.prompt_len + wl.gen_len + 1))
    # non-mask ids: prompt and registers as the oracle has them
    reg = types == 3
    assert (ids[reg] >= wl.model.vocab + 2).all()
    assert (ids[types == 0] == np.asarray(prompt)).all()


def test_step_shapes_cover_every_generated_token():
    b = _bench()
    for name in ("C", "D"):
        wl = synth.WORKLOADS[name]
        plan = synth.make_plan(wl, 0)
        shapes = b.step_shapes(wl, plan)
        assert len(shapes) == wl.n_steps
        assert sum(q for (_, q, _, _) in shapes) == wl.gen_len
        for (R, q, ctx, n_new) in shapes:
            assert R == n_new + q + wl.model.n_reg
