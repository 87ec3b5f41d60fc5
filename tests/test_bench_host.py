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
            assert R == n_new + q + wl.model.n_tail


def test_streamed_parameters_per_step():
    """Weights streamed by one sampling step (every layer plus the LM head) for the five model
    shapes: 1.84 M, 135.5 M, 843.1 M (both text-to-image sizes) and 1652.6 M parameters."""
    b = _bench()
    # (millions, half a unit of the last digit given)
    expect = {"A": (1.84, 0.005), "B": (135.5, 0.05), "C": (843.1, 0.05), "D": (843.1, 0.05),
              "E": (1652.6, 0.05)}
    for name, (n, half) in expect.items():
        m = synth.WORKLOADS[name].model
        got = (m.n_layers * b.layer_params(m) + m.vocab * m.d_model) / 1e6
        assert abs(got - n) <= half, (name, got)


def _cache_before(P, recs, k):
    """(types, labels) of the oracle's KV cache before step k: the prompt, then the tokens
    committed at steps 1..k-2 (the ones of step k-1 are step k's new-cache rows)."""
    types = [oracle.PROMPT] * P
    labels = [0] * P
    for r in recs[:max(k - 2, 0)]:
        types += [oracle.CLEAN] * len(r.committed_pos)
        labels += [r.k] * len(r.committed_pos)
    return np.array(types), np.array(labels)


def test_step_shapes_and_attention_work_match_the_oracle_run():
    """The bench's per-step shapes (rows, decode rows, cache length, new-cache rows) and its
    attention work (sum over rows of visible keys) equal what the oracle's sampling run packs
    and what its step-causal predicate allows, for an order plan and a semi-AR plan."""
    b = _bench()
    for name in ("tiny-f32-cos", "tiny-bf16-semiar"):
        wl = synth.WORKLOADS[name]
        plan = synth.make_plan(wl, 0)
        prompt = synth.make_prompt(wl, 0)
        om = oracle.Model(synth.make_weights(wl.model, wl.seed))
        st, recs = oracle.generate(om, prompt, wl.gen_len, plan)
        shapes = b.step_shapes(wl, plan)
        assert len(shapes) == len(recs)
        for (R, q, ctx, n_new), r in zip(shapes, recs):
            pk = r.packed
            assert R == pk.n and q == len(r.query_pos), (name, r.k)
            assert n_new == int(np.sum(pk.types == oracle.CLEAN)), (name, r.k)
            ct, cl = _cache_before(wl.prompt_len, recs, r.k)
            assert ctx == len(ct), (name, r.k)
            vis = oracle.cross_mask(pk.types, pk.labels, np.concatenate([ct, pk.types]),
                                    np.concatenate([cl, pk.labels]))
            kv_sum = n_new * (ctx + n_new) + (R - n_new) * (ctx + R)
            assert kv_sum == int(vis.sum()), (name, r.k)


def test_length_token_variant_rows_in_the_bench():
    """bench --n-reg 0 (the length-token variant): one [LEN] tail row per step, in the step
    shapes and in the training-form rows, equal to the oracle's trajectory of the same plan."""
    import dataclasses
    b = _bench()
    base = synth.WORKLOADS["tiny-f32-cos"]
    wl = dataclasses.replace(base, model=dataclasses.replace(base.model, n_reg=0, len_token=True))
    plan = synth.make_plan(wl, 0)
    for (R, q, ctx, n_new) in b.step_shapes(wl, plan):
        assert R == n_new + q + 1
    prompt = synth.make_prompt(wl, 0)
    ids, pos, types, labels, lrows = b.trajectory_rows(wl, plan, prompt, 0)
    om = oracle.Model(synth.make_weights(wl.model, wl.seed))
    st, recs = oracle.generate(om, prompt, wl.gen_len, plan)
    o_ids, o_pos, o_types, o_labels, _ = oracle.trajectory(prompt, wl.model, wl.gen_len, recs)
    tail = types == 3
    assert (ids[tail] == wl.model.vocab + 1).all() and (pos[tail] == wl.prompt_len +
                                                         wl.gen_len + 1).all()
    mine = sorted(zip(pos.tolist(), types.tolist(), labels.tolist()))
    ref = sorted(zip(o_pos.tolist(), o_types.tolist(), o_labels.tolist()))
    assert mine == ref
    assert sorted(ids[tail].tolist()) == sorted(o_ids[o_types == 3].tolist())


def test_class_roofline_agrees_with_the_gemm_byte_count():
    """With an unbounded tensor peak every class is HBM-bound, so the GEMM classes' roofline
    times times the bandwidth give back gemm_bytes_per_run, the bytes the bench's roofline
    line divides by the measured GEMM time."""
    b = _bench()
    for name in ("B", "D"):
        wl = synth.WORKLOADS[name]
        plan = synth.make_plan(wl, 0)
        hbm = 1000.0    # GB/s
        cls = b.class_roofline_ms(wl, plan, hbm, 1e12)
        gemm_ms = sum(cls[c] for c in ("gemm_qkv", "gemm_o", "gemm_gateup", "gemm_down",
                                       "gemm_lmhead"))
        assert abs(gemm_ms * 1e-3 * hbm * 1e9 / b.gemm_bytes_per_run(wl, plan) - 1) < 1e-5


def test_batched_cost_counts_every_sequence():
    """A batch of sequences: one prefill per sequence, then one forward per step whose rows are
    the sum of the sequences' rows; for one sequence the cost model is unchanged."""
    b = _bench()
    wl = synth.WORKLOADS["D4"]
    plans = [synth.make_plan(wl, i) for i in range(4)]
    fwd = list(b.run_forwards(wl, plans))
    assert len(fwd) == 4 + wl.n_steps
    singles = [list(b.run_forwards(wl, p)) for p in plans]
    for k in range(wl.n_steps):
        R, q, kv_sum, keys = fwd[4 + k]
        parts = [s[1 + k] for s in singles]
        assert R == sum(p[0] for p in parts) and q == sum(p[1] for p in parts)
        assert kv_sum == sum(p[2] for p in parts) and keys == sum(p[3] for p in parts)


def test_oracle_sample_states_have_the_run_shapes():
    """The CPU baseline times sampling steps on states built from the prefill (not on a full
    run): each such state packs the real step's row count and has the real cache length, for an
    order plan and a semi-AR plan; the sampled prefill and step times extrapolate to a full
    run through the per-step FLOPs."""
    b = _bench()
    for name in ("tiny-f32-cos", "tiny-bf16-semiar"):
        wl = synth.WORKLOADS[name]
        s = b.OracleSample(wl)
        plan = synth.make_plan(wl, 0)
        shapes = b.step_shapes(wl, plan)
        for k in s.steps:
            st, qp = s._state_before(k)
            R, q, ctx, n_new = shapes[k - 1]
            assert st.ctx == ctx and len(qp) == q and st.pack(qp).n == R, (name, k)
        out = s.run(1)
        assert out["value"] > 0 and set(out["sampled_s"]) == set(s.components)
        secs = out["sampled_s"]
        # doubling every sampled time halves the extrapolated rate
        assert abs(s.extrapolate({c: 2 * v for c, v in secs.items()})
                   - 2 * s.extrapolate(secs)) < 1e-9 * s.extrapolate(secs) + 1e-12


def test_oracle_sample_components_time_repeatedly_on_unchanged_states():
    """The single-threaded and the all-cores samples, and the reference arm's rotation, time the
    same step several times: each call must start from the same state (the step appends to its
    cache), so the cache length seen by a step is the same on every call."""
    b = _bench()
    wl = synth.WORKLOADS["tiny-f32-cos"]
    s = b.OracleSample(wl)
    s.run(1)
    s.run(2)
    k = s.steps[-1]
    st0, _ = s._states[k]
    ctx0 = st0.ctx
    for _ in range(3):
        s.time_component(f"step {k}", 1)
        st = s._states[k][0]
        assert st.ctx == ctx0 and all(len(kc) == ctx0 for kc in st.k_cache + st.v_cache)
