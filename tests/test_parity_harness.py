"""The teacher-forced parity harness (`smdm_testlib.run_teacher_forced`) run on CPU against a
stand-in device: an object with the binding's method names whose "kernels" are a second,
independent fp64 oracle state.  A faithful stand-in passes every check; stand-ins with one
planted fault each (a wrong cache length, a wrong packed row, a wrong token, perturbed logits)
fail the check that covers it.  This tests the harness's judgement, not the CUDA path."""
import types

import numpy as np
import pytest
import torch

import oracle
import smdm_testlib
import synth


class _TorchOnCPU:
    """torch with device arguments dropped and a no-op synchronize (the harness asks for CUDA
    tensors; the stand-in device works on host tensors)."""

    def __getattr__(self, name):
        return getattr(torch, name)

    @staticmethod
    def full(*a, device=None, **k):
        return torch.full(*a, **k)

    @staticmethod
    def empty(*a, device=None, **k):
        return torch.empty(*a, **k)

    @staticmethod
    def as_tensor(*a, device=None, **k):
        return torch.as_tensor(*a, **k)

    cuda = types.SimpleNamespace(synchronize=lambda: None)


class StandIn:
    """Emulates the library's sampling entry points with its own oracle states."""

    def __init__(self, om, fault=None, fault_step=2):
        self.om, self.fault, self.fault_step = om, fault, fault_step
        self.st, self.grids, self.rows = {}, {}, None

    def smdm_prefill(self, seq, prompt, gen_len, grid, stream=None):
        self.st[seq] = oracle.Incremental(self.om, prompt.numpy().astype(np.int64), gen_len)
        self.grids[seq] = grid
        grid.fill_(-1)

    def smdm_prefill_given(self, seq, prompt, gen_len, given_pos, given_tok, grid, stream=None):
        self.st[seq] = oracle.Incremental(self.om, prompt.numpy().astype(np.int64), gen_len,
                                          given_pos.numpy(), given_tok.numpy())
        self.grids[seq] = grid
        grid.copy_(torch.as_tensor(self.st[seq].grid, dtype=torch.int32))

    def smdm_step(self, descs, logits=None, tok=None, conf=None, stream=None):
        packs, off = [], 0
        for d in descs:
            st = self.st[d["seq"]]
            if d.get("query_pos") is not None:
                qp = d["query_pos"].numpy().astype(np.int64)
            else:
                qp = oracle.semiar_queries(st.grid, st.P, d["block_lo"], d["block_hi"])
            pk = st.pack(qp)
            k = st.step_k + 1
            if self.fault == "rows" and k == self.fault_step:
                pk.pos = pk.pos.copy()
                pk.pos[-1] += 1
            packs.append(pk)
            lg = st.step_logits(qp)
            if self.fault == "logits" and k == self.fault_step:
                lg = lg + 0.5 * max(1.0, float(np.max(np.abs(lg))))
            policy = oracle.POLICY_TOPN if d["policy"] == 1 else oracle.POLICY_ALL
            tk, cf, rows = oracle.unmask(lg, policy, d.get("n_commit", 0))
            if self.fault == "token" and k == self.fault_step:
                tk = tk.copy()
                tk[0] = int(np.argmin(lg[0]))
            st.commit(qp[rows], tk[rows])
            self.grids[d["seq"]].copy_(torch.as_tensor(st.grid, dtype=torch.int32))
            n = len(qp)
            logits[off:off + n] = torch.as_tensor(lg, dtype=torch.float32)
            tok[off:off + n] = torch.as_tensor(tk, dtype=torch.int32)
            conf[off:off + n] = torch.as_tensor(cf, dtype=torch.float32)
            off += n
        self.rows = packs

    def smdm_debug_rows(self, ids=None, pos=None, types=None, labels=None, stream=None):
        cat = lambda f: torch.as_tensor(np.concatenate([getattr(p, f) for p in self.rows]),
                                        dtype=torch.int32)
        n = sum(p.n for p in self.rows)
        for dst, f in ((ids, "ids"), (pos, "pos"), (types, "types"), (labels, "labels")):
            dst[:n] = cat(f)
        return n

    def smdm_device_status(self, stream=None):
        return 0

    def smdm_context_length(self, seq):
        n = len(self.st[seq].c_types)
        return n + 1 if self.fault == "ctx" and self.st[seq].step_k >= self.fault_step else n


def _runner(name, fault=None, tasks=None):
    wl = synth.WORKLOADS[name]
    r = types.SimpleNamespace()
    r.wl, r.batch, r.tasks = wl, 1, tasks
    r.w = synth.make_weights(wl.model, wl.seed, gain_std=0.02)
    r.om = oracle.Model(r.w)
    r.plans = [t.plan for t in tasks] if tasks else [synth.make_plan(wl, 0)]
    r.prompts = [synth.make_prompt(wl, 0)]
    r.tol = smdm_testlib.TOL[wl.model.dtype]
    # the stand-in device runs its own oracle model from the same weights
    r.model = StandIn(oracle.Model(r.w), fault)
    return r


@pytest.fixture(autouse=True)
def _cpu_torch(monkeypatch):
    monkeypatch.setattr(smdm_testlib, "torch", _TorchOnCPU())


@pytest.mark.parametrize("name", ["tiny-f32-cos", "tiny-bf16-semiar"])
def test_faithful_device_passes_every_check(name):
    checks, grids, states = smdm_testlib.run_teacher_forced(_runner(name), max_steps=4)
    assert len(checks) == 4
    for c in checks:
        assert c.rows_exact and c.tok_ok and c.commit_ok and c.err < 1e-6, c


def test_faithful_device_passes_a_bidirectional_task():
    wl = synth.WORKLOADS["tiny-f32-cos"]
    task = synth.make_bidir_task(wl, "infill")
    checks, _, _ = smdm_testlib.run_teacher_forced(_runner("tiny-f32-cos", tasks=[task]),
                                                   max_steps=3)
    assert all(c.rows_exact and c.tok_ok and c.commit_ok for c in checks)


@pytest.mark.parametrize("fault,field", [("ctx", "rows_exact"), ("rows", "rows_exact"),
                                         ("token", "tok_ok"), ("logits", "err")])
def test_planted_device_fault_is_caught(fault, field):
    checks, _, _ = smdm_testlib.run_teacher_forced(_runner("tiny-f32-cos", fault), max_steps=3)
    bad = checks[1]   # faults are planted at step 2
    good = checks[0]
    assert good.rows_exact and good.tok_ok and good.commit_ok and good.err < 1e-6
    if field == "err":
        assert bad.err > smdm_testlib.TOL[synth.F32]
    else:
        assert not getattr(bad, field)


@pytest.mark.parametrize("name", ["tiny-f32-cos", "tiny-bf16-semiar"])
def test_late_steps_reference_matches_the_incremental_logits(name):
    """Late-step logits judged through one training-form forward of the oracle (no incremental
    oracle run up to them): the faithful stand-in's incremental logits agree to fp64 rounding."""
    r = _runner(name)
    checks, _, _ = smdm_testlib.run_teacher_forced(r, logit_steps=1, late_steps=[3, 6])
    assert len(checks) == r.plans[0].n_steps
    for k in (3, 6):
        c = checks[k - 1]
        assert c.rows_exact and c.tok_ok and c.commit_ok and c.err < 1e-6, c


def test_planted_late_step_logit_fault_is_caught():
    r = _runner("tiny-f32-cos", "logits")
    r.model.fault_step = 5
    checks, _, _ = smdm_testlib.run_teacher_forced(r, logit_steps=1, late_steps=[4, 5])
    assert checks[3].err < 1e-6
    assert checks[4].err > smdm_testlib.TOL[synth.F32]


def test_late_steps_with_a_bidirectional_task():
    wl = synth.WORKLOADS["tiny-f32-cos"]
    task = synth.make_bidir_task(wl, "inpaint")
    r = _runner("tiny-f32-cos", tasks=[task])
    checks, _, _ = smdm_testlib.run_teacher_forced(r, logit_steps=0, late_steps=[2, 4])
    for k in (2, 4):
        assert checks[k - 1].err < 1e-6 and checks[k - 1].tok_ok
