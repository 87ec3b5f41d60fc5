"""Helpers for the GPU parity tests: upload synthetic weights, size a handle for a workload,
and compare the CUDA path against the fp64 oracle step by step (teacher forcing)."""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np
import torch

import masked_discrete_diffusion_sparse_b200 as smdm
import oracle
import synth

TOL = {synth.BF16: 2e-2, synth.F32: 1e-4}


def upload_weights(w: synth.Weights, device="cuda") -> dict:
    bf16 = w.shape.dtype == synth.BF16

    def t(a):
        if bf16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)

    out = {"emb": t(w.emb), "final_norm": t(w.final_norm), "lm_head": t(w.lm_head)}
    for k in ("attn_norm", "w_qkv", "w_o", "mlp_norm", "w_gate", "w_up", "w_down"):
        out[k] = [t(a) for a in getattr(w, k)]
    return out


def step_rows_bound(wl: synth.Workload, plan: synth.Plan) -> int:
    if plan.kind == "order":
        n = list(plan.n_per_step)
        return max((n[i - 1] if i else 0) + n[i] for i in range(len(n))) + wl.model.n_tail
    return plan.commit + plan.block + wl.model.n_tail


def config_for(wl: synth.Workload, batch: int = 1, train_rows: int = 0,
               plans: Optional[List[synth.Plan]] = None) -> smdm.smdm_config:
    m = wl.model
    plans = plans or [synth.make_plan(wl, s) for s in range(batch)]
    msr = max(step_rows_bound(wl, p) for p in plans)
    L = wl.prompt_len + wl.gen_len
    max_rows = max(batch * msr, L, train_rows, 1)
    return smdm.make_config(m.n_layers, m.d_model, m.n_heads, m.d_head, m.d_ffn, m.vocab,
                            n_reg=smdm.SMDM_REG_LEN if m.len_token else m.n_reg,
                            dtype=smdm.SMDM_BF16 if m.dtype == synth.BF16 else smdm.SMDM_F32,
                            rope_theta=m.rope_theta, rms_eps=m.rms_eps, max_batch=batch,
                            max_len=L, max_step_rows=msr, max_rows=max_rows)


def i32(a, device="cuda") -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.int32), device=device)


def logit_err(g: np.ndarray, o: np.ndarray) -> float:
    """max |g - o| relative to the logit scale max(1, max |o|)."""
    return float(np.max(np.abs(g - o)) / max(1.0, float(np.max(np.abs(o)))))


def token_admissible(tok_dev: np.ndarray, ref_logits: np.ndarray, tol: float) -> np.ndarray:
    """Per row: the device token is the oracle argmax, or the oracle's top-2 gap is below the
    tolerance and the device token is inside the near-tie set."""
    scale = max(1.0, float(np.max(np.abs(ref_logits))))
    best = ref_logits.max(axis=1)
    ok = np.empty(len(tok_dev), dtype=bool)
    for r, t in enumerate(tok_dev):
        ok[r] = ref_logits[r, t] >= best[r] - tol * scale
    return ok


def topn_commit_admissible(ref_logits: np.ndarray, rows, n_commit: int, tol: float) -> bool:
    """A TOP-n commit set is admissible when it has min(n, rows) rows and every row in it has an
    oracle confidence within the tolerance of the oracle's n-th highest confidence: a swapped
    row is a near-tie.  The tolerance acts on the logit scale, so the confidence (a softmax
    maximum) may fall by a factor exp(-2 tol scale)."""
    _, oconf, _ = oracle.unmask(ref_logits, oracle.POLICY_TOPN, n_commit)
    n = min(n_commit, len(oconf))
    if len(rows) != n:
        return False
    nth = np.sort(oconf)[::-1][n - 1]
    scale = max(1.0, float(np.max(np.abs(ref_logits))))
    bound = nth * math.exp(-2 * tol * scale)
    return all(oconf[int(r)] >= bound for r in rows)


@dataclass
class StepCheck:
    k: int
    err: float
    rows_exact: bool     # packed rows and every sequence's KV-cache length, bit-exact
    tok_ok: bool
    commit_ok: bool


class Runner:
    """Drives one workload on the device and the oracle side by side."""

    def __init__(self, wl: synth.Workload, batch: int = 1, gain_std: float = 0.02,
                 train_rows: int = 0, weights: Optional[synth.Weights] = None,
                 tasks: Optional[List[synth.BidirTask]] = None):
        """tasks: one bidirectional task per sequence (given generation tokens + the plan over
        the other positions) instead of the workload's own plan."""
        self.wl = wl
        self.batch = batch
        self.w = weights or synth.make_weights(wl.model, wl.seed, gain_std=gain_std)
        self.om = oracle.Model(self.w)
        self.tasks = tasks
        self.plans = ([t.plan for t in tasks] if tasks else
                      [synth.make_plan(wl, s) for s in range(batch)])
        self.prompts = [synth.make_prompt(wl, s) for s in range(batch)]
        self.cfg = config_for(wl, batch, train_rows, self.plans)
        self.dev_w = upload_weights(self.w)
        self.model = smdm.Model(self.cfg, self.dev_w)
        self.tol = TOL[wl.model.dtype]

    def close(self):
        self.model.close()


def run_teacher_forced(r: Runner, max_steps: Optional[int] = None, check_rows: bool = True,
                       logit_steps: Optional[int] = None, late_steps: Sequence[int] = (),
                       late_seqs: Optional[Sequence[int]] = None):
    """Sparse sampling, batch of r.batch sequences in one forward per step, checked against the
    oracle's incremental run per sequence after every step.  Returns a list of StepCheck.

    logit_steps: compare logits only for the first `logit_steps` steps (the oracle's fp64
    forward is the expensive part at full model size); later steps still check packing, the
    commit rule and the scatter bit-exactly, with the oracle adopting the device's tokens.

    late_steps: steps after `logit_steps` whose logits are still compared, without running the
    oracle's incremental form up to them: the device's logits of those steps are kept, and after
    the run ONE training-form forward of the oracle per sequence (`oracle.trajectory` of the
    teacher-forced run + `oracle.forward_stepcausal`) gives every late step's reference logits.
    The two forms agree exactly (the method's invariant (b), pinned on the CPU), so this is the
    same comparison at a fraction of the oracle's cost.  late_seqs: the sequences checked this
    way (default: all)."""
    wl, P, Lg = r.wl, r.wl.prompt_len, r.wl.gen_len
    B = r.batch
    V = wl.model.vocab
    grids = torch.full((B, Lg), -7, dtype=torch.int32, device="cuda")
    states = []
    for s in range(B):
        if r.tasks:
            t = r.tasks[s]
            r.model.smdm_prefill_given(s, i32(r.prompts[s]), Lg, i32(t.preset_pos),
                                       i32(t.preset_tok), grids[s])
            states.append(oracle.Incremental(r.om, r.prompts[s], Lg, t.preset_pos, t.preset_tok))
        else:
            r.model.smdm_prefill(s, i32(r.prompts[s]), Lg, grids[s])
            states.append(oracle.Incremental(r.om, r.prompts[s], Lg))
    # Expected KV-cache length per sequence: block 0 after prefill; a step appends the tokens
    # committed at the step before it (its new-cache rows).
    ctx_exp = [len(st.c_types) for st in states]
    prev_commit = [0] * B
    n_steps = min(p.n_steps for p in r.plans)
    K = n_steps if max_steps is None else min(max_steps, n_steps)
    checks = []
    late = set(int(k) for k in late_steps)
    late_seqs = list(range(B)) if late_seqs is None else list(late_seqs)
    history = [[] for _ in range(B)]      # per sequence: StepRecord of every step (no logits)
    kept = {}                             # (seq, k) -> (device logits, device tokens)
    for k in range(1, K + 1):
        descs, qsets, packs = [], [], []
        for s in range(B):
            plan, st = r.plans[s], states[s]
            qp = oracle.query_set(plan, st, k)
            qsets.append(qp)
            packs.append(st.pack(qp))
            if plan.kind == "order":
                descs.append(dict(seq=s, query_pos=i32(qp), n_query=len(qp),
                                  policy=smdm.SMDM_POLICY_ALL, n_commit=len(qp)))
            else:
                lo, hi = synth.semiar_block(plan, P, k)
                descs.append(dict(seq=s, query_pos=None, n_query=len(qp), block_lo=lo,
                                  block_hi=hi, policy=smdm.SMDM_POLICY_TOPN,
                                  n_commit=plan.commit))
        nq = sum(len(q) for q in qsets)
        logits = torch.empty((nq, V), dtype=torch.float32, device="cuda")
        tok = torch.empty(nq, dtype=torch.int32, device="cuda")
        conf = torch.empty(nq, dtype=torch.float32, device="cuda")
        grid_before = grids.cpu().numpy().copy()
        r.model.smdm_step(descs, logits=logits, tok=tok, conf=conf)
        R = sum(p.n for p in packs)
        if check_rows:
            ids = torch.empty(R, dtype=torch.int32, device="cuda")
            pos, typ, lab = torch.empty_like(ids), torch.empty_like(ids), torch.empty_like(ids)
            n = r.model.smdm_debug_rows(ids, pos, typ, lab)
            assert n == R
        torch.cuda.synchronize()
        assert r.model.smdm_device_status() == 0
        lg = logits.cpu().numpy().astype(np.float64)
        tk = tok.cpu().numpy()
        grid_after = grids.cpu().numpy()
        rows_exact = True
        if check_rows:
            got = np.stack([ids.cpu().numpy(), pos.cpu().numpy(), typ.cpu().numpy(),
                            lab.cpu().numpy()])
            ref = np.concatenate([np.stack([p.ids, p.pos, p.types, p.labels]) for p in packs],
                                 axis=1)
            rows_exact = bool(np.array_equal(got, ref))
        off = 0
        err = 0.0
        tok_ok = True
        commit_ok = True
        with_logits = logit_steps is None or k <= logit_steps
        for s in range(B):
            st, qp = states[s], qsets[s]
            n_q = len(qp)
            tks = tk[off:off + n_q]
            if with_logits:
                ref = st.step_logits(qp)
                g = lg[off:off + n_q]
                err = max(err, logit_err(g, ref))
                tok_ok &= bool(token_admissible(tks, ref, r.tol).all())
            else:
                st.step_k += 1          # packing-only step: no fp64 forward
                ref = None
                if k in late and s in late_seqs:
                    kept[(s, k)] = (lg[off:off + n_q].copy(), tks.copy())
            qidx = {int(p): j for j, p in enumerate(qp)}
            newly = np.nonzero((grid_before[s] < 0) & (grid_after[s] >= 0))[0]
            # committed positions in query-row order (the order of next step's new-cache rows)
            newly = np.array(sorted(newly.tolist(), key=lambda i: qidx.get(i + P + 1, -1)),
                             dtype=np.int64)
            cpos = newly + P + 1
            ctok = grid_after[s][newly]
            # committed set: ALL -> every query; TOPN -> n_commit admissible rows
            if r.plans[s].kind == "order":
                commit_ok &= set(cpos.tolist()) == set(int(p) for p in qp)
            elif ref is None:
                commit_ok &= len(cpos) == min(r.plans[s].commit, n_q)
            else:
                commit_ok &= topn_commit_admissible(ref, [qidx[int(p)] for p in cpos],
                                                    r.plans[s].commit, r.tol)
            # device grid tokens are the device argmax of the committed rows
            commit_ok &= all(int(ctok[i]) == int(tks[qidx[int(p)]]) for i, p in enumerate(cpos))
            # device grid untouched elsewhere
            untouched = np.ones(Lg, bool)
            untouched[newly] = False
            commit_ok &= bool(np.array_equal(grid_before[s][untouched], grid_after[s][untouched]))
            st.commit(cpos, ctok)   # teacher forcing: adopt the device's choice
            history[s].append(oracle.StepRecord(k, None, np.asarray(qp, dtype=np.int64), None,
                                                cpos.astype(np.int64), ctok.astype(np.int64)))
            ctx_exp[s] += prev_commit[s]
            prev_commit[s] = len(cpos)
            rows_exact &= r.model.smdm_context_length(s) == ctx_exp[s]
            if with_logits:
                rows_exact &= len(st.c_types) == ctx_exp[s]
            off += n_q
        checks.append(StepCheck(k, err, rows_exact, tok_ok, commit_ok))
    for s in range(B):
        assert np.array_equal(grids[s].cpu().numpy(), states[s].grid)
    for s in late_seqs:
        steps = sorted(k for (q, k) in kept if q == s)
        if not steps:
            continue
        ref = late_reference(r, s, history[s], steps)
        for k in steps:
            g, tks = kept[(s, k)]
            c = checks[k - 1]
            c.err = max(c.err, logit_err(g, ref[k]))
            c.tok_ok = c.tok_ok and bool(token_admissible(tks, ref[k], r.tol).all())
            if r.plans[s].kind != "order":
                c.commit_ok = c.commit_ok and topn_commit_admissible(
                    ref[k], [int(np.nonzero(history[s][k - 1].query_pos == p)[0][0])
                             for p in history[s][k - 1].committed_pos],
                    r.plans[s].commit, r.tol)
    return checks, grids, states


def late_reference(r: Runner, s: int, history, steps) -> dict:
    """Oracle logits of the given steps of sequence s, from one training-form forward over the
    teacher-forced trajectory: block 0, the tokens committed at every step before the last one
    asked for (clean, labelled by their step) and each asked step's decode set and tail rows
    (labelled by the step).  Returns {k: logits [n_q][V]}."""
    kmax = max(steps)
    t = r.tasks[s] if r.tasks else None
    ids, pos, types, labels, qrows = oracle.trajectory(
        r.prompts[s], r.wl.model, r.wl.gen_len, history[:kmax], steps=steps,
        preset_pos=None if t is None else t.preset_pos,
        preset_tok=None if t is None else t.preset_tok)
    # the tokens committed AT step kmax are not visible to any asked step: leave them out
    keep = ~((types == oracle.CLEAN) & (labels == kmax))
    idx = np.cumsum(keep) - 1
    rows = np.concatenate([idx[qrows[k]] for k in steps])
    lg = oracle.forward_stepcausal(r.om, ids[keep], pos[keep], types[keep], labels[keep], rows)
    out, off = {}, 0
    for k in steps:
        n = len(qrows[k])
        out[k] = lg[off:off + n]
        off += n
    return out
