#!/usr/bin/env python
"""Benchmark: decoded tokens/s of full sparse masked-diffusion sampling runs on B200.

One bench "step" = one full sampling run of the workload: prefill of the prompt plus every
sampling step of the plan (pack -> transformer stack under the step-causal mask -> sparse LM head
-> unmask), i.e. every stage of the hot path once per sampling step.  The timed region replays
the run as one CUDA graph with all inputs resident in HBM; `e2e` repeats the measurement through
the public API (smdm_generate) with the prompt and plan copied from pinned host memory and the
token grid read back every run.

Default workload: text-to-image 4096 tokens — 4-layer bf16 transformer, d=4096, 32 heads x 128,
SwiGLU ffn 11008, vocab 8192; prompt 256, 64x64 grid, 64 registers, 64 cosine steps, stratified
2-D order; batch 1.  Weights are synthetic N(0, 0.02) drawn on the device from a seed (1.69 GB,
far larger than the 126 MB L2, so every run streams them from HBM; no L2 flush is needed).

N > 1 GPUs (torchrun): independent replicas, one sequence set per rank, no collective on the
data path; value = all ranks' decoded tokens / the slowest rank's time.

`--impl reference` times the fp64 CPU oracle, single-threaded, on a bounded sample of the same
workload (the prefill and sampling steps 1, K/2 and K; the full run extrapolated by each step's
algorithmic FLOPs) and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decoded tokens/s per full sparse-MDM sampling run"
UNIT = "tokens/s"
# bf16 models run their GEMMs and attention on fp16 operands (fp16 copies of the weights made at
# handle creation, fp16 activations) with fp32 accumulation and an fp32 residual stream.
COMPUTE_DTYPE = "f16"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10, help="timed full runs")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="D", choices=["A", "B", "C", "D", "D4", "E"])
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--form", default="sampling", choices=["sampling", "training"],
                    help="sampling: full sparse sampling runs (the headline); training: one "
                         "training-form forward over a whole step-labelled trajectory")
    ap.add_argument("--switches", type=int, default=7, choices=range(8),
                    help="Table-6 speed switches as bits (1 cache prompt, 2 cache decoded "
                         "tokens, 4 truncate); 7 = the method (the default run)")
    ap.add_argument("--task", default=None, choices=["inpaint", "outpaint", "infill"],
                    help="bidirectional task: given generation tokens prefilled with the "
                         "prompt, the plan decodes the rest")
    ap.add_argument("--probe", default=None, choices=["late"],
                    help="late: one short eager run for profiling captures, shaped like the "
                         "last sampling step of the 4096-token workload (a prefill of 4151 "
                         "prompt rows, a step decoding 100 tokens, then a step of 100 new-cache "
                         "rows + 101 queries + 64 registers = 265 rows on a 4151-key cache)")
    ap.add_argument("--n-reg", type=int, default=None,
                    help="register rows per step (the method's 64 by default; 0 = the "
                         "length-token variant, one [LEN] row); for the register-count "
                         "sensitivity study")
    return ap.parse_args()


# ----------------------------------------------------------------------------------------------
# workload description and algorithmic roofline (what the method must move / compute)
# ----------------------------------------------------------------------------------------------

def describe(wl: synth.Workload) -> dict:
    m = wl.model
    return {"workload": {"A": "tiny-fp32", "B": "text-semiAR", "C": "T2I-1024", "D": "T2I-4096",
                         "D4": "T2I-4096-batch4", "E": "image-editing"}.get(wl.name, wl.name),
            "layers": m.n_layers, "d_model": m.d_model, "heads": f"{m.n_heads}x{m.d_head}",
            "d_ffn": m.d_ffn, "vocab": m.vocab,
            "registers": "[LEN]" if m.len_token else m.n_reg, "prompt": wl.prompt_len,
            "gen_len": wl.gen_len, "sampling_steps": wl.n_steps, "batch": wl.batch,
            "plan": wl.plan}


def step_shapes(wl: synth.Workload, plan: synth.Plan):
    """Per sampling step: (rows R, decode rows q, cache length ctx before the step, n_new)."""
    P, Lg, m = wl.prompt_len, wl.gen_len, wl.model
    out = []
    ctx, n_new = P, 0
    for k in range(1, wl.n_steps + 1):
        if plan.kind == "order":
            q = int(plan.n_per_step[k - 1])
            c = q
        else:
            j = (k - 1) % plan.steps_per_block
            q = plan.block - j * plan.commit
            c = plan.commit
        R = n_new + q + m.n_tail
        out.append((R, q, ctx, n_new))
        ctx += n_new
        n_new = c
    return out


def layer_params(m: synth.ModelShape) -> int:
    d, f = m.d_model, m.d_ffn
    return 4 * d * d + 3 * d * f


def forward_cost(m: synth.ModelShape, R: int, q: int, kv_sum: int, kv_keys: int, es: int = 2):
    """Algorithmic (bytes, flops) of one forward over R rows with q logit rows.
    kv_sum = sum over rows of visible keys; kv_keys = distinct keys read per layer."""
    d, V, L = m.d_model, m.vocab, m.n_layers
    wbytes = es * (L * layer_params(m) + (V * d if q else 0))
    act = L * R * es * (d + 3 * d + d + d + d + 2 * m.d_ffn + m.d_ffn + d) + L * R * 4 * d * 4
    kv = L * (kv_keys * 2 * d * es + R * 2 * d * es)
    flops = 2 * R * L * layer_params(m) + 2 * q * V * d + L * 4 * d * kv_sum
    return wbytes + act + kv, flops


def run_forwards(wl: synth.Workload, plans):
    """Shapes of the forwards of one full run of the plans' sequences (one plan, or one per
    sequence of a batch): each sequence's prefill, then one batched forward per step.  Yields
    (rows R, decode rows q, visible keys summed over rows, keys read per layer)."""
    if isinstance(plans, synth.Plan):
        plans = [plans]
    P = wl.prompt_len
    if P:
        for _ in plans:
            yield P, 0, P * P, P
    shapes = [step_shapes(wl, p) for p in plans]
    for k in range(min(len(sh) for sh in shapes)):
        R = q = kv_sum = keys = 0
        for sh in shapes:
            Rb, qb, ctx, n_new = sh[k]
            R += Rb
            q += qb
            kv_sum += n_new * (ctx + n_new) + (Rb - n_new) * (ctx + Rb)
            keys += ctx + Rb
        yield R, q, kv_sum, keys


def run_cost(wl: synth.Workload, plans):
    """List of (bytes, flops) per forward of one full run (prefills first)."""
    return [forward_cost(wl.model, R, q, kv_sum, keys)
            for (R, q, kv_sum, keys) in run_forwards(wl, plans)]


# DRAM bytes (read + write) over algorithmic bytes of gemm_tc_kernel, from one ncu capture of the
# four weight GEMMs (QKV, O, gate/up, down) of one layer at the last sampling step of the
# 4096-token workload (265 rows): 445.96 MB measured against 446.81 MB algorithmic.  The
# capture's command and figures are kept with the profiles.  Re-measure whenever the GEMM kernel
# changes.
GEMM_TRAFFIC_RATIO = 445.96 / 446.81


def gemm_bytes_per_run(wl: synth.Workload, plans, es=2):
    """Algorithmic bytes of the GEMM launches of one full run: weights once per launch plus
    activation operand reads and output writes."""
    m = wl.model
    d, f, V, L = m.d_model, m.d_ffn, m.vocab, m.n_layers
    tot = 0
    for R, q, _, _ in run_forwards(wl, plans):
        per_layer = (es * (3 * d * d + R * d + R * 3 * d)            # qkv: W, X, q/k/v out
                     + es * (d * d + R * d) + 4 * 2 * R * d          # o-proj: W, X, x rmw
                     + es * (2 * f * d + R * d + R * f)              # gate/up: W, X, act out
                     + es * (d * f + R * f) + 4 * 2 * R * d)         # down: W, X, x rmw
        tot += L * per_layer
        if q:
            tot += es * (V * d + q * d) + 4 * 3 * q * ((V + 127) // 128)
    return tot


def class_roofline_ms(wl: synth.Workload, plans, hbm_gbs: float, tflops: float,
                      es=2) -> dict:
    """Roofline time per run of each kernel class, max(bytes / HBM, flops / tensor peak) summed
    over the run's forwards: the weight GEMMs (weights, activation reads, outputs; residual
    read-modify-write in fp32), attention (K/V read once per layer and written for the step's
    rows; 4 d flops per visible key) and RMSNorm (fp32 read, activation write)."""
    m = wl.model
    d, f, V, L = m.d_model, m.d_ffn, m.vocab, m.n_layers
    t = lambda byt, fl: max(byt / (hbm_gbs * 1e9), fl / (tflops * 1e12)) * 1e3
    out = dict.fromkeys(["gemm_qkv", "gemm_o", "gemm_gateup", "gemm_down", "gemm_lmhead",
                         "attn", "norm"], 0.0)
    for R, q, kv_sum, keys in run_forwards(wl, plans):
        out["gemm_qkv"] += L * t(es * (3 * d * d + R * d + R * 3 * d), 2 * R * d * 3 * d)
        out["gemm_o"] += L * t(es * (d * d + R * d) + 4 * 2 * R * d, 2 * R * d * d)
        out["gemm_gateup"] += L * t(es * (2 * f * d + R * d + R * f), 2 * R * d * 2 * f)
        out["gemm_down"] += L * t(es * (d * f + R * f) + 4 * 2 * R * d, 2 * R * f * d)
        if q:
            out["gemm_lmhead"] += t(es * (V * d + q * d) + 4 * 3 * q * ((V + 127) // 128),
                                    2 * q * V * d)
        out["attn"] += L * t(keys * 2 * d * es + R * 2 * d * es, 4 * d * kv_sum)
        out["norm"] += t((2 * L * R + q) * (4 * d + es * d), 0)
    return {k: round(v, 4) for k, v in out.items()}


# ----------------------------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"smdm_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(loaded)}


# ----------------------------------------------------------------------------------------------
# CPU oracle (reported baseline and the reference arm)
# ----------------------------------------------------------------------------------------------

class OracleSample:
    """The fp64 oracle on the host cores, timed on a bounded sample of the workload.

    A full fp64 run of the 4096-token workload is about 20 TFLOP, hours on one core, so the
    sample is: the prefill, and the sampling steps 1, K/2 and K (K = 64: steps 1, 32 and 64).
    A step k after the first runs on a state with that step's shape: a KV cache of the step's
    length (the prefill's entries repeated, all visible, as every cached entry is to every row of
    a real step), the tokens decoded at step k-1 as its new-cache rows and its own decode set.
    The full run is extrapolated, not measured: prefill + sum over all K steps of each step's
    algorithmic FLOPs (`forward_cost`) times the sampled steps' seconds per FLOP.  Weights and
    states are built outside the timing.  `threads` pins the BLAS thread pool (1 = the
    single-threaded oracle; numpy's elementwise work is single-threaded either way)."""

    def __init__(self, wl: synth.Workload):
        import oracle
        self.o = oracle
        self.wl = wl
        self.om = oracle.Model(synth.make_weights(wl.model, wl.seed))
        self.prompt = synth.make_prompt(wl)
        self.plan = synth.make_plan(wl)
        K = self.plan.n_steps
        self.steps = sorted({1, max(1, K // 2), K})
        self.components = ["prefill"] + [f"step {k}" for k in self.steps]
        fw = list(run_forwards(wl, self.plan))
        costs = [forward_cost(wl.model, *f)[1] for f in fw]
        self.prefill_flops = costs[0] if wl.prompt_len else 0.0
        self.step_flops = costs[1:] if wl.prompt_len else costs
        self._base = None
        self._states = {}

    def _decode_sets(self, kmax):
        """Positions decoded at steps 1..kmax (semi-AR: the first `commit` still-masked
        positions of the step's block stand in for the most confident ones; only the counts
        matter for the cost)."""
        o, plan, wl = self.o, self.plan, self.wl
        sim = type("S", (), {})()
        sim.P, sim.grid = wl.prompt_len, np.full(wl.gen_len, -1, dtype=np.int64)
        out = []
        for j in range(1, kmax + 1):
            qp = o.query_set(plan, sim, j)
            c = qp if plan.kind == "order" else qp[:plan.commit]
            sim.grid[c - wl.prompt_len - 1] = 0
            out.append((qp, c))
        return out

    def _state_before(self, k):
        import copy
        o, wl = self.o, self.wl
        if self._base is None:
            self._base = o.Incremental(self.om, self.prompt, wl.gen_len)
        base = self._base
        sets = self._decode_sets(k)
        P = wl.prompt_len
        ctx = len(base.c_types) + sum(len(c) for _, c in sets[:max(0, k - 2)])
        st = copy.copy(base)
        reps = np.arange(ctx) % max(1, len(base.c_types))
        st.k_cache = [kc[reps] for kc in base.k_cache]
        st.v_cache = [vc[reps] for vc in base.v_cache]
        st.c_types = np.zeros(ctx, dtype=np.int64)
        st.c_labels = np.zeros(ctx, dtype=np.int64)
        g = np.random.Generator(np.random.PCG64([wl.seed, 9100 + k]))
        st.grid = np.full(wl.gen_len, -1, dtype=np.int64)
        for _, c in sets[:k - 1]:
            st.grid[c - P - 1] = g.integers(0, wl.model.vocab, len(c))
        st.new_pos = sets[k - 2][1] if k >= 2 else np.zeros(0, dtype=np.int64)
        st.step_k = k - 1
        return st, sets[k - 1][0]

    def time_component(self, c: str, threads: int) -> float:
        """Seconds of one sample component ("prefill" or "step k") on `threads` BLAS threads."""
        from threadpoolctl import threadpool_limits
        o, wl = self.o, self.wl
        st = qp = None
        if c != "prefill":
            import copy
            k = int(c.split()[1])
            if k not in self._states:
                self._states[k] = self._state_before(k)
            # a fresh state per call (the step appends to the per-layer cache lists), made
            # outside the timing
            st0, qp = self._states[k]
            st = copy.copy(st0)
            st.k_cache, st.v_cache = list(st0.k_cache), list(st0.v_cache)
            st.grid = st0.grid.copy()
        with threadpool_limits(limits=threads, user_api="blas"):
            t0 = time.perf_counter()
            if c == "prefill":
                o.Incremental(self.om, self.prompt, wl.gen_len)
            else:
                lg = st.step_logits(qp)
                o.unmask(lg, o.POLICY_ALL if self.plan.kind == "order" else o.POLICY_TOPN,
                         self.plan.commit)
            return time.perf_counter() - t0

    def extrapolate(self, secs: dict) -> float:
        """Full-run seconds from the component times: prefill + sum_k FLOPs_k x (sampled
        seconds / sampled FLOPs)."""
        t_steps = sum(secs[f"step {k}"] for k in self.steps)
        f_steps = sum(self.step_flops[k - 1] for k in self.steps)
        return secs["prefill"] + t_steps / f_steps * sum(self.step_flops)

    def describe(self) -> str:
        wl = self.wl
        return (f"fp64 numpy oracle: prefill ({wl.prompt_len} rows) and sampling steps "
                f"{', '.join(map(str, self.steps))} of {self.plan.n_steps} timed (steps after the "
                f"first on a state with that step's cache length, new-cache rows and decode set); "
                f"the full run of {wl.gen_len} decoded tokens is extrapolated by the algorithmic "
                f"FLOPs of every step")

    def run(self, threads: int) -> dict:
        """Time every component once on `threads` BLAS threads; returns the full-run figures."""
        secs = {c: self.time_component(c, threads) for c in self.components}
        full = self.extrapolate(secs)
        return {"value": self.wl.gen_len * self.wl.batch / full, "full_run_s": full,
                "sampled_s": {c: round(v, 3) for c, v in secs.items()},
                "sample_s": sum(secs.values())}


def _cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, wl):
    """The reference arm: the fp64 oracle, single-threaded, as it stands.  Each bench step times
    one component of the oracle sample (prefill, step 1, step K/2, step K, in rotation); the
    value is the extrapolated full-run rate from the mean time of each component over the timed
    steps (a component the timed steps did not reach is timed once more after them)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sample = OracleSample(wl)
    comps = sample.components
    times = {c: [] for c in comps}
    for i in range(args.warmup + args.steps):
        c = comps[i % len(comps)]
        dt = sample.time_component(c, 1)
        if i >= args.warmup:
            times[c].append(dt)
    extra = [c for c in comps if not times[c]]
    for c in extra:
        times[c].append(sample.time_component(c, 1))
    secs = {c: sum(v) / len(v) for c, v in times.items()}
    full = sample.extrapolate(secs)
    value = wl.gen_len * wl.batch / full
    desc = sample.describe() + (f"; one component per bench step, {', '.join(extra)} timed once "
                                f"after the timed steps" if extra else
                                "; one component per bench step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": full * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": describe(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": desc, "extrapolated": True,
                             "sampled_s": {c: round(v, 3) for c, v in secs.items()},
                             "cpu": _cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------------------
# native arm
# ----------------------------------------------------------------------------------------------

def device_weights(wl: synth.Workload, seed: int, device):
    import torch
    m = wl.model
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = torch.bfloat16 if m.dtype == synth.BF16 else torch.float32

    def rnd(*shape):
        return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * 0.02).to(dt)

    def ones(n):
        return torch.ones(n, device=device, dtype=dt)

    d, f, V = m.d_model, m.d_ffn, m.vocab
    w = {"emb": rnd(m.emb_rows, d), "final_norm": ones(d), "lm_head": rnd(V, d)}
    for k in ("attn_norm", "w_qkv", "w_o", "mlp_norm", "w_gate", "w_up", "w_down"):
        w[k] = []
    for _ in range(m.n_layers):
        w["attn_norm"].append(ones(d))
        w["w_qkv"].append(rnd(3 * d, d))
        w["w_o"].append(rnd(d, d))
        w["mlp_norm"].append(ones(d))
        w["w_gate"].append(rnd(f, d))
        w["w_up"].append(rnd(f, d))
        w["w_down"].append(rnd(d, f))
    return w


def trajectory_rows(wl: synth.Workload, plan: synth.Plan, prompt: np.ndarray, seed: int):
    """Rows of a whole sampling trajectory in the step-labelled training form (order plans),
    laid out as the oracle's trajectory: the prompt (label 0); the clean copies of the tokens
    decoded at every step k (label k), step by step; then, step by step, the mask copies of the
    same positions (the decode set C_k) and the step's tail rows (registers or [LEN]), all
    labelled k.  Token values are random (structure and sizes are what the forward's cost
    depends on).  Returns ids, pos, types, labels and the logit rows (the mask copies)."""
    m = wl.model
    P, Lg = wl.prompt_len, wl.gen_len
    L = P + Lg
    g = np.random.Generator(np.random.PCG64([wl.seed, 7000 + seed]))
    ids, pos, types, labels, logit_rows = list(prompt), list(range(1, P + 1)), [0] * P, [0] * P, []
    steps = [plan.query_positions(k) for k in range(1, plan.n_steps + 1)]
    for k, q in enumerate(steps, start=1):      # clean copies
        n = len(q)
        ids += list(g.integers(0, m.vocab, n))
        pos += list(q)
        types += [1] * n
        labels += [k] * n
    for k, q in enumerate(steps, start=1):      # mask copies and tail rows
        n = len(q)
        logit_rows += list(range(len(ids), len(ids) + n))
        ids += [m.vocab] * n
        pos += list(q)
        types += [2] * n
        labels += [k] * n
        if m.len_token:                       # the one [LEN] row
            ids += [m.vocab + 1]
            pos += [L + 1]
        else:                                 # the registers
            ids += [m.vocab + 2 + j for j in range(m.n_reg)]
            pos += [L + 1 + j for j in range(m.n_reg)]
        types += [3] * m.n_tail
        labels += [k] * m.n_tail
    as32 = lambda a: np.asarray(a, dtype=np.int32)
    return as32(ids), as32(pos), as32(types), as32(labels), as32(logit_rows)


def run_training_form(args, wl):
    """Times one training-form forward (smdm_forward_stepcausal) over the whole trajectory of
    the workload's plan: every row of every step in one forward under the label predicate."""
    import torch
    import masked_discrete_diffusion_sparse_b200 as smdm
    if wl.plan == "semiar" or wl.batch != 1:
        raise SystemExit("--form training supports single-sequence order plans")
    m = wl.model
    dev = torch.device("cuda", 0)
    plan = synth.make_plan(wl, 0)
    prompt = synth.make_prompt(wl, 0)
    ids, pos, types, labels, lrows = trajectory_rows(wl, plan, prompt, 0)
    n = len(ids)
    cfg = smdm.make_config(m.n_layers, m.d_model, m.n_heads, m.d_head, m.d_ffn, m.vocab,
                           n_reg=smdm.SMDM_REG_LEN if m.len_token else m.n_reg,
                           dtype=smdm.SMDM_BF16 if m.dtype == synth.BF16 else smdm.SMDM_F32,
                           rope_theta=m.rope_theta, rms_eps=m.rms_eps, max_batch=1,
                           max_len=wl.prompt_len + wl.gen_len, max_step_rows=1, max_rows=n)
    model = smdm.Model(cfg, device_weights(wl, wl.seed + 7919, dev))
    t = lambda a: torch.as_tensor(a, device=dev)
    d_ids, d_pos, d_types, d_labels, d_rows = t(ids), t(pos), t(types), t(labels), t(lrows)
    logits = torch.empty((len(lrows), m.vocab), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def fwd():
        model.smdm_forward_stepcausal(d_ids, d_pos, d_types, d_labels, d_rows, logits,
                                      stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            fwd()
        torch.cuda.synchronize()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            fwd()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / args.steps
    assert model.smdm_device_status(stream) == 0
    print(json.dumps({"metric": "training-form forward rows/s", "value": n / (ms / 1e3),
                      "unit": "rows/s", "n_gpus": 1, "steps": args.steps,
                      "warmup": max(3, args.warmup), "ms_per_step": ms,
                      "higher_is_better": True, "form": "training", "rows": n,
                      "logit_rows": int(len(lrows)), "dtype": COMPUTE_DTYPE if m.dtype == synth.BF16
                      else "f32", "data": "synthetic", "config": describe(wl)}), flush=True)
    model.close()
    return 0


def run_probe(args, wl):
    """--probe late: the launches of the 4096-token workload's late steps without the 60 steps
    before them.  Launch order: prefill (per layer: QKV, attention, O, gate/up, down), step 1
    (the same plus the LM head and unmask), step 2 (the captured shape)."""
    import torch
    import masked_discrete_diffusion_sparse_b200 as smdm
    m = wl.model
    dev = torch.device("cuda", 0)
    P, Lg, n1, n2 = 4151, wl.gen_len, 100, 101
    g = np.random.Generator(np.random.PCG64([wl.seed, 8100]))
    prompt = g.integers(0, m.vocab, P).astype(np.int32)
    order = (g.permutation(Lg)[:n1 + n2] + P + 1).astype(np.int32)
    R2 = n1 + n2 + m.n_tail
    cfg = smdm.make_config(m.n_layers, m.d_model, m.n_heads, m.d_head, m.d_ffn, m.vocab,
                           n_reg=m.n_reg, dtype=smdm.SMDM_BF16, rope_theta=m.rope_theta,
                           rms_eps=m.rms_eps, max_batch=1, max_len=P + Lg, max_step_rows=R2,
                           max_rows=P)
    model = smdm.Model(cfg, device_weights(wl, wl.seed + 7919, dev))
    stream = torch.cuda.Stream(device=dev)
    grid = torch.empty(Lg, dtype=torch.int32, device=dev)
    d_order = torch.as_tensor(order, device=dev)
    with torch.cuda.stream(stream):
        model.smdm_prefill(0, torch.as_tensor(prompt, device=dev), Lg, grid, stream=stream)
        model.smdm_step([dict(seq=0, query_pos=d_order[:n1], n_query=n1)], stream=stream)
        model.smdm_step([dict(seq=0, query_pos=d_order[n1:], n_query=n2)], stream=stream)
    torch.cuda.synchronize()
    assert model.smdm_device_status(stream) == 0
    print(json.dumps({"probe": "late", "prefill_rows": P, "step2_rows": R2,
                      "step2_cache_keys": model.smdm_context_length(0)}), flush=True)
    model.close()
    return 0


def run_switched(args, wl):
    """--switches S (bits 1 cache prompt, 2 cache decoded tokens, 4 truncate; 7 = the method):
    one sequence's sampling run through smdm_step_switched, replayed as a CUDA graph (prefill
    + every step).  One line per setting gives the speed side of the Table-6 ablation."""
    import torch
    import masked_discrete_diffusion_sparse_b200 as smdm
    if wl.plan == "semiar" or wl.batch != 1:
        raise SystemExit("--switches supports single-sequence order plans")
    m = wl.model
    P, Lg = wl.prompt_len, wl.gen_len
    dev = torch.device("cuda", 0)
    plan = synth.make_plan(wl, 0)
    prompt = synth.make_prompt(wl, 0)
    rows = P + Lg + m.n_tail           # the largest step: nothing cached, nothing truncated
    cfg = smdm.make_config(m.n_layers, m.d_model, m.n_heads, m.d_head, m.d_ffn, m.vocab,
                           n_reg=smdm.SMDM_REG_LEN if m.len_token else m.n_reg,
                           dtype=smdm.SMDM_BF16 if m.dtype == synth.BF16 else smdm.SMDM_F32,
                           rope_theta=m.rope_theta, rms_eps=m.rms_eps, max_batch=1,
                           max_len=P + Lg, max_step_rows=rows, max_rows=rows)
    model = smdm.Model(cfg, device_weights(wl, wl.seed + 7919, dev))
    stream = torch.cuda.Stream(device=dev)
    d_prompt = torch.as_tensor(prompt.astype(np.int32), device=dev)
    d_order = torch.as_tensor(plan.order.astype(np.int32), device=dev)
    offs = [int(o) for o in plan.offsets]
    grid = torch.empty(Lg, dtype=torch.int32, device=dev)

    def run():
        model.smdm_prefill(0, d_prompt, Lg, grid, stream=stream)
        for k in range(1, plan.n_steps + 1):
            qp = d_order[offs[k - 1]:offs[k]]
            model.smdm_step_switched(dict(seq=0, query_pos=qp, n_query=int(qp.numel())),
                                     args.switches, stream=stream)

    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    assert model.smdm_device_status(stream) == 0
    assert bool((grid >= 0).all())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / args.steps
    assert model.smdm_device_status(stream) == 0
    names = {1: "cache_prompt", 2: "cache_res", 4: "truncate"}
    cfg_line = describe(wl)
    cfg_line["switches"] = {v: bool(args.switches & b) for b, v in names.items()}
    cfg_line["timed"] = "CUDA-graph replay of prefill + all sampling steps (smdm_step_switched)"
    print(json.dumps({"metric": METRIC, "value": Lg / (ms / 1e3), "unit": UNIT, "n_gpus": 1,
                      "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                      "dtype": COMPUTE_DTYPE if m.dtype == synth.BF16 else "f32",
                      "data": "synthetic", "config": cfg_line}), flush=True)
    del graph
    model.close()
    return 0


def run_task(args, wl):
    """--task inpaint|outpaint|infill: a bidirectional generation task (given generation tokens
    prefilled with the prompt as block-0 clean rows, smdm_prefill_given) whose plan decodes
    only the other positions, step by step through smdm_step, replayed as a CUDA graph."""
    import torch
    import masked_discrete_diffusion_sparse_b200 as smdm
    if wl.plan == "semiar" or wl.batch != 1:
        raise SystemExit("--task supports single-sequence order plans")
    m = wl.model
    P, Lg = wl.prompt_len, wl.gen_len
    dev = torch.device("cuda", 0)
    task = synth.make_bidir_task(wl, args.task)
    plan = task.plan
    prompt = synth.make_prompt(wl, 0)
    n = [int(v) for v in plan.n_per_step]
    msr = max((n[i - 1] if i else 0) + n[i] for i in range(len(n))) + m.n_tail
    n0 = P + len(task.preset_pos)
    cfg = smdm.make_config(m.n_layers, m.d_model, m.n_heads, m.d_head, m.d_ffn, m.vocab,
                           n_reg=smdm.SMDM_REG_LEN if m.len_token else m.n_reg,
                           dtype=smdm.SMDM_BF16 if m.dtype == synth.BF16 else smdm.SMDM_F32,
                           rope_theta=m.rope_theta, rms_eps=m.rms_eps, max_batch=1,
                           max_len=P + Lg, max_step_rows=msr, max_rows=max(msr, n0))
    model = smdm.Model(cfg, device_weights(wl, wl.seed + 7919, dev))
    stream = torch.cuda.Stream(device=dev)
    t32 = lambda a: torch.as_tensor(np.asarray(a, dtype=np.int32), device=dev)
    d_prompt, d_gpos, d_gtok = t32(prompt), t32(task.preset_pos), t32(task.preset_tok)
    d_order = t32(plan.order)
    offs = [int(o) for o in plan.offsets]
    grid = torch.empty(Lg, dtype=torch.int32, device=dev)

    def run():
        model.smdm_prefill_given(0, d_prompt, Lg, d_gpos, d_gtok, grid, stream=stream)
        for k in range(1, plan.n_steps + 1):
            qp = d_order[offs[k - 1]:offs[k]]
            model.smdm_step([dict(seq=0, query_pos=qp, n_query=int(qp.numel()),
                                  policy=smdm.SMDM_POLICY_ALL, n_commit=int(qp.numel()))],
                            stream=stream)

    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    assert model.smdm_device_status(stream) == 0
    assert bool((grid >= 0).all())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / args.steps
    assert model.smdm_device_status(stream) == 0
    decoded = len(plan.order)
    cfg_line = describe(wl)
    cfg_line.update({"task": args.task, "given_tokens": int(len(task.preset_pos)),
                     "decoded_tokens": decoded, "sampling_steps": plan.n_steps,
                     "timed": "CUDA-graph replay of the block-0 prefill (prompt + given "
                              "tokens) + all sampling steps"})
    print(json.dumps({"metric": METRIC, "value": decoded / (ms / 1e3), "unit": UNIT,
                      "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup),
                      "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                      "vs_baseline": None, "dtype": COMPUTE_DTYPE if m.dtype == synth.BF16 else "f32",
                      "data": "synthetic", "config": cfg_line}), flush=True)
    del graph
    model.close()
    return 0


def capacities(wl, plans):
    m = wl.model
    msr = 1
    for plan in plans:
        for (R, q, ctx, n_new) in step_shapes(wl, plan):
            msr = max(msr, R)
    L = wl.prompt_len + wl.gen_len
    return msr, max(wl.batch * msr, wl.prompt_len, L)


def main():
    args = parse()
    wl = synth.WORKLOADS[args.workload]
    if args.n_reg is not None and args.n_reg != wl.model.n_reg:
        if args.n_reg < 0:
            raise SystemExit("--n-reg must be >= 0")
        import dataclasses
        # 0: the length-token variant (one [LEN] row instead of registers)
        wl = dataclasses.replace(wl, name=f"{wl.name}-reg{args.n_reg}" if args.n_reg else
                                 f"{wl.name}-len",
                                 model=dataclasses.replace(wl.model, n_reg=args.n_reg,
                                                           len_token=args.n_reg == 0))
    if args.impl == "reference":
        return run_reference(args, wl)

    if args.probe == "late":
        return run_probe(args, wl)
    if args.form == "training":
        return run_training_form(args, wl)
    if args.switches != 7:
        return run_switched(args, wl)
    if args.task is not None:
        return run_task(args, wl)

    import torch
    import torch.distributed as dist
    import masked_discrete_diffusion_sparse_b200 as smdm
    from masked_discrete_diffusion_sparse_b200.replicas import (aggregate_throughput,
                                                                replica_sequence_ids,
                                                                slowest_time_ms)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    m = wl.model
    B = wl.batch
    seq_ids = replica_sequence_ids(rank, B)   # disjoint sequence sets across ranks
    plans = [synth.make_plan(wl, i) for i in seq_ids]
    prompts_np = np.stack([synth.make_prompt(wl, i) for i in seq_ids])
    msr, max_rows = capacities(wl, plans)
    cfg = smdm.make_config(m.n_layers, m.d_model, m.n_heads, m.d_head, m.d_ffn, m.vocab,
                           n_reg=smdm.SMDM_REG_LEN if m.len_token else m.n_reg,
                           dtype=smdm.SMDM_BF16 if m.dtype == synth.BF16 else smdm.SMDM_F32,
                           rope_theta=m.rope_theta, rms_eps=m.rms_eps, max_batch=B,
                           max_len=wl.prompt_len + wl.gen_len, max_step_rows=msr,
                           max_rows=max_rows)
    weights = device_weights(wl, wl.seed + 7919, dev)   # the same model on every replica
    model = smdm.Model(cfg, weights)
    stream = torch.cuda.Stream(device=dev)

    P, Lg = wl.prompt_len, wl.gen_len
    d_prompts = torch.as_tensor(prompts_np.astype(np.int32), device=dev)
    d_orders = [torch.as_tensor(p.order, device=dev) if p.order is not None else None for p in plans]
    d_grids = torch.empty((B, Lg), dtype=torch.int32, device=dev)

    def plan_dicts():
        out = []
        for i, p in enumerate(plans):
            if p.kind == "order":
                out.append(dict(kind=smdm.SMDM_PLAN_ORDER, n_steps=p.n_steps,
                                n_per_step=list(p.n_per_step), order=d_orders[i]))
            else:
                out.append(dict(kind=smdm.SMDM_PLAN_SEMIAR, n_steps=p.n_steps, block=p.block,
                                steps_per_block=p.steps_per_block, commit=p.commit))
        return out

    pd = plan_dicts()

    def generate(mode=smdm.SMDM_MODE_SPARSE, prompts=d_prompts, plans_=pd, grids=d_grids):
        model.smdm_generate(prompts, Lg, plans_, grids, mode=mode, stream=stream)

    # eager sanity run + per-kernel-class profile (events on the launching stream)
    with torch.cuda.stream(stream):
        generate()
        stream.synchronize()
        assert model.smdm_device_status(stream) == 0
        g = d_grids.cpu().numpy()
        assert (g >= 0).all() and (g < m.vocab).all(), "incomplete generation"
        model.smdm_profile_begin(timed=True)
        generate()
        prof = model.smdm_profile_end(stream)
    launches_per_run = prof["launches"]

    # capture one full run as a CUDA graph
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
        generate()
    torch.cuda.synchronize()

    def timed(fn, n):
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(n):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return ev0.elapsed_time(ev1) / n

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        ms = timed(graph.replay, args.steps)
    clocks = sampler.stop()
    ms_max = slowest_time_ms(ms, world, dist, dev)
    tokens_per_run = Lg * B
    value = aggregate_throughput(tokens_per_run, world, ms_max)
    assert model.smdm_device_status(stream) == 0

    # e2e: public API, pinned host inputs -> device, grid -> host, every run
    e2e = None
    if not args.no_e2e:
        h_prompts = torch.from_numpy(prompts_np.astype(np.int32)).pin_memory()
        h_orders = [torch.from_numpy(p.order.astype(np.int32)).pin_memory() if p.order is not None
                    else None for p in plans]
        h_grid = torch.empty((B, Lg), dtype=torch.int32).pin_memory()
        e_prompts = torch.empty_like(d_prompts)
        e_orders = [torch.empty_like(o) if o is not None else None for o in d_orders]
        e_grids = torch.empty_like(d_grids)
        e_plans = plan_dicts()
        for i, p in enumerate(e_plans):
            if "order" in p:
                p["order"] = e_orders[i]
        h2d = h_prompts.numel() * 4 + sum(o.numel() * 4 for o in h_orders if o is not None)
        d2h = h_grid.numel() * 4

        def e2e_run():
            e_prompts.copy_(h_prompts, non_blocking=True)
            for i, o in enumerate(h_orders):
                if o is not None:
                    e_orders[i].copy_(o, non_blocking=True)
            model.smdm_generate(e_prompts, Lg, e_plans, e_grids, stream=stream)
            h_grid.copy_(e_grids, non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(max(1, args.warmup)):
                e2e_run()
            e_ms = timed(e2e_run, max(3, args.steps // 2))
        e_max = slowest_time_ms(e_ms, world, dist, dev)
        e2e = {"value": aggregate_throughput(tokens_per_run, world, e_max), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e_max, "path": "smdm_generate (eager launches)"}

    # dense comparator: the same library's dense full-sequence MDM step, full run
    dense = None
    if not args.no_dense and rank == 0:
        dgrids = torch.empty_like(d_grids)
        with torch.cuda.stream(stream):
            generate(mode=smdm.SMDM_MODE_DENSE, grids=dgrids)   # warm-up
            d_ms = timed(lambda: generate(mode=smdm.SMDM_MODE_DENSE, grids=dgrids), 1)
        dense = {"value": tokens_per_run / (d_ms / 1e3), "unit": UNIT, "ms_per_run": d_ms,
                 "sparse_speedup": d_ms / ms}

    # roofline
    peaks_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(peaks_path):
        pk = json.load(open(peaks_path))
        hbm, tfl, tfl_s, peak_src = pk["hbm_gbs"], pk["bf16_tflops"], \
            pk.get("bf16_tflops_sustained", pk["bf16_tflops"]), "measured"
    else:
        hbm, tfl, tfl_s, peak_src = 6650.0, 1590.0, 1400.0, "fallback"
    gemm_cls = ["gemm_qkv", "gemm_o", "gemm_gateup", "gemm_down", "gemm_lmhead"]
    # Per-class device time of the graph: the same run captured once more with the library's
    # per-launch event pair around every kernel (event nodes in the graph: no host launch gaps,
    # but no programmatic overlap between neighbours either), replayed once.  The dominant
    # kernel's time per run is its share of that profile times the timed graph's run time.
    gprof = None
    try:
        with torch.cuda.stream(stream):
            pgraph = torch.cuda.CUDAGraph()
            model.smdm_profile_begin(timed=True)
            with torch.cuda.graph(pgraph, stream=stream, capture_error_mode="thread_local"):
                generate()
            pgraph.replay()
            gprof = model.smdm_profile_end(stream)
            del pgraph
    except Exception as exc:   # profiling is reported, never fatal
        gprof = {"error": str(exc)}
        try:
            model.smdm_profile_end(stream)
        except Exception:
            pass
    prof_basis = "eager events"
    cls_ms = prof["class_ms"]
    if gprof and "class_ms" in gprof and sum(gprof["class_ms"].values()) > 0:
        cls_ms, prof_basis = gprof["class_ms"], "graph events"
    share = sum(cls_ms[c] for c in gemm_cls) / sum(cls_ms.values())
    gemm_ms = share * ms
    gemm_n = sum(prof["class_launches"][c] for c in gemm_cls)
    gb = gemm_bytes_per_run(wl, plans)
    achieved = gb / (gemm_ms / 1e3) / 1e9 if gemm_ms > 0 else None
    costs = run_cost(wl, plans)
    roof_s = sum(max(b / (hbm * 1e9), f / (tfl_s * 1e12)) for b, f in costs)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": COMPUTE_DTYPE if m.dtype == synth.BF16 else "f32",
        "data": "synthetic (seeded N(0,0.02) weights drawn on device; seeded prompts/orders)",
        "config": {**describe(wl), "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "weights 1.69 GB >> 126 MB L2 stream from HBM every run (no flush)",
                   "timed": "CUDA-graph replay of prefill + all sampling steps"},
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches_per_run * args.steps,
        "roofline": {"bound": "hbm", "kernel": "gemm_tc_kernel (all weight GEMMs)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": (achieved / hbm) if achieved else None,
                     "traffic": (GEMM_TRAFFIC_RATIO * gb / gemm_n) if gemm_n else None,
                     "traffic_unit": "bytes per launch (measured DRAM/algorithmic ratio x "
                                     "algorithmic bytes per launch)",
                     "peak_source": peak_src,
                     "gemm_ms_per_run": gemm_ms, "gemm_launches_per_run": gemm_n,
                     "gemm_algorithmic_gb_per_run": gb / 1e9,
                     "time_basis": f"GEMM share {share:.3f} of the per-class {prof_basis} x "
                                   f"the timed graph's {ms:.3f} ms per run"},
        "step_roofline": {"roofline_ms_per_run": roof_s * 1e3, "measured_ms_per_run": ms,
                          "frac": roof_s * 1e3 / ms,
                          "peaks": {"hbm_gbs": hbm, "bf16_tflops_sustained": tfl_s}},
        "per_class_ms_per_run": {k: round(v, 4) for k, v in cls_ms.items()},
        "per_class_basis": prof_basis,
        **({"per_class_graph_error": gprof["error"]} if gprof and "error" in gprof else {}),
        "per_class_roofline_ms_per_run": class_roofline_ms(wl, plans, hbm, tfl_s),
        "per_step_ms": ms / wl.n_steps,
        "dense": dense,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        try:
            sample = OracleSample(wl)
            one = sample.run(1)
            cores = os.cpu_count() or 1
            allc = sample.run(cores)
            line["cpu_baseline"] = {"value": one["value"], "unit": UNIT, "cores": 1,
                                    "kind": "oracle", "sample": sample.describe(),
                                    "extrapolated": True, "full_run_s": one["full_run_s"],
                                    "sampled_s": one["sampled_s"],
                                    "all_cores": {"value": allc["value"], "cores": cores,
                                                  "full_run_s": allc["full_run_s"],
                                                  "sampled_s": allc["sampled_s"]},
                                    "cpu": _cpu_model()}
        except MemoryError:
            line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
