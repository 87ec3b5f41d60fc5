"""Seeded synthetic inputs for the sparse masked-diffusion sampler.

This module is shared by the fp64 oracle (``oracle/``) and by the CUDA path's
tests and benchmark.  It holds no arithmetic of the method itself: it only
draws random weights, prompts and unmask plans (the decode order and the
per-step decode-set sizes), which both sides receive as inputs.

Workloads are the five synthetic shapes used throughout this repository:

  A  tiny fp32:      2 layers, d=256, 4x64 heads, ffn 688, vocab 1024,
                     prompt 32, 16x16 grid, 8 steps of 32 from a random
                     permutation, commit all.
  B  text semi-AR:   8 layers bf16, d=1024, 16x64, ffn 2816, vocab 32000,
                     prompt 512 Zipf(1.1) tokens, 512 generated in 4
                     left-to-right blocks of 128, 16 steps per block, commit the
                     8 most confident masked positions of the block per step.
  C  T2I 1024:       4 layers bf16, d=4096, 32x128, ffn 11008, vocab 8192,
                     prompt 128, 32x32 grid, 64 cosine steps, stratified order.
  D  T2I 4096:       same model, prompt 256, 64x64 grid, 64 cosine steps.
  E  editing:        same model at 8 layers, prompt 256 text + 4096 reference
                     image tokens, 64x64 grid, 64 cosine steps.

Plus small bf16 shapes ("tiny-bf16-*") with the same structure that the
oracle finishes in seconds.

Special ids (content vocabulary V): [MASK] = V, [LEN] = V + 1,
register j = V + 2 + j.  The embedding table therefore has V + 2 + n_reg rows.
Positions are 1-based: prompt 1..P, generation P+1..P+Lg, registers
L+1..L+n_reg with L = P + Lg.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclass(frozen=True)
class ModelShape:
    n_layers: int
    d_model: int
    n_heads: int
    d_head: int
    d_ffn: int
    vocab: int
    n_reg: int = 64
    dtype: str = BF16
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    len_token: bool = False   # with n_reg == 0: the length-token variant (one [LEN] row per step)

    def __post_init__(self):
        if self.len_token and self.n_reg != 0:
            raise ValueError("the length-token variant has no registers (n_reg == 0)")

    @property
    def emb_rows(self) -> int:
        return self.vocab + 2 + self.n_reg

    @property
    def n_tail(self) -> int:
        """Rows that close each sampling step: the registers, or the one [LEN] row."""
        return 1 if self.len_token else self.n_reg

    @property
    def mask_id(self) -> int:
        return self.vocab

    @property
    def len_id(self) -> int:
        return self.vocab + 1

    def reg_id(self, j: int) -> int:
        return self.vocab + 2 + j


@dataclass(frozen=True)
class Workload:
    name: str
    model: ModelShape
    prompt_len: int
    gen_len: int
    plan: str                 # "perm" | "cosine" | "semiar"
    n_steps: int              # total sampling steps
    grid_side: int = 0        # image grid side for the stratified order (0 = none)
    step_size: int = 0        # "perm": tokens per step
    block: int = 0            # "semiar": block length
    steps_per_block: int = 0  # "semiar"
    commit: int = 0           # "semiar": tokens committed per step (top-n)
    prompt_dist: str = "uniform"  # "uniform" | "zipf"
    zipf_a: float = 1.1
    batch: int = 1
    seed: int = 0


MODEL_A = ModelShape(2, 256, 4, 64, 688, 1024, dtype=F32)
MODEL_B = ModelShape(8, 1024, 16, 64, 2816, 32000)
MODEL_CD = ModelShape(4, 4096, 32, 128, 11008, 8192)
MODEL_E = ModelShape(8, 4096, 32, 128, 11008, 8192)

WORKLOADS = {
    "A": Workload("A", MODEL_A, 32, 256, "perm", 8, grid_side=16, step_size=32, seed=0x5D1A + 0),
    "B": Workload("B", MODEL_B, 512, 512, "semiar", 64, block=128, steps_per_block=16, commit=8,
                  prompt_dist="zipf", seed=0x5D1A + 1),
    "C": Workload("C", MODEL_CD, 128, 1024, "cosine", 64, grid_side=32, seed=0x5D1A + 2),
    "D": Workload("D", MODEL_CD, 256, 4096, "cosine", 64, grid_side=64, seed=0x5D1A + 3),
    "D4": Workload("D4", MODEL_CD, 256, 4096, "cosine", 64, grid_side=64, batch=4, seed=0x5D1A + 3),
    "E": Workload("E", MODEL_E, 4352, 4096, "cosine", 64, grid_side=64, seed=0x5D1A + 4),
    # Small shapes with the structure of the large ones; the oracle runs them in seconds.
    # Vocab sizes leave ragged tails against 128-wide tiles on purpose.
    "tiny-bf16-cos": Workload("tiny-bf16-cos",
                              ModelShape(2, 256, 2, 128, 704, 1000), 40, 256, "cosine", 12,
                              grid_side=16, seed=0x5D1A + 10),
    "tiny-bf16-semiar": Workload("tiny-bf16-semiar",
                                 ModelShape(2, 256, 4, 64, 512, 1500), 70, 96, "semiar", 12,
                                 block=32, steps_per_block=4, commit=8, prompt_dist="zipf",
                                 seed=0x5D1A + 11),
    "tiny-bf16-batch": Workload("tiny-bf16-batch",
                                ModelShape(2, 256, 2, 128, 704, 1000), 40, 256, "cosine", 12,
                                grid_side=16, batch=3, seed=0x5D1A + 12),
    "tiny-f32-cos": Workload("tiny-f32-cos",
                             ModelShape(2, 128, 2, 64, 320, 300, dtype=F32), 20, 64, "cosine", 8,
                             grid_side=8, seed=0x5D1A + 13),
}


# ----------------------------------------------------------------------------------------------
# bf16 helpers (input encoding only)
# ----------------------------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------------------------
# Weights
# ----------------------------------------------------------------------------------------------

@dataclass
class Weights:
    """Model weights as stored on the device.

    Linear weights are [out_features][in_features] (input features contiguous).
    For bf16 models each array is uint16 bit patterns; for fp32 models float32.
    """
    shape: ModelShape
    emb: np.ndarray                  # [emb_rows][d]
    final_norm: np.ndarray           # [d]
    lm_head: np.ndarray              # [V][d]
    attn_norm: List[np.ndarray] = field(default_factory=list)  # [d]
    w_qkv: List[np.ndarray] = field(default_factory=list)      # [3d][d] rows: q | k | v
    w_o: List[np.ndarray] = field(default_factory=list)        # [d][d]
    mlp_norm: List[np.ndarray] = field(default_factory=list)   # [d]
    w_gate: List[np.ndarray] = field(default_factory=list)     # [ffn][d]
    w_up: List[np.ndarray] = field(default_factory=list)       # [ffn][d]
    w_down: List[np.ndarray] = field(default_factory=list)     # [d][ffn]

    def tensors(self):
        """All arrays in a fixed order (for uploads)."""
        out = [("emb", self.emb), ("final_norm", self.final_norm), ("lm_head", self.lm_head)]
        for l in range(self.shape.n_layers):
            out += [(f"attn_norm.{l}", self.attn_norm[l]), (f"w_qkv.{l}", self.w_qkv[l]),
                    (f"w_o.{l}", self.w_o[l]), (f"mlp_norm.{l}", self.mlp_norm[l]),
                    (f"w_gate.{l}", self.w_gate[l]), (f"w_up.{l}", self.w_up[l]),
                    (f"w_down.{l}", self.w_down[l])]
        return out


def _normal(gen: np.random.Generator, shape, std: float, mean: float = 0.0) -> np.ndarray:
    a = gen.standard_normal(size=shape, dtype=np.float32)
    a *= np.float32(std)
    if mean:
        a += np.float32(mean)
    return a


def make_weights(shape: ModelShape, seed: int, gain_std: float = 0.02, std: float = 0.02) -> Weights:
    """Weights N(0, std) (0.02 by default); RMSNorm gains 1 + N(0, gain_std) (gain_std=0 gives
    all-ones gains).

    Each tensor has its own seeded stream so that tensors can be regenerated independently.
    """
    d, f, V = shape.d_model, shape.d_ffn, shape.vocab

    def tensor(idx: int, shp, std: float, mean: float = 0.0) -> np.ndarray:
        g = np.random.Generator(np.random.PCG64([seed, idx]))
        a = _normal(g, shp, std, mean) if std > 0 else np.full(shp, mean, np.float32)
        return f32_to_bf16_bits(a) if shape.dtype == BF16 else a

    w = Weights(shape,
                emb=tensor(0, (shape.emb_rows, d), std),
                final_norm=tensor(1, (d,), gain_std, 1.0),
                lm_head=tensor(2, (V, d), std))
    for l in range(shape.n_layers):
        b = 16 + 8 * l
        w.attn_norm.append(tensor(b + 0, (d,), gain_std, 1.0))
        w.w_qkv.append(tensor(b + 1, (3 * d, d), std))
        w.w_o.append(tensor(b + 2, (d, d), std))
        w.mlp_norm.append(tensor(b + 3, (d,), gain_std, 1.0))
        w.w_gate.append(tensor(b + 4, (f, d), std))
        w.w_up.append(tensor(b + 5, (f, d), std))
        w.w_down.append(tensor(b + 6, (d, f), std))
    return w


# ----------------------------------------------------------------------------------------------
# Prompts
# ----------------------------------------------------------------------------------------------

def make_prompt(wl: Workload, seq: int = 0) -> np.ndarray:
    """Prompt token ids, int32 [P]."""
    g = np.random.Generator(np.random.PCG64([wl.seed, 1000 + seq]))
    V = wl.model.vocab
    if wl.prompt_dist == "zipf":
        ranks = np.arange(1, V + 1, dtype=np.float64)
        cdf = np.cumsum(ranks ** (-wl.zipf_a))
        cdf /= cdf[-1]
        u = g.random(wl.prompt_len)
        ids = np.minimum(np.searchsorted(cdf, u, side="right"), V - 1)
        return ids.astype(np.int32)
    return g.integers(0, V, size=wl.prompt_len, dtype=np.int64).astype(np.int32)


# ----------------------------------------------------------------------------------------------
# Unmask plans
# ----------------------------------------------------------------------------------------------

def cosine_schedule(gen_len: int, n_steps: int) -> np.ndarray:
    """Tokens decoded per step under a cosine schedule.

    The number still masked after step k is m_k = floor(Lg * cos(pi k / (2K))), forced to drop
    by at least one per step and to reach zero at step K; n_k = m_{k-1} - m_k.
    """
    m_prev = gen_len
    n = []
    for k in range(1, n_steps + 1):
        m = 0 if k == n_steps else int(math.floor(gen_len * math.cos(math.pi * k / (2 * n_steps))))
        m = min(m, m_prev - 1)
        m = max(m, 0)
        n.append(m_prev - m)
        m_prev = m
    out = np.array(n, dtype=np.int32)
    assert out.sum() == gen_len and (out >= 1).all()
    return out


def stratified_order(side: int, g: np.random.Generator, cell: int = 4) -> np.ndarray:
    """A seeded 2-D unmask order over a side x side grid (0-based row-major indices).

    The grid is cut into cell x cell tiles; tiles are shuffled, the cells inside each tile are
    shuffled, and the order takes the j-th cell of every tile before any tile's (j+1)-th.
    """
    c = min(cell, side)
    tiles = []
    for ty in range(0, side, c):
        for tx in range(0, side, c):
            cells = [(ty + y) * side + (tx + x) for y in range(c) for x in range(c)
                     if ty + y < side and tx + x < side]
            tiles.append(np.array(cells, dtype=np.int64))
    perm = g.permutation(len(tiles))
    tiles = [g.permutation(tiles[i]) for i in perm]
    out = []
    for j in range(max(len(t) for t in tiles)):
        for t in tiles:
            if j < len(t):
                out.append(int(t[j]))
    return np.array(out, dtype=np.int64)


@dataclass
class Plan:
    """What the sampler decodes at each step.

    kind == "order": step k (1-based) queries order[offsets[k-1]:offsets[k]] and commits all of
    them.  kind == "semiar": blocks of `block` generation positions are processed left to
    right, or in the order `block_order` gives (block indices from 0; a bidirectional task may
    decode a middle block first); at each step the query set is every still-masked position of
    the current block and the `commit` most confident are committed.
    Positions are 1-based absolute positions (P+1..P+Lg).
    """
    kind: str
    n_steps: int
    order: Optional[np.ndarray] = None       # int32 [Lg], positions
    n_per_step: Optional[np.ndarray] = None  # int32 [K]
    block: int = 0
    steps_per_block: int = 0
    commit: int = 0
    block_order: Optional[np.ndarray] = None  # semiar: processing order of the blocks

    @property
    def offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.n_per_step)]).astype(np.int64)

    def query_positions(self, k: int) -> np.ndarray:
        o = self.offsets
        return self.order[o[k - 1]:o[k]]


def make_plan(wl: Workload, seq: int = 0) -> Plan:
    g = np.random.Generator(np.random.PCG64([wl.seed, 2000 + seq]))
    P, Lg = wl.prompt_len, wl.gen_len
    if wl.plan == "perm":
        order = g.permutation(Lg).astype(np.int64)
        n = np.full(wl.n_steps, wl.step_size, np.int32)
        assert n.sum() == Lg
        return Plan("order", wl.n_steps, (order + P + 1).astype(np.int32), n)
    if wl.plan == "cosine":
        if wl.grid_side and wl.grid_side * wl.grid_side == Lg:
            order = stratified_order(wl.grid_side, g)
        else:
            order = g.permutation(Lg).astype(np.int64)
        n = cosine_schedule(Lg, wl.n_steps)
        return Plan("order", wl.n_steps, (order + P + 1).astype(np.int32), n)
    if wl.plan == "semiar":
        assert Lg % wl.block == 0 and wl.block == wl.steps_per_block * wl.commit
        assert wl.n_steps == (Lg // wl.block) * wl.steps_per_block
        return Plan("semiar", wl.n_steps, block=wl.block, steps_per_block=wl.steps_per_block,
                    commit=wl.commit)
    raise ValueError(wl.plan)


@dataclass
class BidirTask:
    """A bidirectional generation task: some generation positions are given (clean from the
    start, computed with the prompt) and the plan decodes only the others.

    kind "inpaint": a centred square hole of half the grid side is masked, the rest given;
    "outpaint": a centred square of half the grid side is given, the rest masked;
    "infill": a seeded half of the positions (1-D, any workload) is given.
    preset_pos: 1-based absolute positions (ascending); preset_tok: their token ids."""
    kind: str
    preset_pos: np.ndarray
    preset_tok: np.ndarray
    plan: Plan


def make_bidir_task(wl: Workload, kind: str, seq: int = 0, n_steps: Optional[int] = None) -> BidirTask:
    g = np.random.Generator(np.random.PCG64([wl.seed, 3000 + seq]))
    P, Lg = wl.prompt_len, wl.gen_len
    given = np.zeros(Lg, dtype=bool)
    if kind in ("inpaint", "outpaint"):
        side = wl.grid_side
        if not side or side * side != Lg:
            raise ValueError("inpaint / outpaint need a square grid workload")
        lo, hi = side // 4, side // 4 + side // 2
        centre = np.zeros((side, side), dtype=bool)
        centre[lo:hi, lo:hi] = True
        given = (~centre if kind == "inpaint" else centre).reshape(-1)
    elif kind == "infill":
        given[g.permutation(Lg)[:Lg // 2]] = True
    else:
        raise ValueError(kind)
    preset_idx = np.flatnonzero(given)
    masked_idx = np.flatnonzero(~given)
    preset_tok = g.integers(0, wl.model.vocab, size=len(preset_idx)).astype(np.int32)
    order = masked_idx[g.permutation(len(masked_idx))]
    K = min(n_steps if n_steps is not None else wl.n_steps, len(order))
    plan = Plan("order", K, (order + P + 1).astype(np.int32), cosine_schedule(len(order), K))
    return BidirTask(kind, (preset_idx + P + 1).astype(np.int32), preset_tok, plan)


def semiar_block(plan: Plan, prompt_len: int, k: int):
    """1-based absolute position range [lo, hi) of the block processed at step k (semi-AR)."""
    b = (k - 1) // plan.steps_per_block
    if plan.block_order is not None:
        b = int(plan.block_order[b])
    lo = prompt_len + 1 + b * plan.block
    return lo, lo + plan.block


def with_batch(wl: Workload, batch: int) -> Workload:
    return replace(wl, batch=batch)
