"""fp64 CPU oracle for the Sparse-LaViDa sampling step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path: no kernels, tables,
helpers or pre/post-processing.  The only module both sides use is ``synth`` (seeded inputs).

Everything here is plain numpy in float64.  bf16 weights are widened exactly (bf16 -> f64).
Each function cites the passage of the Sparse-LaViDa pages (arXiv 2512.14008; the papernotes.org
CVPR-2026 notes, the paperlayer.ai section summary and the gist.science technical summaries)
that it follows.  Where the pages are silent the reading taken is stated next to the code.

Pinned by ``tests/test_oracle_*.py`` against the worked example, the Figure-3 example, the
two-path training example, brute-force attention, torch CPU fp64 primitives, special cases of the
transformer layer that reduce to closed forms (``test_oracle_layer_pins.py``) and the method's
exactness invariants (training form == incremental form; truncation/dropping of masks outside C).
Logit values of random-init models have no printed counterpart on the pages: beyond those pins
they are "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np

import synth

# Row types.  PROMPT and CLEAN rows are "clean" tokens; MASK and REG rows belong to a masked block.
PROMPT, CLEAN, MASK, REG = 0, 1, 2, 3

POLICY_ALL, POLICY_TOPN = 0, 1


# ----------------------------------------------------------------------------------------------
# Sparse parameterization (papernotes "Key design 1"; paperlayer Sec. 3.1)
# ----------------------------------------------------------------------------------------------

def sparse_encode(seq: Sequence, mask) -> Tuple[list, list, int]:
    """A partially masked sequence -> (clean tokens, their 1-based positions, total length L).

    The masked positions are exactly the positions no clean token occupies, so the triple
    determines the sequence (Sec. 3.1, "I have [m] dog [m] [m] [m]" -> I@1, have@2, dog@4, L=7).
    """
    toks, pos = [], []
    for i, t in enumerate(seq):
        if t != mask:
            toks.append(t)
            pos.append(i + 1)
    return toks, pos, len(seq)


def sparse_decode(toks: Sequence, pos: Sequence[int], length: int, mask) -> list:
    """Inverse of :func:`sparse_encode`: every position not named by a clean token is masked."""
    out = [mask] * length
    for t, p in zip(toks, pos):
        if not 1 <= p <= length:
            raise ValueError("position outside the sequence")
        if out[p - 1] != mask:
            raise ValueError("duplicate position")
        out[p - 1] = t
    return out


# ----------------------------------------------------------------------------------------------
# Step-causal attention mask (papernotes "Key design 3" and the Figure-3 example;
# paperlayer Sec. 3.3 and Appendix 7.3)
# ----------------------------------------------------------------------------------------------

def allowed(tq: int, lq: int, tk: int, lk: int) -> bool:
    """May a query row (type tq, block label lq) attend to a key row (type tk, label lk)?

    Clean rows (prompt = block 0, clean blocks labelled by the step they were decoded at) see
    clean rows of their own or an earlier block.  A masked block -- its mask rows and the
    register rows attached to it, which share its number -- sees every clean row of an earlier
    step and the rows of its own block, never another masked block.  Clean rows never see
    masked or register rows.
    """
    q_clean = tq in (PROMPT, CLEAN)
    k_clean = tk in (PROMPT, CLEAN)
    if k_clean:
        return lk <= lq if q_clean else lk < lq
    if q_clean:
        return False
    return lq == lk


def mask_matrix(types: Sequence[int], labels: Sequence[int]) -> np.ndarray:
    """Boolean [n_query][n_key] visibility for one set of rows (query rows == key rows)."""
    n = len(types)
    m = np.zeros((n, n), dtype=bool)
    for i in range(n):
        for j in range(n):
            m[i, j] = allowed(types[i], labels[i], types[j], labels[j])
    return m


def cross_mask(tq, lq, tk, lk) -> np.ndarray:
    """Visibility of query rows (tq, lq) over key rows (tk, lk) (vectorised predicate)."""
    tq = np.asarray(tq)[:, None]
    lq = np.asarray(lq)[:, None]
    tk = np.asarray(tk)[None, :]
    lk = np.asarray(lk)[None, :]
    q_clean = (tq == PROMPT) | (tq == CLEAN)
    k_clean = (tk == PROMPT) | (tk == CLEAN)
    see_clean = np.where(q_clean, lk <= lq, lk < lq)
    see_masked = (~q_clean) & (lq == lk)
    return np.where(k_clean, see_clean, see_masked)


# ----------------------------------------------------------------------------------------------
# Transformer primitives.  The pages do not describe the base network; the synthetic model is a
# pre-RMSNorm transformer with multi-head attention, SwiGLU MLP, 1-D rotary position embedding on
# the original position ids, and an untied LM head.
# ----------------------------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g, per row."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half 1-D RoPE.  x: [n][H][dh]; pos: [n] original 1-based position ids.

    Pair (i, i + dh/2) is rotated by the angle pos * theta^(-2i/dh).
    """
    dh = x.shape[-1]
    half = dh // 2
    inv = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / dh)
    ang = pos.astype(np.float64)[:, None] * inv[None, :]          # [n][half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, vis: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(dh)) v over the visible keys only.

    q: [nq][H][dh]; k, v: [nk][H][dh]; vis: bool [nq][nk].  Every query must see >= 1 key.
    """
    dh = q.shape[-1]
    qh = np.ascontiguousarray(q.transpose(1, 0, 2))        # [H][nq][dh]
    kh = np.ascontiguousarray(k.transpose(1, 2, 0))        # [H][dh][nk]
    vh = np.ascontiguousarray(v.transpose(1, 0, 2))        # [H][nk][dh]
    s = np.matmul(qh, kh) / math.sqrt(dh)                  # [H][nq][nk]
    s = np.where(vis[None, :, :], s, -np.inf)
    s = s - np.max(s, axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / np.sum(p, axis=-1, keepdims=True)
    return np.matmul(p, vh).transpose(1, 0, 2)             # [nq][H][dh]


class Model:
    """fp64 copy of the synthetic weights (bf16 bit patterns widened exactly)."""

    def __init__(self, w: synth.Weights):
        self.shape = s = w.shape

        def f(a):
            if s.dtype == synth.BF16:
                return synth.bf16_bits_to_f64(a)
            return np.asarray(a, dtype=np.float64)

        self.emb = f(w.emb)
        self.final_norm = f(w.final_norm)
        self.lm_head = f(w.lm_head)
        self.layers = []
        for l in range(s.n_layers):
            self.layers.append(dict(
                attn_norm=f(w.attn_norm[l]), w_qkv=f(w.w_qkv[l]), w_o=f(w.w_o[l]),
                mlp_norm=f(w.mlp_norm[l]), w_gate=f(w.w_gate[l]), w_up=f(w.w_up[l]),
                w_down=f(w.w_down[l])))

    # -- pieces of one layer ------------------------------------------------------------------
    def qkv(self, l: int, x: np.ndarray, pos: np.ndarray):
        s = self.shape
        L = self.layers[l]
        h = rmsnorm(x, L["attn_norm"], s.rms_eps)
        y = h @ L["w_qkv"].T
        d = s.d_model
        q = y[:, :d].reshape(-1, s.n_heads, s.d_head)
        k = y[:, d:2 * d].reshape(-1, s.n_heads, s.d_head)
        v = y[:, 2 * d:].reshape(-1, s.n_heads, s.d_head)
        return rope(q, pos, s.rope_theta), rope(k, pos, s.rope_theta), v

    def attn_out(self, l: int, x: np.ndarray, o: np.ndarray) -> np.ndarray:
        L = self.layers[l]
        return x + o.reshape(o.shape[0], -1) @ L["w_o"].T

    def mlp(self, l: int, x: np.ndarray) -> np.ndarray:
        s = self.shape
        L = self.layers[l]
        u = rmsnorm(x, L["mlp_norm"], s.rms_eps)
        a = silu(u @ L["w_gate"].T) * (u @ L["w_up"].T)
        return x + a @ L["w_down"].T

    def logits(self, x: np.ndarray) -> np.ndarray:
        h = rmsnorm(x, self.final_norm, self.shape.rms_eps)
        return h @ self.lm_head.T


# ----------------------------------------------------------------------------------------------
# Training (parallel) form: one forward over a step-labelled sequence (paperlayer Sec. 3.3,
# Appendix 7.3; papernotes "Key design 3")
# ----------------------------------------------------------------------------------------------

def forward_stepcausal(m: Model, ids, pos, types, labels, logit_rows) -> np.ndarray:
    """Logits [len(logit_rows)][V] of a full forward under the step-causal mask."""
    ids = np.asarray(ids, dtype=np.int64)
    pos = np.asarray(pos, dtype=np.int64)
    vis = cross_mask(types, labels, types, labels)
    x = m.emb[ids]
    for l in range(m.shape.n_layers):
        q, k, v = m.qkv(l, x, pos)
        x = m.attn_out(l, x, attention(q, k, v, vis))
        x = m.mlp(l, x)
    return m.logits(x[np.asarray(logit_rows, dtype=np.int64)])


# ----------------------------------------------------------------------------------------------
# Incremental form: one sampling step over the sparse row set with a KV cache
# (papernotes "a complete example" / Figure 3; paperlayer Sec. 3.2)
# ----------------------------------------------------------------------------------------------

def tail_rows(shape: synth.ModelShape, L: int) -> Tuple[List[int], List[int]]:
    """(ids, positions) of the rows that close a step's sequence and stand for its truncated
    masks (papernotes "Key design 2"; paperlayer Sec. 3.1, Appendix 7.2): n_reg registers
    REG_0.. at positions L+1..L+n_reg.  The register-count ablation (the paper notes' Table 7)
    has a 0-register row: read as the single length token the notes describe before registers
    were added, one [LEN] row at position L+1 (``shape.len_token``).  Either kind takes the
    type REG and the step's label: it follows the masked block's attention rule."""
    if shape.n_reg == 0 and shape.len_token:
        return [shape.len_id], [L + 1]
    return [shape.reg_id(j) for j in range(shape.n_reg)], [L + 1 + j for j in range(shape.n_reg)]


@dataclass
class Packed:
    """The sparse rows of one step: [new-cache | query | register]."""
    ids: np.ndarray
    pos: np.ndarray
    types: np.ndarray
    labels: np.ndarray

    @property
    def n(self) -> int:
        return len(self.ids)


def pack_step(shape: synth.ModelShape, prompt_len: int, gen_len: int, grid: np.ndarray,
              new_pos: Sequence[int], query_pos: Sequence[int], k: int) -> Packed:
    """Rows fed to the network at step k (paperlayer Appendix 7.2: |A| + |C| + m tokens).

    new_pos: positions decoded at step k-1 (enter the cache this step, label k-1, their ids
    read from the grid); query_pos: the decode set C_k (id [MASK], label k); then the tail rows
    (`tail_rows`: n_reg registers with ids REG_0.. and position ids L+1..L+n_reg, label k).
    """
    L = prompt_len + gen_len
    new_pos = np.asarray(new_pos, dtype=np.int64)
    query_pos = np.asarray(query_pos, dtype=np.int64)
    t_ids, t_pos = tail_rows(shape, L)
    n_new, n_q, m = len(new_pos), len(query_pos), len(t_ids)
    ids = np.concatenate([grid[new_pos - prompt_len - 1],
                          np.full(n_q, shape.mask_id),
                          np.asarray(t_ids, dtype=np.int64)]).astype(np.int64)
    if n_new and (ids[:n_new] < 0).any():
        raise ValueError("new-cache position is still masked")
    pos = np.concatenate([new_pos, query_pos, np.asarray(t_pos, dtype=np.int64)]).astype(np.int64)
    types = np.concatenate([np.full(n_new, CLEAN), np.full(n_q, MASK), np.full(m, REG)])
    labels = np.concatenate([np.full(n_new, k - 1), np.full(n_q, k), np.full(m, k)])
    return Packed(ids, pos, types.astype(np.int64), labels.astype(np.int64))


class Incremental:
    """Cached, step-by-step sampler state for one sequence.

    Decoded tokens enter the cache one step after they are sampled: at step k the tokens
    decoded at k-1 are re-embedded with their ids and computed alongside the step-k masks and
    registers; the K/V they get then are kept for every later step (Figure 3; Sec. 3.2).
    """

    def __init__(self, m: Model, prompt: np.ndarray, gen_len: int,
                 preset_pos: Optional[Sequence[int]] = None,
                 preset_tok: Optional[Sequence[int]] = None):
        """preset_pos / preset_tok: generation positions given from the start (bidirectional
        tasks: inpainting, outpainting, infilling).  They are clean tokens of block 0, computed
        with the prompt and cached; the sampler decodes only the other positions."""
        self.m = m
        s = m.shape
        self.P = len(prompt)
        self.Lg = gen_len
        self.L = self.P + gen_len
        self.grid = np.full(gen_len, -1, dtype=np.int64)
        self.k_cache = [np.zeros((0, s.n_heads, s.d_head)) for _ in range(s.n_layers)]
        self.v_cache = [np.zeros((0, s.n_heads, s.d_head)) for _ in range(s.n_layers)]
        self.c_types = np.zeros(0, dtype=np.int64)
        self.c_labels = np.zeros(0, dtype=np.int64)
        self.new_pos = np.zeros(0, dtype=np.int64)   # decoded at the previous step
        self.step_k = 0
        pp = np.zeros(0, dtype=np.int64) if preset_pos is None else np.asarray(preset_pos, np.int64)
        pt = np.zeros(0, dtype=np.int64) if preset_tok is None else np.asarray(preset_tok, np.int64)
        if len(pp) != len(pt) or (len(pp) and ((pp <= self.P).any() or (pp > self.L).any()
                                               or len(np.unique(pp)) != len(pp))):
            raise ValueError("preset positions must be distinct generation positions")
        self.grid[pp - self.P - 1] = pt
        if self.P or len(pp):
            self._prefill(np.asarray(prompt, dtype=np.int64), pp, pt)

    def _prefill(self, prompt: np.ndarray, preset_pos: np.ndarray, preset_tok: np.ndarray):
        """Block 0 — the prompt and any given generation tokens — is computed once and its K/V
        stored (Sec. 3.2); its rows see each other (label 0)."""
        n = self.P + len(preset_pos)
        ids = np.concatenate([prompt, preset_tok]).astype(np.int64)
        pos = np.concatenate([np.arange(1, self.P + 1), preset_pos])
        types = np.concatenate([np.full(self.P, PROMPT), np.full(len(preset_pos), CLEAN)])
        labels = np.zeros(n, dtype=np.int64)
        self._run_rows(self.m.emb[ids], pos, types, labels, keep=np.ones(n, bool))

    def _run_rows(self, x, pos, types, labels, keep) -> np.ndarray:
        """Run all layers for the given rows against the cache; append the `keep` rows' K/V."""
        m = self.m
        vis = cross_mask(types, labels,
                         np.concatenate([self.c_types, types]),
                         np.concatenate([self.c_labels, labels]))
        for l in range(m.shape.n_layers):
            q, k, v = m.qkv(l, x, pos)
            kk = np.concatenate([self.k_cache[l], k])
            vv = np.concatenate([self.v_cache[l], v])
            x = m.attn_out(l, x, attention(q, kk, vv, vis))
            x = m.mlp(l, x)
            self.k_cache[l] = np.concatenate([self.k_cache[l], k[keep]])
            self.v_cache[l] = np.concatenate([self.v_cache[l], v[keep]])
        self.c_types = np.concatenate([self.c_types, types[keep]])
        self.c_labels = np.concatenate([self.c_labels, labels[keep]])
        return x

    @property
    def ctx(self) -> int:
        return len(self.c_types)

    def pack(self, query_pos) -> Packed:
        return pack_step(self.m.shape, self.P, self.Lg, self.grid, self.new_pos, query_pos,
                         self.step_k + 1)

    def step_logits(self, query_pos) -> np.ndarray:
        """Advance to step k+1: run the sparse rows, return logits [n_q][V] for C only."""
        rows = self.pack(query_pos)
        self.step_k += 1
        n_new = len(self.new_pos)
        keep = rows.types == CLEAN
        x = self._run_rows(self.m.emb[rows.ids], rows.pos, rows.types, rows.labels, keep)
        return self.m.logits(x[n_new:n_new + len(query_pos)])

    def commit(self, positions, tokens):
        """Write sampled tokens into the grid; they become next step's new-cache rows."""
        positions = np.asarray(positions, dtype=np.int64)
        tokens = np.asarray(tokens, dtype=np.int64)
        if (self.grid[positions - self.P - 1] >= 0).any():
            raise ValueError("position already decoded")
        self.grid[positions - self.P - 1] = tokens
        self.new_pos = positions


# ----------------------------------------------------------------------------------------------
# Unmasking (papernotes Figure-3 example; paperlayer Sec. 3.2)
# ----------------------------------------------------------------------------------------------

def unmask(logits: np.ndarray, policy: int, n_commit: int = 0):
    """Greedy unmask of the decode set.

    tok = argmax over the content vocabulary (ties -> lowest id); conf = the maximum softmax
    probability.  POLICY_ALL commits every row; POLICY_TOPN commits the n_commit rows of highest
    confidence (ties -> lowest row, i.e. lowest position since rows are in position order).
    Returns (tok [n], conf [n], committed row indices in ascending row order).
    """
    tok = np.argmax(logits, axis=1)
    mx = logits[np.arange(len(tok)), tok]
    conf = 1.0 / np.sum(np.exp(logits - mx[:, None]), axis=1)
    n = len(tok)
    if policy == POLICY_ALL:
        rows = np.arange(n)
    else:
        order = sorted(range(n), key=lambda r: (-conf[r], r))
        rows = np.array(sorted(order[:min(n_commit, n)]), dtype=np.int64)
    return tok, conf, rows


# ----------------------------------------------------------------------------------------------
# Whole runs
# ----------------------------------------------------------------------------------------------

def semiar_queries(grid: np.ndarray, prompt_len: int, lo: int, hi: int) -> np.ndarray:
    """Semi-AR decode set: every still-masked position of the current block, in position order."""
    p = np.arange(lo, hi)
    return p[grid[p - prompt_len - 1] < 0]


@dataclass
class StepRecord:
    k: int
    packed: Packed
    query_pos: np.ndarray
    logits: np.ndarray
    committed_pos: np.ndarray
    committed_tok: np.ndarray


def query_set(plan: synth.Plan, state: Incremental, k: int) -> np.ndarray:
    if plan.kind == "order":
        return np.asarray(plan.query_positions(k), dtype=np.int64)
    lo, hi = synth.semiar_block(plan, state.P, k)
    return semiar_queries(state.grid, state.P, lo, hi)


class Switched(Incremental):
    """Sampler state under the speed switches of the pages' Table 6 (the paper notes' ablation
    section: cache the prompt, cache decoded responses, truncate the masked responses).

    Every switch on is the sparse step of `Incremental`.  Off switches put rows back into each
    step: cache_prompt=False recomputes the prompt (label 0) every step; cache_res=False
    recomputes every decoded token (label = the step it was decoded at) every step instead of
    caching it; truncate=False adds every other still-masked position as a mask row of the step
    (label k, so the decode set sees it).  The step's rows are ordered by label: prompt,
    decoded tokens by decode step (then position), the decode set, the other masks, registers.
    Logits are taken for the decode set only.
    """

    def __init__(self, m: Model, prompt: np.ndarray, gen_len: int, cache_prompt: bool = True,
                 cache_res: bool = True, truncate: bool = True):
        self.cache_prompt, self.cache_res, self.truncate = cache_prompt, cache_res, truncate
        self.prompt_ids = np.asarray(prompt, dtype=np.int64)
        self.decoded_at = np.full(gen_len, -1, dtype=np.int64)
        super().__init__(m, prompt if cache_prompt else np.zeros(0, dtype=np.int64), gen_len)
        self.P = len(prompt)            # positions stay absolute whether or not the prompt is cached
        self.L = self.P + gen_len

    def rows(self, query_pos):
        """(Packed rows of the next step in label order, index of the decode set's first row,
        keep mask of the rows whose K/V enter the cache)."""
        s = self.m.shape
        k = self.step_k + 1
        P, L = self.P, self.L
        query_pos = np.asarray(query_pos, dtype=np.int64)
        ids, pos, types, labels, keep = [], [], [], [], []
        if not self.cache_prompt:
            ids += list(self.prompt_ids); pos += list(range(1, P + 1))
            types += [PROMPT] * P; labels += [0] * P; keep += [False] * P
        if self.cache_res:
            dec = np.asarray(self.new_pos, dtype=np.int64)
        else:
            done = np.flatnonzero(self.grid >= 0)
            done = done[np.lexsort((done, self.decoded_at[done]))]   # by decode step, position
            dec = done + P + 1
        ids += list(self.grid[dec - P - 1]); pos += list(dec); types += [CLEAN] * len(dec)
        labels += list(self.decoded_at[dec - P - 1]); keep += [self.cache_res] * len(dec)
        c0 = len(ids)
        ids += [s.mask_id] * len(query_pos); pos += list(query_pos)
        types += [MASK] * len(query_pos); labels += [k] * len(query_pos); keep += [False] * len(query_pos)
        if not self.truncate:
            inq = set(query_pos.tolist())
            rest = [p for p in range(P + 1, L + 1) if self.grid[p - P - 1] < 0 and p not in inq]
            ids += [s.mask_id] * len(rest); pos += rest; types += [MASK] * len(rest)
            labels += [k] * len(rest); keep += [False] * len(rest)
        t_ids, t_pos = tail_rows(s, L)
        ids += t_ids; pos += t_pos
        types += [REG] * len(t_ids); labels += [k] * len(t_ids); keep += [False] * len(t_ids)
        a = lambda v: np.asarray(v, dtype=np.int64)
        return Packed(a(ids), a(pos), a(types), a(labels)), c0, np.asarray(keep, dtype=bool)

    def step_logits(self, query_pos) -> np.ndarray:
        rows, c0, keep = self.rows(query_pos)
        self.step_k += 1
        x = self._run_rows(self.m.emb[rows.ids], rows.pos, rows.types, rows.labels, keep)
        return self.m.logits(x[c0:c0 + len(query_pos)])

    def commit(self, positions, tokens):
        super().commit(positions, tokens)
        self.decoded_at[np.asarray(positions, dtype=np.int64) - self.P - 1] = self.step_k


def generate(m: Model, prompt: np.ndarray, gen_len: int, plan: synth.Plan,
             max_steps: Optional[int] = None, teacher=None,
             preset_pos: Optional[Sequence[int]] = None,
             preset_tok: Optional[Sequence[int]] = None) -> Tuple[Incremental, List[StepRecord]]:
    """Full sparse sampling run.  `teacher(k, query_pos, logits, tok, rows)` may return
    (positions, tokens) to adopt instead of the oracle's own choice (used by parity tests).
    preset_pos / preset_tok: given generation tokens (bidirectional tasks; see Incremental)."""
    st = Incremental(m, prompt, gen_len, preset_pos, preset_tok)
    recs = []
    K = plan.n_steps if max_steps is None else min(max_steps, plan.n_steps)
    for k in range(1, K + 1):
        qp = query_set(plan, st, k)
        packed = st.pack(qp)
        lg = st.step_logits(qp)
        policy = POLICY_ALL if plan.kind == "order" else POLICY_TOPN
        tok, conf, rows = unmask(lg, policy, plan.commit)
        cpos, ctok = qp[rows], tok[rows]
        if teacher is not None:
            got = teacher(k, qp, lg, tok, conf, rows)
            if got is not None:
                cpos, ctok = got
        st.commit(cpos, ctok)
        recs.append(StepRecord(k, packed, qp, lg, np.asarray(cpos), np.asarray(ctok)))
    return st, recs


def trajectory(prompt: np.ndarray, shape: synth.ModelShape, gen_len: int,
               recs: List[StepRecord], steps: Optional[Sequence[int]] = None,
               preset_pos: Optional[Sequence[int]] = None,
               preset_tok: Optional[Sequence[int]] = None):
    """Training-form sequence that reproduces the queried steps of a finished run in ONE forward.

    Rows: the prompt and any given generation tokens (block 0); for every step j the tokens
    committed at j (clean block j); for every queried step k the decode set C_k as mask rows
    plus its tail rows (`tail_rows`), all labelled k.  Returns (ids, pos, types, labels,
    {k: row indices of C_k}).
    """
    P = len(prompt)
    L = P + gen_len
    ids = list(np.asarray(prompt, dtype=np.int64))
    pos = list(range(1, P + 1))
    types = [PROMPT] * P
    labels = [0] * P
    if preset_pos is not None:
        ids += list(np.asarray(preset_tok, dtype=np.int64))
        pos += list(np.asarray(preset_pos, dtype=np.int64))
        types += [CLEAN] * len(preset_pos)
        labels += [0] * len(preset_pos)
    for r in recs:
        ids += list(r.committed_tok)
        pos += list(r.committed_pos)
        types += [CLEAN] * len(r.committed_pos)
        labels += [r.k] * len(r.committed_pos)
    qrows = {}
    for r in recs:
        if steps is not None and r.k not in steps:
            continue
        start = len(ids)
        nq = len(r.query_pos)
        t_ids, t_pos = tail_rows(shape, L)
        ids += [shape.mask_id] * nq + t_ids
        pos += list(r.query_pos) + t_pos
        types += [MASK] * nq + [REG] * len(t_ids)
        labels += [r.k] * (nq + len(t_ids))
        qrows[r.k] = np.arange(start, start + nq)
    return (np.array(ids), np.array(pos), np.array(types), np.array(labels), qrows)


# ----------------------------------------------------------------------------------------------
# Dense comparator: the standard MDM step (papernotes "Key design 1": every one of the L tokens,
# masks included, goes through full attention and an L x V logit tensor is produced).
# ----------------------------------------------------------------------------------------------

def dense_step_logits(m: Model, prompt: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Logits [Lg][V] of a dense MDM step: all P+Lg rows, [MASK] at undecoded positions,
    no registers, no cache, full bidirectional attention."""
    P = len(prompt)
    ids = np.concatenate([np.asarray(prompt, dtype=np.int64),
                          np.where(grid < 0, m.shape.mask_id, grid)])
    pos = np.arange(1, len(ids) + 1)
    vis = np.ones((len(ids), len(ids)), dtype=bool)
    x = m.emb[ids]
    for l in range(m.shape.n_layers):
        q, k, v = m.qkv(l, x, pos)
        x = m.attn_out(l, x, attention(q, k, v, vis))
        x = m.mlp(l, x)
    return m.logits(x[P:])
