"""Pins for the oracle's transformer stack: special cases in which the pre-norm layer reduces to
a closed form or to torch CPU fp64 library routines, and invariants that single out each
operand.  The Sparse-LaViDa pages do not describe the base network, so these pin the synthetic
architecture itself (pre-RMSNorm blocks, rotary q/k, SwiGLU MLP, untied LM head): a dropped
residual, a rotated value, a swapped gate/up pair, a post-norm block, a missing rotation or a
missing 1/sqrt(dh) each fails one of them.  CPU only."""
import copy
import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle
import synth


def _model(n_layers=1, eps=1e-6, seed=21, std=0.3):
    shape = synth.ModelShape(n_layers=n_layers, d_model=32, n_heads=2, d_head=16, d_ffn=48,
                             vocab=40, n_reg=4, dtype=synth.F32, rms_eps=eps)
    return oracle.Model(synth.make_weights(shape, seed, gain_std=0.2, std=std))


def _t(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def _head(m, x):
    """Final RMSNorm and LM head with torch primitives."""
    d = m.shape.d_model
    return F.linear(F.rms_norm(x, (d,), _t(m.final_norm), eps=m.shape.rms_eps), _t(m.lm_head))


def _swiglu_torch(m, l, x):
    """x + W_down (silu(W_gate u) * (W_up u)), u = RMSNorm(x) with the block's MLP gain."""
    L = m.layers[l]
    u = F.rms_norm(x, (m.shape.d_model,), _t(L["mlp_norm"]), eps=m.shape.rms_eps)
    return x + F.linear(F.silu(F.linear(u, _t(L["w_gate"]))) * F.linear(u, _t(L["w_up"])),
                        _t(L["w_down"]))


# ------------------------------------------------------------------------------------------
# (1) Residual stream, final norm and LM head: with every sublayer's output projection zeroed,
#     each row's logits are the normalised embedding times the LM head.
# ------------------------------------------------------------------------------------------

def err_zero_sublayers(m) -> float:
    m = copy.deepcopy(m)
    for L in m.layers:
        L["w_o"][:] = 0.0
        L["w_down"][:] = 0.0
    g = np.random.Generator(np.random.PCG64(31))
    n = 9
    ids = g.integers(0, m.shape.emb_rows, n)
    pos = g.integers(1, 300, n)
    types = np.array([oracle.PROMPT] * 3 + [oracle.CLEAN] * 2 + [oracle.MASK] * 2 +
                     [oracle.REG] * 2)
    labels = np.array([0, 0, 0, 1, 2, 3, 3, 3, 3])
    rows = np.array([8, 0, 4, 5, 2])
    got = oracle.forward_stepcausal(m, ids, pos, types, labels, rows)
    ref = _head(m, _t(m.emb[ids[rows]])).numpy()
    return float(np.max(np.abs(got - ref)))


def test_zero_sublayers_reduce_to_normed_embedding_times_head():
    assert err_zero_sublayers(_model(n_layers=2)) < 1e-12


# ------------------------------------------------------------------------------------------
# (2) One visible key: a row that sees only itself gets softmax weight 1 on its own value, so
#     the block is x + W_o v, v = W_v RMSNorm(x) (no rotation), followed by the SwiGLU MLP.
# ------------------------------------------------------------------------------------------

def err_single_key_block(m) -> float:
    d = m.shape.d_model
    L = m.layers[0]
    w_v = _t(L["w_qkv"][2 * d:3 * d])
    err = 0.0
    for tok, p, ty, lab in ((3, 1, oracle.PROMPT, 0), (17, 250, oracle.PROMPT, 0),
                            (m.shape.mask_id, 77, oracle.MASK, 2),
                            (m.shape.reg_id(1), 301, oracle.REG, 5)):
        got = oracle.forward_stepcausal(m, [tok], [p], [ty], [lab], [0])
        x = _t(m.emb[[tok]])
        h = F.rms_norm(x, (d,), _t(L["attn_norm"]), eps=m.shape.rms_eps)
        x = x + F.linear(F.linear(h, w_v), _t(L["w_o"]))
        ref = _head(m, _swiglu_torch(m, 0, x)).numpy()
        err = max(err, float(np.max(np.abs(got - ref))))
    return err


def test_single_visible_key_block_is_closed_form():
    assert err_single_key_block(_model()) < 1e-12


# ------------------------------------------------------------------------------------------
# (3) SwiGLU: the MLP's update is linear in the up projection and not in the gate projection.
# ------------------------------------------------------------------------------------------

def swiglu_linearity(m):
    """(error of linearity in W_up, departure from linearity in W_gate) for a scale of 3."""
    g = np.random.Generator(np.random.PCG64(32))
    x = g.standard_normal((6, m.shape.d_model))
    base = m.mlp(0, x) - x
    m3 = copy.deepcopy(m)
    m3.layers[0]["w_up"] = 3.0 * m3.layers[0]["w_up"]
    up = m3.mlp(0, x) - x
    m3 = copy.deepcopy(m)
    m3.layers[0]["w_gate"] = 3.0 * m3.layers[0]["w_gate"]
    gate = m3.mlp(0, x) - x
    scale = float(np.max(np.abs(base)))
    return (float(np.max(np.abs(up - 3.0 * base))) / scale,
            float(np.max(np.abs(gate - 3.0 * base))) / scale)


def test_swiglu_is_linear_in_up_only():
    lin_up, lin_gate = swiglu_linearity(_model())
    assert lin_up < 1e-13
    assert lin_gate > 1e-2


# ------------------------------------------------------------------------------------------
# (4) Pre-norm: with eps = 0 each sublayer's update is invariant under scaling its input by a
#     power of two (the normalised input is then bit-identical; only the residual add rounds).
# ------------------------------------------------------------------------------------------

def pre_norm_scale_error(m) -> float:
    g = np.random.Generator(np.random.PCG64(33))
    n = 5
    x = g.standard_normal((n, m.shape.d_model))
    pos = np.arange(1, n + 1)
    vis = np.ones((n, n), bool)

    def updates(xx):
        q, k, v = m.qkv(0, xx, pos)
        return m.attn_out(0, xx, oracle.attention(q, k, v, vis)) - xx, m.mlp(0, xx) - xx

    a1, m1 = updates(x)
    err = 0.0
    for c in (0.25, 4.0):
        ac, mc = updates(c * x)
        err = max(err, float(np.max(np.abs(ac - a1))), float(np.max(np.abs(mc - m1))))
    return err


def test_sublayer_updates_are_scale_free_pre_norm():
    assert pre_norm_scale_error(_model(eps=0.0)) < 1e-13


# ------------------------------------------------------------------------------------------
# (5) Two mutually visible rows: the scores are Re sum_i zq_i conj(zk_i) exp(i (p_q - p_k) w_i)
#     / sqrt(dh), with z = x[:dh/2] + i x[dh/2:] and w_i = theta^(-2i/dh) (the relative form
#     of rotary attention), then a softmax over the two keys.
# ------------------------------------------------------------------------------------------

def err_two_row_rotary(m, p0=5, p1=64) -> float:
    m = copy.deepcopy(m)
    s = m.shape
    d, H, dh, half = s.d_model, s.n_heads, s.d_head, s.d_head // 2
    m.layers[0]["w_down"][:] = 0.0
    L = m.layers[0]
    ids = np.array([7, 29])
    pos = np.array([p0, p1])
    got = oracle.forward_stepcausal(m, ids, pos, [oracle.PROMPT] * 2, [0, 0], [0, 1])
    x = _t(m.emb[ids])
    h = F.rms_norm(x, (d,), _t(L["attn_norm"]), eps=s.rms_eps)
    y = F.linear(h, _t(L["w_qkv"])).numpy()
    q = y[:, :d].reshape(2, H, dh)
    k = y[:, d:2 * d].reshape(2, H, dh)
    v = y[:, 2 * d:].reshape(2, H, dh)
    zq = q[..., :half] + 1j * q[..., half:]
    zk = k[..., :half] + 1j * k[..., half:]
    w = np.array([s.rope_theta ** (-2.0 * i / dh) for i in range(half)])
    o = np.zeros((2, H, dh))
    for r in range(2):
        for hh in range(H):
            sc = [float(np.real(np.sum(zq[r, hh] * np.conj(zk[j, hh]) *
                                       np.exp(1j * (pos[r] - pos[j]) * w)))) / math.sqrt(dh)
                  for j in range(2)]
            e = [math.exp(a - max(sc)) for a in sc]
            o[r, hh] = (e[0] * v[0, hh] + e[1] * v[1, hh]) / (e[0] + e[1])
    xo = x + F.linear(_t(o.reshape(2, d)), _t(L["w_o"]))
    ref = _head(m, xo).numpy()
    return float(np.max(np.abs(got - ref)))


def test_two_row_rotary_attention_is_relative_form():
    m = _model()
    for p0, p1 in ((5, 64), (300, 2), (1, 1)):
        assert err_two_row_rotary(m, p0, p1) < 1e-12


# ------------------------------------------------------------------------------------------
# Planted mistakes: each one trips the pin named in its test.
# ------------------------------------------------------------------------------------------

def test_planted_dropped_residual_is_caught(monkeypatch):
    monkeypatch.setattr(oracle.Model, "attn_out",
                        lambda self, l, x, o: o.reshape(o.shape[0], -1) @ self.layers[l]["w_o"].T)
    assert err_zero_sublayers(_model(n_layers=2)) > 1e-3


def test_planted_wrong_final_gain_is_caught(monkeypatch):
    def logits(self, x):
        h = oracle.rmsnorm(x, self.layers[-1]["mlp_norm"], self.shape.rms_eps)
        return h @ self.lm_head.T

    monkeypatch.setattr(oracle.Model, "logits", logits)
    assert err_zero_sublayers(_model(n_layers=2)) > 1e-3


def test_planted_rotated_value_is_caught(monkeypatch):
    orig = oracle.Model.qkv

    def qkv(self, l, x, pos):
        q, k, v = orig(self, l, x, pos)
        return q, k, oracle.rope(v, pos, self.shape.rope_theta)

    monkeypatch.setattr(oracle.Model, "qkv", qkv)
    assert err_single_key_block(_model()) > 1e-3


def test_planted_mlp_before_attention_is_caught(monkeypatch):
    def forward(m, ids, pos, types, labels, logit_rows):
        ids = np.asarray(ids, dtype=np.int64)
        pos = np.asarray(pos, dtype=np.int64)
        vis = oracle.cross_mask(types, labels, types, labels)
        x = m.emb[ids]
        for l in range(m.shape.n_layers):
            x = m.mlp(l, x)
            q, k, v = m.qkv(l, x, pos)
            x = m.attn_out(l, x, oracle.attention(q, k, v, vis))
        return m.logits(x[np.asarray(logit_rows, dtype=np.int64)])

    monkeypatch.setattr(oracle, "forward_stepcausal", forward)
    assert err_single_key_block(_model()) > 1e-3


def test_planted_gate_up_swap_is_caught(monkeypatch):
    def mlp(self, l, x):
        L = self.layers[l]
        u = oracle.rmsnorm(x, L["mlp_norm"], self.shape.rms_eps)
        return x + (oracle.silu(u @ L["w_up"].T) * (u @ L["w_gate"].T)) @ L["w_down"].T

    monkeypatch.setattr(oracle.Model, "mlp", mlp)
    lin_up, _ = swiglu_linearity(_model())
    assert lin_up > 1e-2


def test_planted_post_norm_is_caught(monkeypatch):
    def mlp(self, l, x):
        L = self.layers[l]
        y = x + (oracle.silu(x @ L["w_gate"].T) * (x @ L["w_up"].T)) @ L["w_down"].T
        return oracle.rmsnorm(y, L["mlp_norm"], self.shape.rms_eps)

    monkeypatch.setattr(oracle.Model, "mlp", mlp)
    assert pre_norm_scale_error(_model(eps=0.0)) > 1e-3


def test_planted_unrotated_keys_are_caught(monkeypatch):
    def qkv(self, l, x, pos):
        s = self.shape
        L = self.layers[l]
        h = oracle.rmsnorm(x, L["attn_norm"], s.rms_eps)
        y = h @ L["w_qkv"].T
        d = s.d_model
        q, k, v = (y[:, i * d:(i + 1) * d].reshape(-1, s.n_heads, s.d_head) for i in range(3))
        return oracle.rope(q, pos, s.rope_theta), k, v

    monkeypatch.setattr(oracle.Model, "qkv", qkv)
    assert err_two_row_rotary(_model(), 5, 64) > 1e-3


def test_planted_missing_score_scale_is_caught(monkeypatch):
    def attention(q, k, v, vis):
        s = np.einsum("qhd,khd->hqk", q, k)
        s = np.where(vis[None], s, -np.inf)
        p = np.exp(s - s.max(-1, keepdims=True))
        p /= p.sum(-1, keepdims=True)
        return np.einsum("hqk,khd->qhd", p, v)

    monkeypatch.setattr(oracle, "attention", attention)
    assert err_two_row_rotary(_model(), 5, 64) > 1e-3
