"""Arithmetic of the opt-in device paths, restated and checked against the oracle (CPU).

The split-QKV finalize kernel (SMDM_QKV_SPLIT=1) rotates q and k itself from the fp32 sums:
for head h and i < dh/2, the pair (h*dh + i, h*dh + i + dh/2) becomes
(x1 cos - x2 sin, x2 cos + x1 sin) with the angle table entry [pos][i] = (cos, sin) of
pos * theta^(-2i/dh).  This restates that indexing and checks it against the oracle's
rotate-half RoPE, so a swapped sign or partner in the kernel's formula shows here first."""
import numpy as np

import oracle


def finalize_rotation(x, pos, n_heads, dh, theta):
    """x: [rows][n_heads * dh] fp64; the finalize kernel's pairs and angle table."""
    half = dh // 2
    inv = theta ** (-(2.0 * np.arange(half)) / dh)
    table = np.stack([np.cos(np.outer(np.arange(pos.max() + 1), inv)),
                      np.sin(np.outer(np.arange(pos.max() + 1), inv))], axis=-1)
    out = np.empty_like(x)
    for r in range(x.shape[0]):
        for t in range(n_heads * half):
            h, i = divmod(t, half)
            f1, f2 = h * dh + i, h * dh + i + half
            c, s = table[pos[r], i]
            out[r, f1] = x[r, f1] * c - x[r, f2] * s
            out[r, f2] = x[r, f2] * c + x[r, f1] * s
    return out


def test_finalize_rotation_is_the_oracle_rope():
    g = np.random.Generator(np.random.PCG64(29))
    rows, H, dh, theta = 5, 3, 16, 10000.0
    x = g.standard_normal((rows, H * dh))
    pos = g.integers(1, 900, rows)
    ref = oracle.rope(x.reshape(rows, H, dh), pos, theta).reshape(rows, H * dh)
    np.testing.assert_allclose(finalize_rotation(x, pos, H, dh, theta), ref, rtol=0, atol=1e-12)
