"""Pins of the decoder-layer oracle (oracle/decoder_ref.py) against closed forms and the
defining properties of each piece, and of the true-sequential composition."""

from types import SimpleNamespace

import numpy as np
import torch

import oracle.decoder_ref as D
from oracle import gptq_ref as O


def test_rmsnorm_unit_rms_and_constant_rows():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 64)) * 3.0
    y = D.rmsnorm(x, np.ones(64), 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, atol=1e-14)
    c = np.full((1, 8), -2.0)
    g = np.arange(1, 9, dtype=np.float64)
    assert np.allclose(D.rmsnorm(c, g, 0.0), -g, atol=1e-15)


def test_rope_identity_at_zero_norm_preserving_and_relative():
    rng = np.random.default_rng(1)
    heads, d, L = 2, 16, 32
    x = rng.standard_normal((L, heads * d))
    y = D.rope(x, heads, L, 10000.0)
    assert np.allclose(y[0], x[0], atol=0)  # position 0: no rotation
    xr, yr = x.reshape(L, heads, d), y.reshape(L, heads, d)
    nx = xr[:, :, :d // 2] ** 2 + xr[:, :, d // 2:] ** 2
    ny = yr[:, :, :d // 2] ** 2 + yr[:, :, d // 2:] ** 2
    assert np.allclose(nx, ny, rtol=1e-13)
    # <rope(q at m), rope(k at n)> depends only on m - n
    q, k = rng.standard_normal(d), rng.standard_normal(d)

    def at(v, p):
        z = np.zeros((L, d))
        z[p] = v
        return D.rope(z, 1, L, 10000.0)[p]
    assert np.isclose(at(q, 7) @ at(k, 3), at(q, 20) @ at(k, 16), rtol=1e-12)
    # the first pair rotates by exactly pos radians (inverse frequency 1)
    z = np.zeros((L, d))
    z[:, 0] = 1.0
    r = D.rope(z, 1, L, 10000.0)
    assert np.allclose(r[:, 0], np.cos(np.arange(L)), atol=1e-15)
    assert np.allclose(r[:, d // 2], np.sin(np.arange(L)), atol=1e-15)


def test_attention_closed_forms_and_causality():
    rng = np.random.default_rng(2)
    heads, d, L = 2, 8, 12
    v = rng.standard_normal((2 * L, heads * d))
    q = rng.standard_normal((2 * L, heads * d))
    k = np.ones((2 * L, heads * d))  # equal keys: uniform weights over the causal prefix
    out = D.attention(q, k, v, heads, L)
    for s0 in (0, L):
        cm = np.cumsum(v[s0:s0 + L], axis=0) / np.arange(1, L + 1)[:, None]
        assert np.allclose(out[s0:s0 + L], cm, atol=1e-13)
    # the first token of each sequence attends only to itself
    k2 = rng.standard_normal(k.shape)
    o2 = D.attention(q, k2, v, heads, L)
    assert np.allclose(o2[[0, L]], v[[0, L]], atol=1e-14)
    # changing later tokens leaves earlier outputs unchanged
    k3, v3 = k2.copy(), v.copy()
    k3[5:L] += 1.0
    v3[5:L] -= 2.0
    o3 = D.attention(q, k3, v3, heads, L)
    assert np.array_equal(o3[:5], o2[:5])


def test_silu_mul_values():
    g = np.array([0.0, 1.0, -1.0, 40.0])
    y = D.silu_mul(g, np.ones(4))
    assert y[0] == 0.0
    assert np.isclose(y[1], 1.0 / (1.0 + np.exp(-1.0)), rtol=1e-15)
    assert np.isclose(y[1] - y[2], 1.0, rtol=1e-15)  # silu(x) - silu(-x) = x
    assert np.isclose(y[3], 40.0, rtol=1e-15)


def test_true_sequential_composition():
    """Group inputs follow the block's definition; feeding a run its own inputs back
    changes nothing; and at 8 bits the quantized layer's output stays close to the
    unquantized forward of the same block."""
    from post_weight_quantization_layer_b200 import synth
    hidden, inter, heads, L, T = 64, 128, 2, 16, 256
    h, W, gam = synth.decoder_layer_inputs(hidden, inter, T, 3)
    h, gam = h.double().numpy(), [g.double().numpy() for g in gam]
    Wn = {k: w.double().numpy() for k, w in W.items()}
    cfg = SimpleNamespace(bits=8, group_size=32, damp_percent=0.01, sym=True, desc_act=True, static_groups=False)
    r = D.true_sequential_layer(h, Wn, gam, heads, L, cfg)
    r16 = lambda a: O.round16(a, "bfloat16")  # noqa: E731
    assert np.array_equal(r["inputs"][0], r16(D.rmsnorm(h, gam[0], 1e-5)))
    r2 = D.true_sequential_layer(h, Wn, gam, heads, L, cfg, given=r["checkpoints"], given_inputs=r["inputs"])
    assert np.array_equal(r2["output"], r["output"])
    for name in Wn:
        assert np.array_equal(r2["results"][name]["codes"], r["results"][name]["codes"])
    # unquantized forward of the same block in float64
    x = D.rmsnorm(h, gam[0], 1e-5)
    q, k = D.rope(x @ Wn["q"].T, heads, L, 1e4), D.rope(x @ Wn["k"].T, heads, L, 1e4)
    a = D.attention(q, k, x @ Wn["v"].T, heads, L)
    h1 = h + a @ Wn["o"].T
    y = D.rmsnorm(h1, gam[1], 1e-5)
    h2 = h1 + D.silu_mul(y @ Wn["gate"].T, y @ Wn["up"].T) @ Wn["down"].T
    assert np.linalg.norm(r["output"] - h2) / np.linalg.norm(h2) < 1e-2
