"""Float64 CPU oracle of quantizing a decoder layer in execution order (test infrastructure).

Only the tests use this module; it shares no code with the CUDA path.

[examples §1.4; OLMo §三] BaseQuantizeConfig.true_sequential: the layer's modules are
quantized in the order the layer runs them, each group's calibration input produced by the
earlier modules with their weights already quantized.  The pages do not spell the block
out; the configurations name Llama-2-shaped layers, and this restates the Llama-2 block
(reading):
    x  = rmsnorm(h) * g1
    a  = attention(rope(x Wq^T), rope(x Wk^T), x Wv^T)      causal, per head
    h1 = h + a Wo^T
    y  = rmsnorm(h1) * g2
    m  = silu(y Wg^T) * (y Wu^T)
    h2 = h1 + m Wd^T
with the groups (q, k, v) on x, (o) on a, (gate, up) on y and (down) on m.  Each group is
quantized by the oracle's GPTQ (gptq_ref.gptq_quantize) on its own Hessian 2 X^T X, and
the forward then uses the quantized weight in its checkpoint form (half-precision scales,
gptq_ref.export_tensors), rounded to the activations' 16-bit type as a 16-bit matrix
multiply takes it.  Every stored activation is rounded to that 16-bit type (nearest even)
at the same points as the GPU pipeline; all arithmetic is float64.
"""

from __future__ import annotations

import numpy as np

from . import gptq_ref as G

GROUPS = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))


def rmsnorm(x, gamma, eps):
    """x / sqrt(mean(x^2) + eps) * gamma, per row (RMS normalisation of the Llama block)."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps) * np.asarray(gamma, np.float64)[None, :]


def rope(x, heads, seq_len, base):
    """Rotary position embedding: in each head of width d the pairs (i, i + d/2) rotate by
    pos * base^(-2i/d), pos = token index within its sequence."""
    x = np.asarray(x, np.float64)
    T, D = x.shape
    d = D // heads
    half = d // 2
    pos = (np.arange(T) % seq_len).astype(np.float64)
    inv = base ** (-2.0 * np.arange(half) / d)
    ang = pos[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    y = x.copy().reshape(T, heads, d)
    a, b = y[:, :, :half].copy(), y[:, :, half:].copy()
    y[:, :, :half] = a * c[:, None, :] - b * s[:, None, :]
    y[:, :, half:] = b * c[:, None, :] + a * s[:, None, :]
    return y.reshape(T, D)


def attention(q, k, v, heads, seq_len):
    """softmax(q k^T / sqrt(d)) v per sequence and head, each query seeing the keys at or
    before it (causal)."""
    q, k, v = (np.asarray(t, np.float64) for t in (q, k, v))
    T, D = q.shape
    d = D // heads
    out = np.empty_like(q)
    mask = np.tril(np.ones((seq_len, seq_len), bool))
    for s0 in range(0, T, seq_len):
        for hh in range(heads):
            cols = slice(hh * d, (hh + 1) * d)
            sc = q[s0:s0 + seq_len, cols] @ k[s0:s0 + seq_len, cols].T / np.sqrt(d)
            sc = np.where(mask, sc, -np.inf)
            sc -= sc.max(axis=1, keepdims=True)
            p = np.exp(sc)
            p /= p.sum(axis=1, keepdims=True)
            out[s0:s0 + seq_len, cols] = p @ v[s0:s0 + seq_len, cols]
    return out


def silu_mul(g, u):
    """silu(g) * u = g / (1 + exp(-g)) * u."""
    g = np.asarray(g, np.float64)
    return g / (1.0 + np.exp(-g)) * np.asarray(u, np.float64)


def true_sequential_layer(h, weights, gammas, heads, seq_len, qcfg, act="bfloat16", rope_base=10000.0, eps=1e-5,
                          given=None, given_inputs=None):
    """Quantize the seven linears of one layer in execution order.

    h [tokens, hidden] and gammas hold 16-bit values; weights {name: W}.  qcfg has bits,
    group_size, damp_percent, sym, desc_act, static_groups.  given / given_inputs as in
    the GPU pipeline (checkpoints {name: (qweight, qzeros, scales16, g_idx)} and group
    inputs {group: X} that replace this run's own).  Returns dict(results {name:
    gptq_quantize output}, checkpoints {name: tuple}, inputs {group: X}, output h2,
    forward {group: X computed by the forward}).
    """
    r16 = lambda a: G.round16(a, act)  # noqa: E731
    given = given or {}
    gin = given_inputs or {}
    bits = qcfg.bits
    out = dict(results={}, checkpoints={}, inputs={}, forward={})
    W16 = {}

    def run_group(gi, X):
        out["inputs"][gi] = X
        H = G.hessian(X)
        for name in GROUPS[gi]:
            r = G.gptq_quantize(np.asarray(weights[name], np.float64), H, bits, qcfg.group_size, qcfg.damp_percent,
                                qcfg.sym, qcfg.desc_act, qcfg.static_groups)
            out["results"][name] = r
            S16, qz = G.export_tensors(r["scales"], r["zeros"], bits)
            ck = given.get(name) or (r["qweight"], qz, S16, r["g_idx"])
            out["checkpoints"][name] = ck
            W16[name] = r16(G.dequantize_checkpoint(ck[0], ck[1], ck[2], ck[3], bits))

    def lin(X, name):
        return r16(G.quantized_linear(X, W16[name]))

    h = np.asarray(h, np.float64)
    x = r16(rmsnorm(h, gammas[0], eps))
    x = gin.get(0, x)
    run_group(0, x)
    q, k, v = lin(x, "q"), lin(x, "k"), lin(x, "v")
    q, k = r16(rope(q, heads, seq_len, rope_base)), r16(rope(k, heads, seq_len, rope_base))
    a = r16(attention(q, k, v, heads, seq_len))
    out["forward"][1] = a
    a = gin.get(1, a)
    run_group(1, a)
    h1 = r16(h + lin(a, "o"))
    y = r16(rmsnorm(h1, gammas[1], eps))
    out["forward"][2] = y
    y = gin.get(2, y)
    run_group(2, y)
    m = r16(silu_mul(lin(y, "gate"), lin(y, "up")))
    out["forward"][3] = m
    m = gin.get(3, m)
    run_group(3, m)
    out["output"] = r16(h1 + lin(m, "down"))
    return out
