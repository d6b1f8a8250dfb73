"""Quantize a Llama-style decoder layer in execution order (true_sequential).

AutoGPTQ examples guide §1.4 / OLMo quick-start §三: with true_sequential the modules of a
layer are quantized one group at a time in the order the layer runs them, and each group's
calibration input is produced by the layer's earlier modules with their weights already
quantized.  For the Llama block (rmsnorm, attention, rmsnorm, gated MLP) the groups are
(q, k, v) on the attention input, (o) on the attention output, (gate, up) on the MLP input
and (down) on the MLP's gated product.  Every step runs in the native library: the forward
pieces (gptq_rmsnorm, gptq_rope, gptq_attention, gptq_silu_mul, gptq_add), the linears on
the quantized checkpoints (gptq_quantized_linear), and for each group the Hessian, one
factor and one sweep per module (as layer.py) followed by the checkpoint export.  This
module only sequences the calls.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import api
from .export import export_layer

GROUPS = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))


@dataclass
class DecoderShape:
    hidden: int
    heads: int
    inter: int
    seq_len: int
    rope_base: float = 10000.0
    eps: float = 1e-5

    @property
    def head_dim(self):
        return self.hidden // self.heads


@dataclass
class SequentialResult:
    results: dict = field(default_factory=dict)      # module -> QuantResult (fp32 scales, zeros)
    checkpoints: dict = field(default_factory=dict)  # module -> checkpoint tensors used by the forward
    inputs: dict = field(default_factory=dict)       # group index -> calibration input X of that group
    output: torch.Tensor | None = None               # the layer's output hidden states
    forward: dict = field(default_factory=dict)      # group -> X computed by the forward (given-input runs)


def _quantize_group(X, names, weights, qcfg, stream):
    n = X.shape[1]
    H = torch.zeros(n, n, dtype=torch.float32, device=X.device)
    api.accumulate_hessian(X, H, stream=stream)
    # one factor, the group's sweeps side by side (gptq_quantize_linears)
    _, res = api.quantize_linears([H], [(weights[name], 0) for name in names], qcfg.bits, qcfg.group_size,
                                  qcfg.damp_percent, qcfg.sym, qcfg.desc_act, qcfg.static_groups, qcfg.blocksize,
                                  stream=stream)
    return dict(zip(names, res))


def quantize_decoder_layer_sequential(h, weights, gammas, shape: DecoderShape, qcfg, given=None, given_inputs=None,
                                      stream=None):
    """Quantize the seven linears of one decoder layer in execution order.

    h:       [tokens, hidden] calibration hidden states entering the layer (fp16/bf16;
             tokens = whole sequences of shape.seq_len)
    weights: {q, k, v, o, gate, up, down: [n_out, n_in] weight}
    gammas:  (attention-norm weight, MLP-norm weight), each [hidden] in h's dtype
    qcfg:    bits, group_size, damp_percent, sym, desc_act, static_groups, blocksize
    given:   optional {module: checkpoint tensors} used by the forward in place of this
             run's own quantization of that module (to check a later group on an earlier
             group's reference result); the module is still quantized and reported.
    given_inputs: optional {group index: X} used as that group's calibration input (and as
             the forward's value at that point) in place of the computed one; with `given`
             this checks every forward step and every group's quantization on the same
             inputs as a reference run.
    Returns a SequentialResult.
    """
    given = given or {}
    gin = given_inputs or {}
    stream = stream or torch.cuda.current_stream()
    res = SequentialResult()
    heads, L, bits = shape.heads, shape.seq_len, qcfg.bits

    def run_group(g, X):
        res.inputs[g] = X
        out = _quantize_group(X, GROUPS[g], weights, qcfg, stream)
        for name, r in out.items():
            res.results[name] = r
            res.checkpoints[name] = given.get(name) or export_layer(r, bits, stream=stream)

    def lin(X, name):
        return api.quantized_linear(X, res.checkpoints[name], bits, stream=stream)

    with torch.cuda.stream(stream):
        x = gin.get(0, None)
        x = api.rmsnorm(h, gammas[0], shape.eps, stream=stream) if x is None else x
        run_group(0, x)
        q, k, v = lin(x, "q"), lin(x, "k"), lin(x, "v")
        api.rope_(q, heads, L, shape.rope_base, stream=stream)
        api.rope_(k, heads, L, shape.rope_base, stream=stream)
        a = gin.get(1, None)
        a = api.attention(q, k, v, heads, L, stream=stream) if a is None else a
        run_group(1, a)
        h1 = api.add(h, lin(a, "o"), stream=stream)
        y = gin.get(2, None)
        y = api.rmsnorm(h1, gammas[1], shape.eps, stream=stream) if y is None else y
        run_group(2, y)
        m = gin.get(3, None)
        m = api.silu_mul(lin(y, "gate"), lin(y, "up"), stream=stream) if m is None else m
        run_group(3, m)
        res.output = api.add(h1, lin(m, "down"), stream=stream)
        # the forward's own values where inputs were given, for comparison
        res.forward = {}
        if gin:
            res.forward[1] = api.attention(q, k, v, heads, L, stream=stream) if 1 in gin else a
            res.forward[2] = api.rmsnorm(h1, gammas[1], shape.eps, stream=stream) if 2 in gin else y
            res.forward[3] = api.silu_mul(lin(y, "gate"), lin(y, "up"), stream=stream) if 3 in gin else m
    return res
