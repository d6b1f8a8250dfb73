"""Seeded synthetic weights and calibration activations.

This module only draws random numbers; it holds none of the quantization
arithmetic.  Both the test suite (for the CPU oracle) and the CUDA-path tests
and benchmark take their inputs from here, so the two sides see the same
tensors.

The pages calibrate real models (OPT-125m, Llama-2-7B/70B) on WikiText-2, C4
or Alpaca text.  Neither the models nor the datasets are available, so these
generators stand in for them with the same shapes and the value structure the
pages describe: Gaussian weights with a few large outliers per row, and
activations with a small set of heavy input channels or heavy-tailed
per-channel scales.

Every draw uses a torch.Generator on the target device, so a tensor is a
function of (seed, shape, device).  Activations are produced in fixed-size
token chunks, each chunk from its own seed, so any chunk can be regenerated
on its own (needed when the full activation matrix is larger than memory).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = [
    "gaussian_weight",
    "outlier_weight",
    "HeavyChannelActs",
    "StudentTActs",
    "LayerSpec",
    "ConfigSpec",
    "CONFIGS",
    "weight_for",
    "acts_for",
    "checkpoint_parts",
    "decoder_layer_inputs",
]

MODULE_INDEX = {"q": 0, "k": 1, "v": 2, "o": 3, "gate": 4, "fc1": 4, "up": 5, "down": 6, "fc2": 6}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian_weight(n_out, n_in, seed, std=0.02, dtype=torch.float32, device="cpu"):
    """W ~ N(0, std^2), drawn in float32 and rounded to ``dtype``."""
    g = _gen(seed, device)
    w = torch.randn(n_out, n_in, generator=g, device=device, dtype=torch.float32) * std
    return w.to(dtype)


def outlier_weight(n_out, n_in, seed, std=0.02, frac=0.005, lo=3.0, hi=5.0,
                   dtype=torch.float16, device="cpu"):
    """Gaussian weights with ceil(frac * n_in) outliers per row.

    In each row the outlier positions are chosen uniformly without
    replacement and set to +-U(lo, hi) times the row's largest |w| of the
    Gaussian part, with an equiprobable sign.
    """
    g = _gen(seed, device)
    w = torch.randn(n_out, n_in, generator=g, device=device, dtype=torch.float32) * std
    k = max(1, math.ceil(frac * n_in))
    rowmax = w.abs().amax(dim=1, keepdim=True)
    keys = torch.rand(n_out, n_in, generator=g, device=device)
    pos = keys.topk(k, dim=1).indices
    mag = lo + (hi - lo) * torch.rand(n_out, k, generator=g, device=device)
    sign = torch.where(torch.rand(n_out, k, generator=g, device=device) < 0.5, -1.0, 1.0)
    w.scatter_(1, pos, sign * mag * rowmax)
    return w.to(dtype)


@dataclass
class HeavyChannelActs:
    """X[t, c] ~ N(0, 1), with ceil(frac * n) channels multiplied by ``mult``.

    The heavy channels are drawn once from ``seed``; token chunk i is drawn
    from seed ``seed * 7919 + 1 + i``.
    """

    n: int
    tokens: int
    seed: int
    frac: float
    mult: float
    dtype: torch.dtype = torch.float16
    chunk: int = 8192

    def _channel_scale(self, device):
        g = _gen(self.seed, device)
        k = max(1, math.ceil(self.frac * self.n))
        idx = torch.randperm(self.n, generator=g, device=device)[:k]
        s = torch.ones(self.n, device=device)
        s[idx] = self.mult
        return s

    @property
    def n_chunks(self):
        return (self.tokens + self.chunk - 1) // self.chunk

    def chunk_rows(self, i):
        t0 = i * self.chunk
        return t0, min(self.tokens, t0 + self.chunk)

    def get_chunk(self, i, device="cpu"):
        t0, t1 = self.chunk_rows(i)
        g = _gen(self.seed * 7919 + 1 + i, device)
        z = torch.randn(t1 - t0, self.n, generator=g, device=device)
        return (z * self._channel_scale(device)).to(self.dtype)

    def full(self, device="cpu"):
        return torch.cat([self.get_chunk(i, device) for i in range(self.n_chunks)], 0)


@dataclass
class StudentTActs(HeavyChannelActs):
    """X[t, c] = sigma_c * z, z ~ N(0, 1), sigma_c = 1 + |tau_c|, tau_c ~ t(nu).

    tau_c is drawn once per channel from ``seed`` (as z / sqrt(chi2_nu / nu)).
    """

    frac: float = 0.0
    mult: float = 1.0
    nu: int = 3

    def _channel_scale(self, device):
        g = _gen(self.seed, device)
        z = torch.randn(self.n, generator=g, device=device)
        chi2 = (torch.randn(self.nu, self.n, generator=g, device=device) ** 2).sum(0)
        tau = z / torch.sqrt(chi2 / self.nu)
        return 1.0 + tau.abs()


def checkpoint_parts(n_out, n_in, bits, group_size, seed, act_order=False, scale_range=(0.002, 0.02)):
    """Random parts of a quantized linear (uniform codes and zero points, log-uniform
    scales rounded to float16, and group indices): codes [n_out, n_in], zeros [G, n_out],
    scales [G, n_out] float16, g_idx [n_in].  With act_order the groups are runs of
    group_size columns in a random column order (g_idx not monotone), as desc_act makes
    them.  Random numbers only; packing is up to the caller."""
    g = _gen(seed, "cpu")
    G = 1 if group_size == -1 else n_in // group_size
    gsz = n_in if group_size == -1 else group_size
    codes = torch.randint(0, 2 ** bits, (n_out, n_in), generator=g)
    zeros = torch.randint(0, 2 ** bits, (G, n_out), generator=g)
    lo, hi = math.log(scale_range[0]), math.log(scale_range[1])
    scales = torch.exp(lo + (hi - lo) * torch.rand(G, n_out, generator=g)).half()
    order = torch.randperm(n_in, generator=g) if act_order else torch.arange(n_in)
    g_idx = torch.empty(n_in, dtype=torch.int32)
    g_idx[order] = (torch.arange(n_in) // gsz).to(torch.int32)
    return codes, zeros, scales, g_idx


def decoder_layer_inputs(hidden, inter, tokens, seed, dtype=torch.bfloat16):
    """Calibration hidden states and weights of one synthetic Llama-style decoder layer:
    h [tokens, hidden] with heavy-tailed channels (the Llama-shaped configs' activation
    law), the seven linear weights with the outlier law (fp16), and the two norm weights
    1 + 0.1 N(0, 1).  Random numbers only."""
    h = StudentTActs(hidden, tokens, seed, dtype=dtype).full()
    shapes = {"q": (hidden, hidden), "k": (hidden, hidden), "v": (hidden, hidden), "o": (hidden, hidden),
              "gate": (inter, hidden), "up": (inter, hidden), "down": (hidden, inter)}
    weights = {name: outlier_weight(no, ni, seed * 10 + MODULE_INDEX[name]) for name, (no, ni) in shapes.items()}
    g = _gen(seed * 10 + 9, "cpu")
    gammas = tuple((1.0 + 0.1 * torch.randn(hidden, generator=g)).to(dtype) for _ in range(2))
    return h, weights, gammas


@dataclass
class LayerSpec:
    name: str
    n_out: int
    n_in: int
    h_index: int


@dataclass
class ConfigSpec:
    key: str
    number: int
    layers: list
    hessian_n: list
    tokens: int
    x_kind: str
    x_dtype: torch.dtype
    w_dtype: torch.dtype
    w_outliers: bool
    bits: int = 4
    group_size: int = 128
    sym: bool = True
    damp_percent: float = 0.01
    desc_act: bool = False
    static_groups: bool = False
    blocksize: int = 128
    x_chunk: int = 8192
    extra: dict = field(default_factory=dict)


def _decoder(hidden, inter, kv=None):
    kv = hidden if kv is None else kv
    return [LayerSpec("q", hidden, hidden, 0), LayerSpec("k", kv, hidden, 0),
            LayerSpec("v", kv, hidden, 0), LayerSpec("o", hidden, hidden, 1),
            LayerSpec("gate", inter, hidden, 2), LayerSpec("up", inter, hidden, 2),
            LayerSpec("down", hidden, inter, 3)]


CONFIGS = {
    "tiny": ConfigSpec("tiny", 1, [LayerSpec("linear", 64, 256, 0)], [256], 512,
                       "heavy", torch.float16, torch.float32, False, bits=4, group_size=32,
                       blocksize=32, x_chunk=512, extra=dict(frac=0.01, mult=20.0)),
    "opt125m": ConfigSpec("opt125m", 2,
                          [LayerSpec("q", 768, 768, 0), LayerSpec("k", 768, 768, 0),
                           LayerSpec("v", 768, 768, 0), LayerSpec("o", 768, 768, 1),
                           LayerSpec("fc1", 3072, 768, 2), LayerSpec("fc2", 768, 3072, 3)],
                          [768, 768, 768, 3072], 128 * 2048, "heavy", torch.float16,
                          torch.float16, True, extra=dict(frac=0.02, mult=30.0)),
    "llama7b": ConfigSpec("llama7b", 3, _decoder(4096, 11008), [4096, 4096, 4096, 11008],
                          128 * 2048, "student_t", torch.bfloat16, torch.float16, True,
                          desc_act=True, static_groups=True),
    "sweep": ConfigSpec("sweep", 4, [LayerSpec("down", 4096, 11008, 0)], [11008], 65536,
                        "student_t", torch.bfloat16, torch.float16, True),
    "llama70b": ConfigSpec("llama70b", 5, _decoder(8192, 28672, kv=1024),
                           [8192, 8192, 8192, 28672], 128 * 4096, "student_t",
                           torch.bfloat16, torch.float16, True),
}


def _w_seed(cfg: ConfigSpec, layer: LayerSpec) -> int:
    if cfg.number == 1:
        return 0
    return 1000 * cfg.number + MODULE_INDEX[layer.name]


def _x_seed(cfg: ConfigSpec, h_index: int) -> int:
    return 1000 * cfg.number + 100 + h_index


def weight_for(cfg: ConfigSpec, layer: LayerSpec, device="cpu", n_out=None):
    """The synthetic weight of one linear layer of a config (optionally only
    its first ``n_out`` rows, which are identical to the full tensor's rows
    only for the Gaussian law; the outlier law is drawn for the full shape)."""
    seed = _w_seed(cfg, layer)
    rows = layer.n_out if n_out is None else n_out
    if cfg.w_outliers:
        return outlier_weight(rows, layer.n_in, seed, dtype=cfg.w_dtype, device=device)
    return gaussian_weight(rows, layer.n_in, seed, dtype=cfg.w_dtype, device=device)


def acts_for(cfg: ConfigSpec, h_index: int, tokens=None):
    """The calibration activations feeding Hessian ``h_index`` of a config."""
    n = cfg.hessian_n[h_index]
    T = cfg.tokens if tokens is None else tokens
    seed = _x_seed(cfg, h_index)
    if cfg.x_kind == "heavy":
        return HeavyChannelActs(n, T, seed, cfg.extra["frac"], cfg.extra["mult"],
                                cfg.x_dtype, chunk=cfg.x_chunk)
    return StudentTActs(n, T, seed, dtype=cfg.x_dtype, chunk=cfg.x_chunk)
