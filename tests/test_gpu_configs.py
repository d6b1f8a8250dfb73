"""Parity for every configuration on its own Hessians, at full calibration token counts.

Configurations: the OPT-125m-shaped decoder layer (6 linears, 262,144 fp16 tokens), the
Llama-2-7B-shaped decoder layer (7 linears, 262,144 bf16 tokens, desc_act + static
groups) and the 4096 x 11008 bit-width / grouping sweep (65,536 bf16 tokens, 24 cells at
damp 0.005 and 0.01).  The tiny layer is covered in test_gpu_quantize.py and the
Llama-2-70B-shaped layer in test_gpu_70b.py.

Each phase is compared on its own, so that a later phase's parity does not absorb an
earlier phase's rounding:

* Hessian: the GPU accumulates H = 2 X^T X over all of the configuration's tokens,
  streamed in 8,192-token chunks; the oracle accumulates the same chunks in float64
  (relative Frobenius error <= 1e-5, full matrices).
* Factor and sweep: the oracle's float64 H, rounded to fp32 (the API's Hessian type), is
  the input of both sides.  The GPU runs the benched path (layer.quantize_decoder_layer:
  every distinct Hessian of the layer factored in one batched call, each linear swept
  against its factor); the oracle factors the same fp32 H and sweeps the same rows.
  Rows of W are independent once the factor is fixed, so for the large linears the
  oracle sweeps a seeded sample of rows and those rows are compared element by element.

Bars (the same as every GPU parity test): H rel-Frobenius <= 1e-5; U row-relative
<= 1e-7; permutation and g_idx exact; codes >= 99.5 % identical; scales within 1e-3
relative and zeros equal in >= 99.9 % of groups; layer loss within 1 %.
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import synth
from post_weight_quantization_layer_b200.layer import quantize_decoder_layer
from tests.gpu_util import CODE_MATCH, H_REL_FROB, LOSS_RTOL, PARAM_MATCH, PARAM_RTOL, device, rel_frob

pytestmark = pytest.mark.gpu

U_ROW_RTOL = 1e-7


def stream_hessian(cfg, h_index, tokens=None):
    """The GPU's and the oracle's H over the same token chunks (drawn on the GPU).
    Returns (H_gpu as float64 numpy, H_oracle float64)."""
    dev = device()
    acts = synth.acts_for(cfg, h_index, tokens=tokens)
    n = acts.n
    Hg = torch.zeros(n, n, dtype=torch.float32, device=dev)
    Hr = np.zeros((n, n))
    for i in range(acts.n_chunks):
        X = acts.get_chunk(i, device=dev)
        gq.accumulate_hessian(X, Hg)
        Hr += O.hessian(X.cpu().double().numpy())
        del X
    torch.cuda.synchronize()
    assert gq.device_status() == 0
    return Hg.double().cpu().numpy(), Hr


def oracle_factor(H64, damp, desc_act):
    perm = O.act_order_perm(H64) if desc_act else np.arange(H64.shape[0])
    U = O.inverse_cholesky_upper(O.dampen(H64[np.ix_(perm, perm)], damp))
    return perm, U


def u_row_error(Ug, Ur):
    return float((np.abs(Ug - Ur).max(axis=1) / np.abs(Ur).max(axis=1)).max())


def sweep_rows_metrics(Wn, H64, perm, U, res, cfg, rows, bits, g, sym, static):
    """GPU outputs of the given rows against the oracle's sweep of the same rows."""
    n_in = Wn.shape[1]
    Ws = Wn[rows]
    r = O.gptq_sweep(Ws[:, perm], U, bits, sym, g, perm, static, Ws, cfg.blocksize)
    codes_ref = np.empty_like(r["codes"])
    codes_ref[:, perm] = r["codes"]
    What_ref = np.empty_like(r["xhat"])
    What_ref[:, perm] = r["xhat"]
    qw = res.qweight.cpu().numpy()[:, rows]
    sc = res.scales.cpu().numpy()[:, rows]
    zr = res.zeros.cpu().numpy()[:, rows]
    gi = res.g_idx.cpu().numpy()
    codes = O.unpack(qw, bits, n_in)
    s_ref = r["scales"].astype(np.float64)
    g_ref = np.empty(n_in, np.int64)
    g_ref[perm] = r["gsweep"]
    What = O.dequantize(qw, sc, zr, gi, bits, n_in)
    return dict(code_match=float(np.mean(codes == codes_ref)),
                param_match=float(np.mean((np.abs(sc - s_ref) <= PARAM_RTOL * np.abs(s_ref)) & (zr == r["zeros"]))),
                loss_gpu=O.layer_loss_h(Ws, What, H64), loss_ref=O.layer_loss_h(Ws, What_ref, H64),
                g_idx_equal=bool(np.array_equal(gi, g_ref)))


def assert_sweep(m, what):
    assert m["code_match"] >= CODE_MATCH, (what, m)
    assert m["param_match"] >= PARAM_MATCH, (what, m)
    assert abs(m["loss_gpu"] - m["loss_ref"]) <= LOSS_RTOL * m["loss_ref"], (what, m)
    assert m["g_idx_equal"], (what, m)


class LayerCase:
    """One decoder-layer configuration: Hessians on both sides, the benched GPU path on the
    oracle's fp32 Hessians, and the oracle's factors of the same Hessians."""

    def __init__(self, cfgname):
        cfg = synth.CONFIGS[cfgname]
        dev = device()
        self.cfg = cfg
        self.h_err = {}
        self.H64 = {}
        for h in range(len(cfg.hessian_n)):
            Hg, Hr = stream_hessian(cfg, h)
            self.h_err[h] = rel_frob(Hg, Hr)
            del Hg
            self.H64[h] = Hr.astype(np.float32).astype(np.float64)  # the shared fp32 input
        self.W = {m.name: synth.weight_for(cfg, m) for m in cfg.layers}
        Hdev = {h: torch.from_numpy(H.astype(np.float32)).to(dev) for h, H in self.H64.items()}
        self.results, _ = quantize_decoder_layer(None, {k: w.to(dev) for k, w in self.W.items()}, cfg.layers, cfg,
                                                 hessians=Hdev, hessians_given=True)
        # the factors the layer path computed internally, by the same batched call
        keys = sorted(Hdev)
        outs = gq.factor_hessians([Hdev[h] for h in keys], cfg.damp_percent, cfg.desc_act)
        torch.cuda.synchronize()
        self.gpu_factor = {h: (U.cpu().numpy(), p.cpu().numpy()) for h, (U, p) in zip(keys, outs)}
        del Hdev, outs
        self.ref_factor = {h: oracle_factor(H, cfg.damp_percent, cfg.desc_act) for h, H in self.H64.items()}


_cases = {}


def layer_case(name):
    if name not in _cases:
        _cases.clear()  # keep one configuration's matrices alive at a time
        _cases[name] = LayerCase(name)
    return _cases[name]


# ------------------------------------------------------------------ OPT-125m-shaped layer (all rows)
OPT = synth.CONFIGS["opt125m"]


@pytest.mark.parametrize("h", range(len(OPT.hessian_n)))
def test_opt125m_hessian_full_tokens(h):
    c = layer_case("opt125m")
    assert c.h_err[h] <= H_REL_FROB, (h, c.h_err[h])


@pytest.mark.parametrize("h", range(len(OPT.hessian_n)))
def test_opt125m_factor(h):
    c = layer_case("opt125m")
    Ug, pg = c.gpu_factor[h]
    pr, Ur = c.ref_factor[h]
    assert np.array_equal(pg, pr)
    assert u_row_error(Ug, Ur) <= U_ROW_RTOL


@pytest.mark.parametrize("name", [m.name for m in OPT.layers])
def test_opt125m_linear_all_rows(name):
    c = layer_case("opt125m")
    mod = next(m for m in OPT.layers if m.name == name)
    Wn = c.W[name].double().numpy()
    perm, U = c.ref_factor[mod.h_index]
    m = sweep_rows_metrics(Wn, c.H64[mod.h_index], perm, U, c.results[name], OPT, np.arange(mod.n_out),
                           OPT.bits, OPT.group_size, OPT.sym, OPT.static_groups)
    assert_sweep(m, name)


# ------------------------------------------------------------------ Llama-2-7B-shaped layer (the benched one)
L7 = synth.CONFIGS["llama7b"]
L7_ROWS = 64


@pytest.mark.parametrize("h", range(len(L7.hessian_n)))
def test_llama7b_hessian_full_tokens(h):
    c = layer_case("llama7b")
    assert c.h_err[h] <= H_REL_FROB, (h, c.h_err[h])


@pytest.mark.parametrize("h", range(len(L7.hessian_n)))
def test_llama7b_factor(h):
    c = layer_case("llama7b")
    Ug, pg = c.gpu_factor[h]
    pr, Ur = c.ref_factor[h]
    assert np.array_equal(pg, pr)  # desc_act order, ties by index
    assert u_row_error(Ug, Ur) <= U_ROW_RTOL


@pytest.mark.parametrize("name", [m.name for m in L7.layers])
def test_llama7b_linear_sampled_rows(name):
    c = layer_case("llama7b")
    mod = next(m for m in L7.layers if m.name == name)
    Wn = c.W[name].double().numpy()
    perm, U = c.ref_factor[mod.h_index]
    rows = np.sort(np.random.default_rng(3000 + mod.n_out + 7 * mod.h_index).choice(mod.n_out, L7_ROWS,
                                                                                     replace=False))
    m = sweep_rows_metrics(Wn, c.H64[mod.h_index], perm, U, c.results[name], L7, rows, L7.bits, L7.group_size,
                           L7.sym, L7.static_groups)
    assert_sweep(m, name)
    # static groups: g_idx is the plain c // g even under act order
    assert np.array_equal(c.results[name].g_idx.cpu().numpy(), np.arange(mod.n_in) // L7.group_size)


# ------------------------------------------------------------------ bit-width / grouping sweep (4096 x 11008)
SW = synth.CONFIGS["sweep"]
SW_ROWS = 16
CELLS = [(b, g, s) for b in (2, 3, 4, 8) for g in (32, 128, -1) for s in (True, False)]
DAMPS = (0.005, 0.01)


class SweepCase:
    def __init__(self):
        dev = device()
        Hg, Hr = stream_hessian(SW, 0)
        self.h_err = rel_frob(Hg, Hr)
        del Hg
        self.H64 = Hr.astype(np.float32).astype(np.float64)
        H32 = torch.from_numpy(self.H64.astype(np.float32)).to(dev)
        self.W = synth.weight_for(SW, SW.layers[0])
        self.Wdev = self.W.to(dev)
        self.gpu = {}
        self.ref = {}
        for d in DAMPS:
            U, p = gq.factor_hessian(H32, d, False)
            self.gpu[d] = (U, p)
            self.ref[d] = oracle_factor(self.H64, d, False)
        torch.cuda.synchronize()


_sweep = []


def sweep_case():
    if not _sweep:
        _cases.clear()
        _sweep.append(SweepCase())
    return _sweep[0]


def test_sweep_config_hessian_full_tokens():
    c = sweep_case()
    assert c.h_err <= H_REL_FROB, c.h_err


@pytest.mark.parametrize("damp", DAMPS)
def test_sweep_config_factor(damp):
    c = sweep_case()
    U, p = c.gpu[damp]
    pr, Ur = c.ref[damp]
    assert np.array_equal(p.cpu().numpy(), pr)
    assert u_row_error(U.cpu().numpy(), Ur) <= U_ROW_RTOL


@pytest.mark.parametrize("damp", DAMPS)
@pytest.mark.parametrize("bits,g,sym", CELLS)
def test_sweep_config_cell(damp, bits, g, sym):
    c = sweep_case()
    U, p = c.gpu[damp]
    res = gq.quantize_layer_factored(c.Wdev, U, p, bits, g, sym, False, SW.blocksize)
    torch.cuda.synchronize()
    perm, Ur = c.ref[damp]
    rows = np.sort(np.random.default_rng(bits * 1000 + (g % 1000) * 3 + sym).choice(SW.layers[0].n_out, SW_ROWS,
                                                                                    replace=False))
    m = sweep_rows_metrics(c.W.double().numpy(), c.H64, perm, Ur, res, SW, rows, bits, g, sym, False)
    assert_sweep(m, (damp, bits, g, sym))
