"""Parity at the configs' full layer widths, on sampled output rows.

Rows of W are independent once the factor U is fixed, so the oracle can
recompute any subset of rows exactly: the GPU quantizes the whole layer, the
oracle sweeps a seeded sample of rows against its own fp64 factor of the same
Hessian, and the sampled rows are compared element by element.  The Hessian
comes from the oracle (fp64 2 X^T X of seeded activations on the CPU, rounded
to fp32 for both sides); to keep the CPU work to seconds it uses fewer tokens
than the full calibration set (the Hessian kernel's own full-token parity is in
test_gpu_hessian.py)."""

import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_layer_b200 import synth
import post_weight_quantization_layer_b200 as gq
from tests.gpu_util import CODE_MATCH, LOSS_RTOL, PARAM_MATCH, PARAM_RTOL, device

pytestmark = pytest.mark.gpu

_cache = {}


def _setup(cfgname, layer_name, tokens):
    key = (cfgname, layer_name, tokens)
    if key in _cache:
        return _cache[key]
    cfg = synth.CONFIGS[cfgname]
    layer = next(m for m in cfg.layers if m.name == layer_name)
    W = synth.weight_for(cfg, layer)
    X = synth.acts_for(cfg, layer.h_index, tokens=tokens).full().double().numpy()
    H = O.hessian(X).astype(np.float32)
    _cache[key] = (cfg, layer, W, H)
    return _cache[key]


def _compare_rows(W, H, res, bits, g, sym, desc_act, static, rows, damp):
    n_in = W.shape[1]
    Wn = W.double().numpy()
    Hn = H.astype(np.float64)
    key = ("U", id(H), desc_act, damp)
    if key not in _cache:
        perm = O.act_order_perm(Hn) if desc_act else np.arange(n_in)
        U = O.inverse_cholesky_upper(O.dampen(Hn[np.ix_(perm, perm)], damp))
        _cache[key] = (perm, U)
    perm, U = _cache[key]
    Ws = Wn[rows]
    r = O.gptq_sweep(Ws[:, perm], U, bits, sym, g, perm, static, Ws, 128)
    codes_ref = np.empty_like(r["codes"])
    codes_ref[:, perm] = r["codes"]
    qw = res.qweight.cpu().numpy()[:, rows]
    codes = O.unpack(qw, bits, n_in)
    code_match = float(np.mean(codes == codes_ref))
    sc = res.scales.cpu().numpy()[:, rows]
    zr = res.zeros.cpu().numpy()[:, rows]
    s_ref = r["scales"].astype(np.float64)
    param_match = float(np.mean((np.abs(sc - s_ref) <= PARAM_RTOL * np.abs(s_ref)) & (zr == r["zeros"])))
    gi = res.g_idx.cpu().numpy()
    What = O.dequantize(qw, sc, zr, gi, bits, n_in)
    What_ref = np.empty_like(r["xhat"])
    What_ref[:, perm] = r["xhat"]
    l_gpu = O.layer_loss_h(Ws, What, Hn)
    l_ref = O.layer_loss_h(Ws, What_ref, Hn)
    return dict(code_match=code_match, param_match=param_match, loss_gpu=l_gpu, loss_ref=l_ref)


SWEEP_CASES = [(4, 32, True), (4, 128, True), (3, -1, False), (2, 32, False), (8, 128, True), (3, 128, False)]


@pytest.mark.parametrize("bits,g,sym", SWEEP_CASES)
def test_down_proj_sweep_config(bits, g, sym):
    """4096 x 11008 down_proj shape (the bit-width / grouping sweep), damp 0.01."""
    cfg, layer, W, H = _setup("sweep", "down", 4096)
    dev = device()
    res = gq.quantize_layer(W.to(dev), torch.from_numpy(H).to(dev), bits, g, 0.01, sym, False, False, 128)
    torch.cuda.synchronize()
    rows = np.random.default_rng(bits * 100 + g).choice(layer.n_out, 12, replace=False)
    m = _compare_rows(W, H, res, bits, g, sym, False, False, rows, 0.01)
    assert m["code_match"] >= CODE_MATCH, m
    assert m["param_match"] >= PARAM_MATCH, m
    assert abs(m["loss_gpu"] - m["loss_ref"]) <= LOSS_RTOL * m["loss_ref"], m


def test_llama7b_q_proj_act_order_static():
    """4096 x 4096 q_proj with desc_act and static groups (the 7B decoder-layer setting)."""
    cfg, layer, W, H = _setup("llama7b", "q", 4096)
    dev = device()
    res = gq.quantize_layer(W.to(dev), torch.from_numpy(H).to(dev), 4, 128, 0.01, True, True, True, 128)
    torch.cuda.synchronize()
    rows = np.random.default_rng(7).choice(layer.n_out, 24, replace=False)
    m = _compare_rows(W, H, res, 4, 128, True, True, True, rows, 0.01)
    assert m["code_match"] >= CODE_MATCH, m
    assert m["param_match"] >= PARAM_MATCH, m
    assert abs(m["loss_gpu"] - m["loss_ref"]) <= LOSS_RTOL * m["loss_ref"], m
    assert np.array_equal(res.g_idx.cpu().numpy(), np.arange(4096) // 128)
