"""True-sequential quantization of a synthetic Llama-style decoder layer (hidden 512, 4
heads of 128, MLP 1536, 16 sequences of 256 bf16 tokens; 4-bit, group 128, act order)
against the float64 oracle of the same sequence (oracle/decoder_ref.py).

* Forward pieces (rmsnorm, rope, attention, silu * up, residual add) on the same inputs:
  each GPU output within 1 unit in the last place of the 16-bit output type of the
  oracle's exact value (2 for attention, whose fp32 softmax adds a few rounding errors);
  the add is exact.
* Stage by stage: the GPU pipeline is given the oracle's group inputs and checkpoints, so
  every forward step and every group's quantization sees the oracle's inputs: the
  forward's values within the same bounds, and each module's codes, group parameters and
  layer loss at the parity bars.
* End to end (each side on its own): the attention input within 1 unit in the last place,
  the first group's codes at the parity bar, and the layer's output and every module's
  layer loss close to the oracle's (later groups see inputs that already differ by the
  first groups' near-tie code choices).
"""

from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle as O
import oracle.decoder_ref as D
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import synth
from post_weight_quantization_layer_b200.sequential import DecoderShape, quantize_decoder_layer_sequential
from tests.gpu_util import CODE_MATCH, LOSS_RTOL, PARAM_MATCH, PARAM_RTOL, device

pytestmark = pytest.mark.gpu

SHAPE = DecoderShape(hidden=512, heads=4, inter=1536, seq_len=256)
TOKENS = 16 * 256
QCFG = SimpleNamespace(bits=4, group_size=128, damp_percent=0.01, sym=True, desc_act=True, static_groups=False,
                       blocksize=128)
MANT = {torch.bfloat16: 7, torch.float16: 10}


def within_propagated(got, exact, dtype):
    """Elementwise |got - exact| <= 2 ulp(|exact|) + 8 ulp(rms(exact)): values computed from
    16-bit inputs that already differ by near-tie rounding flips (the fp32 and the float64
    accumulation of the linear before them round a few values to neighbouring 16-bit
    numbers); such a flip moves a value by about one unit at the tensor's own scale, which
    is what the second term allows for near-zero values."""
    e = np.asarray(exact, np.float64)
    rms = float(np.sqrt(np.mean(e * e)))
    ulp_e = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(e), 2.0 ** -14))) - MANT[dtype])
    ulp_rms = 2.0 ** (np.floor(np.log2(rms)) - MANT[dtype])
    bound = 2.0 * ulp_e + 8.0 * ulp_rms
    return np.abs(np.asarray(got, np.float64) - e) <= bound, ulps(got, exact, dtype)


def ulps(got, exact, dtype):
    """|got - exact| in units in the last place of `dtype` at |exact| (normal range)."""
    e = np.asarray(exact, np.float64)
    mag = np.maximum(np.abs(e), 2.0 ** -14)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - MANT[dtype])
    return np.abs(np.asarray(got, np.float64) - e) / ulp


_case = {}


def case():
    if not _case:
        h, W, gam = synth.decoder_layer_inputs(SHAPE.hidden, SHAPE.inter, TOKENS, 42)
        ref = D.true_sequential_layer(h.double().numpy(), {k: w.double().numpy() for k, w in W.items()},
                                      [g.double().numpy() for g in gam], SHAPE.heads, SHAPE.seq_len, QCFG)
        _case.update(h=h, W=W, gam=gam, ref=ref)
    return _case


def _dev(x, dtype=None):
    t = torch.as_tensor(x)
    return (t.to(dtype) if dtype is not None else t).to(device()).contiguous()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_forward_pieces_match_oracle(dtype):
    heads, L, T, Dm = 4, 128, 512, 256
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(T, Dm, generator=g) * 2).to(dtype)
    gam = (1 + 0.1 * torch.randn(Dm, generator=g)).to(dtype)
    q, k, v = ((torch.randn(T, Dm, generator=g)).to(dtype) for _ in range(3))
    xn, gn, qn, kn, vn = (t.double().numpy() for t in (x, gam, q, k, v))
    y = gq.api.rmsnorm(_dev(x), _dev(gam), 1e-5)
    assert ulps(y.cpu().double().numpy(), D.rmsnorm(xn, gn, 1e-5), dtype).max() <= 1.0
    r = _dev(q)
    gq.api.rope_(r, heads, L, 10000.0)
    assert ulps(r.cpu().double().numpy(), D.rope(qn, heads, L, 10000.0), dtype).max() <= 1.0
    a = gq.api.attention(_dev(q), _dev(k), _dev(v), heads, L)
    ea = D.attention(qn, kn, vn, heads, L)
    assert ulps(a.cpu().double().numpy(), ea, dtype).max() <= 2.0
    s = gq.api.silu_mul(_dev(q), _dev(k))
    assert ulps(s.cpu().double().numpy(), D.silu_mul(qn, kn), dtype).max() <= 1.0
    ad = gq.api.add(_dev(q), _dev(k))
    torch.cuda.synchronize()
    assert np.array_equal(ad.cpu().double().numpy(), O.round16(qn + kn, "bfloat16" if dtype == torch.bfloat16
                                                                else "float16"))


def _module_metrics(res, ref, W, X):
    bits, n_in = QCFG.bits, W.shape[1]
    codes = O.unpack(res.qweight.cpu().numpy(), bits, n_in)
    sc, zr, gi = res.scales.cpu().numpy(), res.zeros.cpu().numpy(), res.g_idx.cpu().numpy()
    s_ref = ref["scales"].astype(np.float64)
    H = O.hessian(X)
    What = O.dequantize(res.qweight.cpu().numpy(), sc, zr, gi, bits, n_in)
    return dict(code_match=float(np.mean(codes == ref["codes"])),
                param_match=float(np.mean((np.abs(sc - s_ref) <= PARAM_RTOL * np.abs(s_ref)) & (zr == ref["zeros"]))),
                loss_gpu=O.layer_loss_h(W, What, H), loss_ref=O.layer_loss_h(W, ref["What"], H),
                g_idx_equal=bool(np.array_equal(gi, ref["g_idx"])))


def test_stage_by_stage_on_the_oracles_inputs():
    c = case()
    ref = c["ref"]
    dt = torch.bfloat16
    given = {name: {"qweight": _dev(ck[0]), "qzeros": _dev(ck[1]), "scales": _dev(ck[2]),
                    "g_idx": _dev(ck[3].astype(np.int32))} for name, ck in ref["checkpoints"].items()}
    gin = {gi: _dev(X, dt) for gi, X in ref["inputs"].items()}
    out = quantize_decoder_layer_sequential(_dev(c["h"]), {k: _dev(w) for k, w in c["W"].items()},
                                            tuple(_dev(g) for g in c["gam"]), SHAPE, QCFG, given=given,
                                            given_inputs=gin)
    torch.cuda.synchronize()
    assert gq.device_status() == 0
    for gi in (1, 2, 3):
        ok, u = within_propagated(out.forward[gi].cpu().double().numpy(), ref["forward"][gi], dt)
        assert ok.all() and np.mean(u == 0) >= 0.95, (gi, float(u.max()), float(np.mean(u == 0)))
    ok, u = within_propagated(out.output.cpu().double().numpy(), ref["output"], dt)
    assert ok.all() and np.mean(u == 0) >= 0.95, (float(u.max()), float(np.mean(u == 0)))
    for name, W in c["W"].items():
        gi = next(i for i, grp in enumerate(D.GROUPS) if name in grp)
        m = _module_metrics(out.results[name], ref["results"][name], W.double().numpy(), ref["inputs"][gi])
        assert m["code_match"] >= CODE_MATCH, (name, m)
        assert m["param_match"] >= PARAM_MATCH, (name, m)
        assert abs(m["loss_gpu"] - m["loss_ref"]) <= LOSS_RTOL * m["loss_ref"], (name, m)
        assert m["g_idx_equal"], (name, m)


def _unquantized_output(c):
    """The same block in float64 with the original weights (no quantization)."""
    h = c["h"].double().numpy()
    W = {k: w.double().numpy() for k, w in c["W"].items()}
    g1, g2 = (g.double().numpy() for g in c["gam"])
    x = D.rmsnorm(h, g1, SHAPE.eps)
    q = D.rope(x @ W["q"].T, SHAPE.heads, SHAPE.seq_len, SHAPE.rope_base)
    k = D.rope(x @ W["k"].T, SHAPE.heads, SHAPE.seq_len, SHAPE.rope_base)
    h1 = h + D.attention(q, k, x @ W["v"].T, SHAPE.heads, SHAPE.seq_len) @ W["o"].T
    y = D.rmsnorm(h1, g2, SHAPE.eps)
    return h1 + D.silu_mul(y @ W["gate"].T, y @ W["up"].T) @ W["down"].T


def test_end_to_end_against_the_oracles_run():
    """Each side quantizes the layer on its own; after the first group their inputs differ
    by the earlier groups' near-tie code choices, so the later groups are compared through
    their effect: the two runs' outputs differ by less than half of what quantization itself
    changes in the output, and every module's layer loss is within 10 % of the oracle's."""
    c = case()
    ref = c["ref"]
    dt = torch.bfloat16
    out = quantize_decoder_layer_sequential(_dev(c["h"]), {k: _dev(w) for k, w in c["W"].items()},
                                            tuple(_dev(g) for g in c["gam"]), SHAPE, QCFG)
    torch.cuda.synchronize()
    assert gq.device_status() == 0
    x0_ulps = float(ulps(out.inputs[0].cpu().double().numpy(), ref["inputs"][0], dt).max())
    first = {name: _module_metrics(out.results[name], ref["results"][name], c["W"][name].double().numpy(),
                                   ref["inputs"][0]) for name in ("q", "k", "v")}
    o, e = out.output.cpu().double().numpy(), ref["output"]
    ratio = float(np.linalg.norm(o - e) / np.linalg.norm(e - _unquantized_output(c)))
    losses = {}
    for name, W in c["W"].items():
        gi = next(i for i, grp in enumerate(D.GROUPS) if name in grp)
        Wn = W.double().numpy()
        r = out.results[name]
        What = O.dequantize(r.qweight.cpu().numpy(), r.scales.cpu().numpy(), r.zeros.cpu().numpy(),
                            r.g_idx.cpu().numpy(), QCFG.bits, Wn.shape[1])
        losses[name] = (O.layer_loss(Wn, What, out.inputs[gi].cpu().double().numpy()),
                        O.layer_loss(Wn, ref["results"][name]["What"], ref["inputs"][gi]))
    info = dict(x0_ulps=x0_ulps, first={k: (m["code_match"], m["param_match"]) for k, m in first.items()},
                output_diff_over_quant_error=ratio, losses=losses)
    assert x0_ulps <= 1.0, info
    for name, m in first.items():
        assert m["code_match"] >= CODE_MATCH and m["param_match"] >= PARAM_MATCH, info
    assert ratio <= 0.5, info
    for name, (lg, lr) in losses.items():
        assert abs(lg - lr) <= 0.10 * lr, info
