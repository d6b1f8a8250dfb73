"""GPU parity of gptq_quantize_layer and the factor/sweep split against the oracle.

Both sides receive the same W and the same fp32 Hessian (computed by the oracle
from seeded activations and rounded to fp32)."""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import synth
from tests.gpu_util import assert_parity, compare_quant, device

pytestmark = pytest.mark.gpu


def _problem(n_out, n_in, T, seed, w_dtype=torch.float16, x_dtype=torch.float16, outliers=True):
    if outliers:
        W = synth.outlier_weight(n_out, n_in, seed, dtype=w_dtype)
    else:
        W = synth.gaussian_weight(n_out, n_in, seed, dtype=w_dtype)
    X = synth.StudentTActs(n_in, T, seed + 1, dtype=x_dtype).full()
    H = torch.from_numpy(O.hessian(X.double().numpy())).float()
    return W, H


def _run(W, H, bits, g, sym, desc_act, static, blocksize=128, damp=0.01):
    dev = device()
    res = gq.quantize_layer(W.to(dev), H.to(dev), bits, g, damp, sym, desc_act, static, blocksize, stats=True)
    torch.cuda.synchronize()
    Wn, Hn = W.double().numpy(), H.double().numpy()
    ref = O.gptq_quantize(Wn, Hn, bits, g, damp, sym, desc_act, static)  # eager sweep defines the result
    return res, ref, compare_quant(res, ref, Wn, Hn, bits, W.shape[1])


def test_tiny_config():
    cfg = synth.CONFIGS["tiny"]
    W = synth.weight_for(cfg, cfg.layers[0])
    X = synth.acts_for(cfg, 0).full()
    H = torch.from_numpy(O.hessian(X.double().numpy())).float()
    res, ref, m = _run(W, H, cfg.bits, cfg.group_size, cfg.sym, cfg.desc_act, cfg.static_groups, cfg.blocksize)
    assert_parity(m, "tiny")
    assert abs(res.stats["damped_loss"] - ref["damped_loss"]) <= 0.01 * ref["damped_loss"]


GRID = [(b, g, s, d, st) for b in (2, 3, 4, 8) for g in (32, 128, -1) for s in (True, False)
        for d, st in ((False, False), (True, False), (True, True))]


@pytest.mark.parametrize("bits,g,sym,desc_act,static", GRID)
def test_config_grid(bits, g, sym, desc_act, static):
    W, H = _problem(96, 512, 2048, 100 + bits * 7 + (g % 97))
    _, _, m = _run(W, H, bits, g, sym, desc_act, static)
    assert_parity(m, (bits, g, sym, desc_act, static))


@pytest.mark.parametrize("n_out,n_in,g,bits", [(1, 256, 32, 4), (7, 200, -1, 4), (130, 264, 8, 4),
                                              (33, 512, 256, 3), (64, 384, 384, 2), (5, 96, 96, 8),
                                              (40, 1160, 40, 4)])
def test_edge_shapes(n_out, n_in, g, bits):
    """n_out = 1 and not a multiple of 4 (scalar pack path), ragged panels, groups wider
    than a panel, a single group spanning all inputs, a group width not dividing 128."""
    W, H = _problem(n_out, n_in, 4 * n_in, n_out * 31 + n_in, w_dtype=torch.float32)
    _, _, m = _run(W, H, bits, g, True, False, False)
    assert_parity(m, (n_out, n_in, g, bits))


@pytest.mark.parametrize("blocksize", [1, 32, 128, 1000])
def test_blocksize_does_not_change_results(blocksize):
    W, H = _problem(64, 256, 1024, 9)
    dev = device()
    a = gq.quantize_layer(W.to(dev), H.to(dev), 4, 32, 0.01, True, True, False, blocksize)
    b = gq.quantize_layer(W.to(dev), H.to(dev), 4, 32, 0.01, True, True, False, 128)
    assert torch.equal(a.qweight, b.qweight) and torch.equal(a.scales, b.scales)


@pytest.mark.parametrize("w_dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_weight_dtypes(w_dtype):
    W, H = _problem(48, 256, 1024, 21, w_dtype=w_dtype)
    _, _, m = _run(W, H, 4, 64, False, False, False)
    assert_parity(m, str(w_dtype))


def test_factored_sweep_with_oracle_factor():
    """Sweep alone: GPU sweep given the oracle's U and permutation."""
    W, H = _problem(128, 512, 2048, 33)
    Hn = H.double().numpy()
    perm = O.act_order_perm(Hn)
    U = O.inverse_cholesky_upper(O.dampen(Hn[np.ix_(perm, perm)], 0.01))
    dev = device()
    res = gq.quantize_layer_factored(W.to(dev), torch.from_numpy(U).to(dev),
                                     torch.from_numpy(perm.astype(np.int32)).to(dev), 4, 64, True, False, 128)
    torch.cuda.synchronize()
    ref = O.gptq_quantize(W.double().numpy(), Hn, 4, 64, 0.01, True, True, False)
    m = compare_quant(res, ref, W.double().numpy(), Hn, 4, 512)
    assert_parity(m, "factored")


def test_factor_once_sweep_many_equals_quantize_layer():
    W1, H = _problem(64, 256, 1024, 44)
    W2 = synth.outlier_weight(80, 256, 45)
    dev = device()
    U, perm = gq.factor_hessian(H.to(dev), 0.01, True)
    for W in (W1, W2):
        a = gq.quantize_layer_factored(W.to(dev), U, perm, 4, 32, True, False, 128)
        b = gq.quantize_layer(W.to(dev), H.to(dev), 4, 32, 0.01, True, True, False, 128)
        assert torch.equal(a.qweight, b.qweight)
        assert torch.equal(a.g_idx, b.g_idx)


def test_invalid_permutation_is_rejected():
    dev = device()
    W, H = _problem(16, 64, 256, 3)
    U, _ = gq.factor_hessian(H.to(dev), 0.01, False)
    bad = torch.zeros(64, dtype=torch.int32, device=dev)
    with pytest.raises(gq.GPTQError) as e:
        gq.quantize_layer_factored(W.to(dev), U, bad, 4, 32)
    assert e.value.status == 1


def test_not_pd_through_quantize_layer():
    dev = device()
    W = torch.randn(16, 64, device=dev)
    with pytest.raises(gq.GPTQError) as e:
        gq.quantize_layer(W, torch.zeros(64, 64, device=dev), 4, 32)
    assert e.value.status == 3


def test_trim_workspace_keeps_library_usable():
    from post_weight_quantization_layer_b200 import _native
    dev = device()
    W, H = _problem(32, 128, 512, 8)
    a = gq.quantize_layer(W.to(dev), H.to(dev), 4, 32)
    assert _native.lib().gptq_trim_workspace() == 0
    b = gq.quantize_layer(W.to(dev), H.to(dev), 4, 32)
    assert torch.equal(a.qweight, b.qweight)


@pytest.mark.parametrize("n_out,n_in,g", [(20, 48, 3), (33, 120, 15), (17, 200, 25)])
def test_odd_group_sizes(n_out, n_in, g):
    """Odd group sizes make odd panel widths (63, 60, 50 columns) and odd panel starts."""
    W, H = _problem(n_out, n_in, 8 * n_in, n_in + g, w_dtype=torch.float32)
    _, _, m = _run(W, H, 4, g, False, False, False)
    assert_parity(m, (n_out, n_in, g))


@pytest.mark.parametrize("desc_act", [False, True])
def test_pipelined_linears_equal_factor_then_sweeps(desc_act):
    """quantize_linears (each Hessian's factor on its own stream, each linear's sweep started
    when its factor is done) gives exactly the factors of factor_hessians and the codes of one
    quantize_layer_factored per linear; one linear is also checked against the oracle."""
    dev = device()
    shapes = [(512, 2048, 61), (256, 1024, 62), (1024, 4096, 63)]
    Hs, Ws = [], []
    for n, T, seed in shapes:
        W, H = _problem(8, n, T, seed)
        Hs.append(H.to(dev))
    lin = [(synth.outlier_weight(96, 512, 70), 0), (synth.outlier_weight(40, 256, 71), 1),
           (synth.outlier_weight(64, 512, 72), 0), (synth.outlier_weight(200, 1024, 73), 2),
           (synth.outlier_weight(24, 1024, 74), 2)]
    lin = [(W.to(dev), h) for W, h in lin]
    factors, res = gq.quantize_linears(Hs, lin, 4, 32, 0.01, True, desc_act, desc_act, 128)
    torch.cuda.synchronize()
    ref_f = gq.factor_hessians(Hs, 0.01, desc_act)
    for (U, p), (U1, p1) in zip(factors, ref_f):
        assert torch.equal(p, p1)
        assert torch.equal(U, U1)
    for (W, h), r in zip(lin, res):
        U1, p1 = ref_f[h]
        b = gq.quantize_layer_factored(W, U1, p1, 4, 32, True, desc_act, 128)
        for x, y in zip((r.qweight, r.scales, r.zeros, r.g_idx), (b.qweight, b.scales, b.zeros, b.g_idx)):
            assert torch.equal(x, y)
    W, h = lin[3]
    Wn, Hn = W.double().cpu().numpy(), Hs[h].double().cpu().numpy()
    ref = O.gptq_quantize(Wn, Hn, 4, 32, 0.01, True, desc_act, desc_act)
    assert_parity(compare_quant(res[3], ref, Wn, Hn, 4, 1024), "pipelined")


def test_pipelined_linears_report_the_failing_linear():
    dev = device()
    _, good = _problem(8, 256, 1024, 81)
    good = good.to(dev)
    bad = -torch.eye(128, device=dev)
    lin = [(synth.outlier_weight(32, 256, 82).to(dev), 0), (torch.randn(16, 128, device=dev).half(), 1)]
    with pytest.raises(gq.GPTQError) as e:
        gq.quantize_linears([good, bad], lin, 4, 32, 0.01, True, True)
    assert e.value.status == 3 and "linear 1" in str(e.value)
    with pytest.raises(ValueError):
        gq.quantize_linears([good], [(lin[0][0], 1)], 4, 32)
    # the context stays usable and the good Hessian's linear matches the two-call route
    factors, res = gq.quantize_linears([good], lin[:1], 4, 32, 0.01, True, True)
    U1, p1 = gq.factor_hessian(good, 0.01, True)
    b = gq.quantize_layer_factored(lin[0][0], U1, p1, 4, 32, True, False, 128)
    assert torch.equal(res[0].qweight, b.qweight)


@pytest.mark.parametrize("cfgname", ["opt125m", "llama7b"])
def test_layer_driver_routes_agree(cfgname):
    """The layer driver's pipelined route (the largest Hessian accumulated first, its factor
    started while the others accumulate on a side stream, every sweep on its own stream)
    against the two-phase route on the very Hessians the pipelined run accumulated: the same
    codes, scales, zero points and g_idx, bit for bit."""
    from post_weight_quantization_layer_b200.layer import quantize_decoder_layer
    dev = device()
    cfg = synth.CONFIGS[cfgname]
    acts = {h: synth.acts_for(cfg, h, tokens=4096).full(device=dev) for h in range(len(cfg.hessian_n))}
    weights = {m.name: synth.weight_for(cfg, m, device=dev) for m in cfg.layers}
    Hbuf = {h: torch.empty(n, n, dtype=torch.float32, device=dev) for h, n in enumerate(cfg.hessian_n)}
    a, ta = quantize_decoder_layer(acts, weights, cfg.layers, cfg, hessians=Hbuf, timing=True, pipelined=True)
    torch.cuda.synchronize()
    given = {h: H.clone() for h, H in Hbuf.items()}
    b, tb = quantize_decoder_layer(None, weights, cfg.layers, cfg, hessians=given, timing=True,
                                   hessians_given=True, pipelined=False)
    torch.cuda.synchronize()
    for m in cfg.layers:
        ra, rb = a[m.name], b[m.name]
        for x, y in zip((ra.qweight, ra.scales, ra.zeros, ra.g_idx), (rb.qweight, rb.scales, rb.zeros, rb.g_idx)):
            assert torch.equal(x, y), m.name
    for h, X in acts.items():
        # every Hessian was accumulated (the largest on the caller's stream, the rest on the
        # side stream): its leading 64 x 64 block against the oracle
        ref = O.hessian(X[:, :64].double().cpu().numpy())
        got = Hbuf[h][:64, :64].double().cpu().numpy()
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max(), h
    assert ta.total_ms > 0 and tb.total_ms > 0 and tb.factor_ms > 0 and tb.sweep_ms > 0
