"""GPU parity of gptq_factor_hessian: damping, act-order permutation and the
upper Cholesky factor of the inverse, against the oracle's literal route."""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import synth
from tests.gpu_util import device

pytestmark = pytest.mark.gpu


def _h(n, T, seed, dtype=torch.float16):
    X = synth.HeavyChannelActs(n, T, seed, 0.02, 30.0, dtype).full()
    return torch.from_numpy(O.hessian(X.double().numpy())).float()


@pytest.mark.parametrize("n,T", [(256, 512), (264, 2000), (1032, 4096), (2056, 4112), (3000, 6000)])
@pytest.mark.parametrize("desc_act", [False, True])
def test_factor_matches_oracle(n, T, desc_act):
    """Orders above 1792 take the int8 route (seven-slice products) for the nodes whose right
    part is at least 1024 wide; 2056 and 3000 leave ragged tiles in every product."""
    H = _h(n, T, n + T)
    U, perm = gq.factor_hessian(H.to(device()), 0.01, desc_act)
    torch.cuda.synchronize()
    Hd64 = H.double().numpy()
    p_ref = O.act_order_perm(Hd64) if desc_act else np.arange(n)
    assert np.array_equal(perm.cpu().numpy(), p_ref)
    Hd = O.dampen(Hd64[np.ix_(p_ref, p_ref)], 0.01)
    U_ref = O.inverse_cholesky_upper(Hd)
    Ug = U.cpu().double().numpy()
    assert np.all(np.tril(Ug, -1) == 0)
    assert np.all(np.diag(Ug) > 0)
    # row-relative error of the compensation coefficients: the GPU factor works in fp64
    # from the same fp32 Hessian, so only fp64 rounding (times the condition number) remains
    err = np.abs(Ug - U_ref).max(axis=1) / np.abs(U_ref).max(axis=1)
    assert err.max() < 1e-7, err.max()
    R = Ug.T @ Ug @ Hd - np.eye(n)
    assert np.abs(R).max() < 1e-7


def test_not_positive_definite_is_reported():
    dev = device()
    with pytest.raises(gq.GPTQError) as e:
        gq.factor_hessian(torch.zeros(64, 64, device=dev), 0.01)
    assert e.value.status == 3
    H = -torch.eye(128, device=dev)
    with pytest.raises(gq.GPTQError) as e:
        gq.factor_hessian(H, 0.01)
    assert e.value.status == 3
    # the context stays usable after the error
    U, _ = gq.factor_hessian(torch.eye(64, device=dev) * 2, 0.01)
    torch.cuda.synchronize()
    assert torch.allclose(torch.diag(U).cpu(), torch.full((64,), (1 / 2.02) ** 0.5, dtype=torch.float64),
                          rtol=1e-12)


def test_act_order_ties_are_stable():
    dev = device()
    d = torch.tensor([3.0, 5.0, 3.0, 7.0, 5.0, 1.0, 7.0, 2.0])
    H = torch.diag(d)
    _, perm = gq.factor_hessian(H.to(dev), 0.01, True)
    assert perm.cpu().tolist() == sorted(range(8), key=lambda i: (-float(d[i]), i))


@pytest.mark.parametrize("desc_act", [False, True])
def test_batched_factor_is_bit_identical_to_single_calls(desc_act):
    """Concurrent factorisation of several Hessians gives exactly the single-call results."""
    dev = device()
    Hs = [_h(n, T, 7 * n + T).to(dev) for n, T in [(1032, 4096), (256, 512), (520, 1500), (264, 2000)]]
    outs = gq.factor_hessians(Hs, 0.01, desc_act)
    torch.cuda.synchronize()
    for H, (U, perm) in zip(Hs, outs):
        U1, p1 = gq.factor_hessian(H, 0.01, desc_act)
        torch.cuda.synchronize()
        assert torch.equal(perm, p1)
        assert torch.equal(U, U1)


def test_batched_factor_reports_the_failing_item():
    dev = device()
    good = _h(256, 512, 11).to(dev)
    bad = -torch.eye(128, device=dev)
    with pytest.raises(gq.GPTQError) as e:
        gq.factor_hessians([good, bad], 0.01, True)
    assert e.value.status == 3 and "item 1" in str(e.value)
    # after a failing batch the context stays usable and batched results still match
    outs = gq.factor_hessians([good, good * 2], 0.01, True)
    torch.cuda.synchronize()
    U1, _ = gq.factor_hessian(good, 0.01, True)
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], U1)
