"""Parity at the Llama-2-70B decoder-layer sizes (q/o 8192x8192, k/v 1024x8192, gate/up
28672x8192, down 8192x28672; Hessians of order 8192 and 28672; 524,288 bf16 calibration
tokens streamed in 8,192-token chunks).

Each check is one the float64 oracle computes exactly in seconds:

* Hessians over all 524,288 tokens (n = 8192 and n = 28672): sampled 256 x 256 blocks,
  diagonal blocks among them, against the oracle's blocks of the same chunks (each block
  needs only its 512 channels of X).
* Factor and sweep of q/k/v, o and gate/up: the oracle builds each Hessian from 32,768
  tokens (four times the order, so H is full rank and its spectrum is set by the
  heavy-tailed channels, not by the damping), rounded to fp32 for both sides; the GPU
  factors all three in one batched call (as the layer driver does) and sweeps every
  linear; the oracle's factors are compared in full and its sweep on sampled rows.
* down (8192 x 28672): the order-28672 factor is beyond the oracle in a test, so the
  GPU's factor of the full-token Hessian is checked through an identity that holds at any
  size, U^T U H_d x = x, and the sweep through the identities that define it, on sampled
  rows: with err = (W - W_hat) U^-1 (the normalised errors, W - W_hat = err U), every
  group's scale and zero must be the quantizer's parameters of that group's current
  weights when the sweep reaches it, W[:, group] - err[:, :j0] U[:j0, group], and every
  code must be the quantizer's code of the current value W_hat_j + err_j U_jj.
"""

import numpy as np
import pytest
import torch
import oracle as O
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import synth
from tests.gpu_util import CODE_MATCH, H_REL_FROB, LOSS_RTOL, PARAM_MATCH, PARAM_RTOL, device
from tests.sweep_identities import sweep_decisions

pytestmark = pytest.mark.gpu

CFG = synth.CONFIGS["llama70b"]
BS = 256
SWEEP_TOKENS = 32768
DECISION_MATCH = 0.9999  # per-decision identities (no cascade): at most 1 in 10^4
_keep = {}


def _blocks(n, seed):
    rng = np.random.default_rng(seed)
    nb = n // BS
    diag = [(int(i), int(i)) for i in rng.choice(nb, 3, replace=False)]
    off = [(int(i), int(j)) for i, j in rng.integers(0, nb, size=(5, 2))]
    return diag + off


@pytest.mark.parametrize("h_index", [0, 3])
def test_hessian_full_tokens_sampled_blocks(h_index):
    """H += 2 X^T X over all 64 chunks of 8,192 tokens; 8 blocks of 256 x 256 against the
    oracle's float64 blocks (relative Frobenius <= 1e-5), both triangles."""
    dev = device()
    acts = synth.acts_for(CFG, h_index)
    assert acts.tokens == 128 * 4096
    n = acts.n
    blocks = _blocks(n, 70000 + h_index)
    cols = sorted({b * BS + c for ij in blocks for b in ij for c in range(BS)})
    pos = {c: k for k, c in enumerate(cols)}
    idx = {b: [pos[b * BS + c] for c in range(BS)] for ij in blocks for b in ij}
    cols_t = torch.tensor(cols, device=dev)
    H = torch.zeros(n, n, dtype=torch.float32, device=dev)
    ref = {blk: np.zeros((BS, BS)) for blk in blocks}
    for i in range(acts.n_chunks):
        X = acts.get_chunk(i, device=dev)
        gq.accumulate_hessian(X, H)
        Xs = X.index_select(1, cols_t).cpu().double().numpy()
        del X
        for bi, bj in blocks:
            ref[(bi, bj)] += O.hessian(np.concatenate([Xs[:, idx[bi]], Xs[:, idx[bj]]], 1))[:BS, BS:]
    torch.cuda.synchronize()
    assert gq.device_status() == 0
    for bi, bj in blocks:
        got = H[bi * BS:(bi + 1) * BS, bj * BS:(bj + 1) * BS].double().cpu().numpy()
        r = ref[(bi, bj)]
        rel = np.linalg.norm(got - r) / np.linalg.norm(r)
        assert rel <= H_REL_FROB, (bi, bj, rel)
        got_t = H[bj * BS:(bj + 1) * BS, bi * BS:(bi + 1) * BS].double().cpu().numpy()
        assert np.abs(got_t - got.T).max() <= 1e-6 * np.abs(got).max(), (bi, bj)
    if h_index == 3:
        _keep["H28672"] = H  # the down-projection test factors this full-token Hessian
    else:
        del H


def _full_token_h28672():
    """The GPU's full-token Hessian of the down-projection input (kept from the sampled-block
    test above when it ran first in this session, else accumulated here)."""
    if "H28672" in _keep:
        return _keep.pop("H28672")
    dev = device()
    acts = synth.acts_for(CFG, 3)
    H = torch.zeros(acts.n, acts.n, dtype=torch.float32, device=dev)
    for i in range(acts.n_chunks):
        gq.accumulate_hessian(acts.get_chunk(i, device=dev), H)
    torch.cuda.synchronize()
    assert gq.device_status() == 0
    return H


_sweep = {}


def _sweep_case():
    """Oracle Hessians (32,768 tokens) of the attention input, the o_proj input and the MLP
    input; the GPU's batched factor and the oracle's factor of each."""
    if _sweep:
        return _sweep
    dev = device()
    H64 = {}
    for h in (0, 1, 2):
        X = synth.acts_for(CFG, h, tokens=SWEEP_TOKENS).full().double().numpy()
        H64[h] = O.hessian(X).astype(np.float32).astype(np.float64)
        del X
    Hdev = {h: torch.from_numpy(H.astype(np.float32)).to(dev) for h, H in H64.items()}
    outs = gq.factor_hessians([Hdev[h] for h in (0, 1, 2)], CFG.damp_percent, CFG.desc_act)
    torch.cuda.synchronize()
    _sweep.update(H64=H64, gpu={h: o for h, o in zip((0, 1, 2), outs)},
                  ref={h: O.inverse_cholesky_upper(O.dampen(H64[h], CFG.damp_percent)) for h in (0, 1, 2)})
    return _sweep


@pytest.mark.parametrize("h", [0, 1, 2])
def test_factor_8192_matches_oracle(h):
    c = _sweep_case()
    U, perm = c["gpu"][h]
    assert np.array_equal(perm.cpu().numpy(), np.arange(8192))
    Ug, Ur = U.cpu().numpy(), c["ref"][h]
    assert np.all(np.tril(Ug, -1) == 0) and np.all(np.diag(Ug) > 0)
    err = np.abs(Ug - Ur).max(axis=1) / np.abs(Ur).max(axis=1)
    assert err.max() <= 1e-7, err.max()


@pytest.mark.parametrize("name,rows", [("q", 16), ("k", 16), ("v", 16), ("o", 16), ("gate", 12), ("up", 12)])
def test_sweep_8192_sampled_rows(name, rows):
    """4-bit, group 128, sym, no act order (the 70B setting): sampled rows against the
    oracle's sweep with its own factor of the same fp32 Hessian."""
    c = _sweep_case()
    layer = next(m for m in CFG.layers if m.name == name)
    U, perm = c["gpu"][layer.h_index]
    W = synth.weight_for(CFG, layer)
    dev = device()
    res = gq.quantize_layer_factored(W.to(dev), U, perm, CFG.bits, CFG.group_size, CFG.sym, CFG.static_groups,
                                     CFG.blocksize)
    torch.cuda.synchronize()
    sel = np.sort(np.random.default_rng(len(name) * 977 + layer.n_out).choice(layer.n_out, rows, replace=False))
    n_in = layer.n_in
    Ws = W.double().numpy()[sel]
    r = O.gptq_sweep(Ws, c["ref"][layer.h_index], CFG.bits, CFG.sym, CFG.group_size, np.arange(n_in), False, Ws,
                     CFG.blocksize)
    qw = res.qweight.cpu().numpy()[:, sel]
    codes = O.unpack(qw, CFG.bits, n_in)
    assert np.mean(codes == r["codes"]) >= CODE_MATCH
    sc = res.scales.cpu().numpy()[:, sel]
    zr = res.zeros.cpu().numpy()[:, sel]
    s_ref = r["scales"].astype(np.float64)
    assert np.mean((np.abs(sc - s_ref) <= PARAM_RTOL * np.abs(s_ref)) & (zr == r["zeros"])) >= PARAM_MATCH
    What = O.dequantize(qw, sc, zr, res.g_idx.cpu().numpy(), CFG.bits, n_in)
    Hd = c["H64"][layer.h_index]
    l_gpu = O.layer_loss_h(Ws, What, Hd)
    l_ref = O.layer_loss_h(Ws, r["xhat"], Hd)
    assert abs(l_gpu - l_ref) <= LOSS_RTOL * l_ref
    assert np.array_equal(res.g_idx.cpu().numpy(), np.arange(n_in) // CFG.group_size)


def test_down_proj_28672_factor_identity_and_sweep_identities():
    """down (8192 x 28672) on the full-token Hessian of its input."""
    dev = device()
    H = _full_token_h28672()
    n = H.shape[0]
    U, perm = gq.factor_hessian(H, CFG.damp_percent, False)
    torch.cuda.synchronize()
    assert np.array_equal(perm.cpu().numpy(), np.arange(n))
    # factor: U^T U H_d x = x, on the host in float64, U read in slabs of rows
    Hd = O.dampen(H.double().cpu().numpy(), CFG.damp_percent)
    del H
    x = np.random.default_rng(5).standard_normal((n, 3))
    t = Hd @ x
    del Hd
    Uh = np.empty((n, n))
    z = np.zeros_like(x)
    slab = 2048
    for r0 in range(0, n, slab):
        Us = U[r0:r0 + slab].cpu().numpy()
        Uh[r0:r0 + Us.shape[0]] = Us
        z += Us.T @ (Us @ t)
        rr = np.arange(Us.shape[0])
        assert np.all(Us[rr, r0 + rr] > 0)
        assert not np.any(np.tril(Us[:, r0:r0 + Us.shape[0]], -1))
        assert not np.any(Us[:, :r0])
    rel = np.linalg.norm(z - x, axis=0) / np.linalg.norm(x, axis=0)
    assert rel.max() < 1e-7, rel

    layer = next(m for m in CFG.layers if m.name == "down")
    W = synth.weight_for(CFG, layer)
    res = gq.quantize_layer_factored(W.to(dev), U, perm, CFG.bits, CFG.group_size, CFG.sym, CFG.static_groups,
                                     CFG.blocksize)
    torch.cuda.synchronize()
    del U
    g = CFG.group_size
    sel = np.sort(np.random.default_rng(28672).choice(layer.n_out, 8, replace=False))
    Ws = W.double().numpy()[sel]
    qw = res.qweight.cpu().numpy()[:, sel]
    sc = res.scales.cpu().numpy()[:, sel]
    zr = res.zeros.cpu().numpy()[:, sel]
    gi = res.g_idx.cpu().numpy()
    assert np.array_equal(gi, np.arange(n) // g)
    codes = O.unpack(qw, CFG.bits, n)
    What = O.dequantize(qw, sc, zr, gi, CFG.bits, n)
    p_ok, c_ok = sweep_decisions(Ws, What, codes, sc, zr, Uh, CFG.bits, CFG.sym, g)
    # each decision is checked against the outputs' own history (no cascade), so only a
    # value within fp64 recomputation error of a rounding boundary may disagree
    assert p_ok >= PARAM_MATCH, p_ok
    assert c_ok >= DECISION_MATCH, c_ok
