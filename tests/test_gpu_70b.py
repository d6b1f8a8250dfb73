"""Parity at the Llama-2-70B decoder-layer sizes (q/o 8192x8192, k/v 1024x8192, gate/up
28672x8192, down 8192x28672; Hessians of order 8192 and 28672).

The float64 oracle cannot afford the n = 28672 problems whole, so each check is one the
oracle computes exactly at a cost of seconds:

* the n = 28672 Hessian, streamed in 8,192-token chunks, on sampled 256 x 256 blocks
  (each block needs only its 512 channels of X);
* the n = 8192 Hessian's factor in full, and sampled output rows of the q, k and gate
  sweeps against the oracle's own factor of the same (oracle-built) Hessian;
* the n = 28672 factor through an identity that holds at any size: U^T U H_d x = x for
  random x, with H built by the oracle from a short token sample and H_d x, U x and
  U^T y evaluated on the host in float64.
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import synth
from tests.gpu_util import CODE_MATCH, LOSS_RTOL, PARAM_MATCH, PARAM_RTOL, device

pytestmark = pytest.mark.gpu

CFG = synth.CONFIGS["llama70b"]


def test_hessian_28672_streamed_sampled_blocks():
    """H += 2 X^T X over 8 chunks of 8,192 tokens (n = 28672); 8 blocks of 256 x 256
    compared with the oracle's float64 blocks (relative Frobenius <= 1e-5)."""
    dev = device()
    acts = synth.acts_for(CFG, 3, tokens=8 * 8192)
    n = acts.n
    rng = np.random.default_rng(28672)
    blocks = [(int(i), int(j)) for i, j in rng.integers(0, n // 256, size=(8, 2))]
    cols = sorted({b * 256 + c for ij in blocks for b in ij for c in range(256)})
    pos = {c: k for k, c in enumerate(cols)}
    cols_t = torch.tensor(cols, device=dev)
    H = torch.zeros(n, n, dtype=torch.float32, device=dev)
    xs = []
    for i in range(acts.n_chunks):
        X = acts.get_chunk(i, device=dev)
        gq.accumulate_hessian(X, H)
        xs.append(X.index_select(1, cols_t).cpu())
        del X
    torch.cuda.synchronize()
    Xs = torch.cat(xs, 0).double().numpy()
    for bi, bj in blocks:
        I = [pos[bi * 256 + c] for c in range(256)]
        J = [pos[bj * 256 + c] for c in range(256)]
        ref = O.hessian(np.concatenate([Xs[:, I], Xs[:, J]], 1))[:256, 256:]  # H[I, J]
        got = H[bi * 256:(bi + 1) * 256, bj * 256:(bj + 1) * 256].double().cpu().numpy()
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel <= 1e-5, (bi, bj, rel)
        # both triangles are written (the same sums, added by atomics in either order)
        got_t = H[bj * 256:(bj + 1) * 256, bi * 256:(bi + 1) * 256].double().cpu().numpy()
        assert np.abs(got_t - got.T).max() <= 1e-6 * np.abs(got).max(), (bi, bj)


_h8192 = {}


def _oracle_h8192():
    if not _h8192:
        X = synth.acts_for(CFG, 0, tokens=8192).full().double().numpy()
        H = O.hessian(X).astype(np.float32)
        U = O.inverse_cholesky_upper(O.dampen(H.astype(np.float64), CFG.damp_percent))
        _h8192.update(H=H, U=U)
    return _h8192["H"], _h8192["U"]


def test_factor_8192_matches_oracle():
    H, U_ref = _oracle_h8192()
    U, perm = gq.factor_hessian(torch.from_numpy(H).to(device()), CFG.damp_percent, False)
    torch.cuda.synchronize()
    assert np.array_equal(perm.cpu().numpy(), np.arange(8192))
    Ug = U.cpu().numpy()
    assert np.all(np.tril(Ug, -1) == 0) and np.all(np.diag(Ug) > 0)
    err = np.abs(Ug - U_ref).max(axis=1) / np.abs(U_ref).max(axis=1)
    assert err.max() < 1e-7, err.max()


@pytest.mark.parametrize("name,rows", [("q", 12), ("k", 12), ("gate", 12)])
def test_sweep_8192_sampled_rows(name, rows):
    """q (8192x8192), k (1024x8192) and gate (28672x8192): 4-bit, group 128, sym,
    no act order (the 70B setting), sampled rows against the oracle's sweep with its
    own factor."""
    H, U = _oracle_h8192()
    layer = next(m for m in CFG.layers if m.name == name)
    W = synth.weight_for(CFG, layer)
    dev = device()
    res = gq.quantize_layer(W.to(dev), torch.from_numpy(H).to(dev), CFG.bits, CFG.group_size, CFG.damp_percent,
                            CFG.sym, False, False, CFG.blocksize)
    torch.cuda.synchronize()
    sel = np.random.default_rng(len(name) * 977 + layer.n_out).choice(layer.n_out, rows, replace=False)
    n_in = layer.n_in
    Ws = W.double().numpy()[sel]
    r = O.gptq_sweep(Ws, U, CFG.bits, CFG.sym, CFG.group_size, np.arange(n_in), False, Ws, 128)
    codes = O.unpack(res.qweight.cpu().numpy()[:, sel], CFG.bits, n_in)
    assert np.mean(codes == r["codes"]) >= CODE_MATCH
    sc = res.scales.cpu().numpy()[:, sel]
    zr = res.zeros.cpu().numpy()[:, sel]
    s_ref = r["scales"].astype(np.float64)
    assert np.mean((np.abs(sc - s_ref) <= PARAM_RTOL * np.abs(s_ref)) & (zr == r["zeros"])) >= PARAM_MATCH
    What = O.dequantize(res.qweight.cpu().numpy()[:, sel], sc, zr, res.g_idx.cpu().numpy(), CFG.bits, n_in)
    Hd = H.astype(np.float64)
    l_gpu = O.layer_loss_h(Ws, What, Hd)
    l_ref = O.layer_loss_h(Ws, r["xhat"], Hd)
    assert abs(l_gpu - l_ref) <= LOSS_RTOL * l_ref


def test_factor_28672_inverse_identity():
    """n = 28672 (the down-projection Hessian's order): U^T U H_d x = x for random x."""
    X = synth.acts_for(CFG, 3, tokens=1024).full().double().numpy()
    H = O.hessian(X).astype(np.float32)
    del X
    n = H.shape[0]
    dev = device()
    U, perm = gq.factor_hessian(torch.from_numpy(H).to(dev), CFG.damp_percent, False)
    torch.cuda.synchronize()
    assert np.array_equal(perm.cpu().numpy(), np.arange(n))
    Hd = O.dampen(H.astype(np.float64), CFG.damp_percent)
    del H
    x = np.random.default_rng(5).standard_normal((n, 3))
    t = Hd @ x
    del Hd
    z = np.zeros_like(x)
    slab = 2048
    for r0 in range(0, n, slab):
        Us = U[r0:r0 + slab].cpu().numpy()
        y = Us @ t          # rows r0.. of U t
        z += Us.T @ y       # their contribution to U^T (U t)
        # strictly lower part of these rows is exactly zero, diagonal positive
        rr = np.arange(Us.shape[0])
        assert np.all(Us[rr, r0 + rr] > 0)
        assert not np.any(np.tril(Us[:, r0:r0 + Us.shape[0]], -1))
        assert not np.any(Us[:, :r0])
    # same bound as the factor tests' U^T U H_d - I (fp64 route; this Hessian's heavy
    # channels give cond(H_d) ~ 1e4-1e5, and the residual measured 2.2e-8)
    rel = np.linalg.norm(z - x, axis=0) / np.linalg.norm(x, axis=0)
    assert rel.max() < 1e-7, rel
