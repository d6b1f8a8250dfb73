"""Helpers shared by the GPU parity tests (comparison metrics, device setup)."""

import numpy as np
import torch

import oracle as O

# Tolerances of the parity bar (codes, group parameters, layer loss, Hessian).
H_REL_FROB = 1e-5
CODE_MATCH = 0.995
PARAM_MATCH = 0.999
PARAM_RTOL = 1e-3
LOSS_RTOL = 0.01


def device():
    assert torch.cuda.is_available(), "GPU test without a CUDA device"
    return torch.device("cuda:0")


def rel_frob(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def gpu_outputs_np(res):
    return (res.qweight.cpu().numpy(), res.scales.cpu().numpy(), res.zeros.cpu().numpy(),
            res.g_idx.cpu().numpy())


def compare_quant(res, ref, W, H, bits, n_in):
    """Parity metrics of a GPU quantization against the oracle's result.

    Returns dict(code_match, param_match, loss_gpu, loss_ref, g_idx_equal)."""
    qw, sc, zr, gi = gpu_outputs_np(res)
    codes = O.unpack(qw, bits, n_in)
    code_match = float(np.mean(codes == ref["codes"]))
    s_ref = ref["scales"].astype(np.float64)
    s_ok = np.abs(sc.astype(np.float64) - s_ref) <= PARAM_RTOL * np.abs(s_ref)
    z_ok = zr == ref["zeros"]
    param_match = float(np.mean(s_ok & z_ok))
    What = O.dequantize(qw, sc, zr, gi, bits, n_in)
    l_gpu = O.layer_loss_h(W, What, H)
    l_ref = O.layer_loss_h(W, ref["What"], H)
    return dict(code_match=code_match, param_match=param_match, loss_gpu=l_gpu, loss_ref=l_ref,
                g_idx_equal=bool(np.array_equal(gi, ref["g_idx"])))


def assert_parity(m, what=""):
    assert m["code_match"] >= CODE_MATCH, (what, m)
    assert m["param_match"] >= PARAM_MATCH, (what, m)
    assert abs(m["loss_gpu"] - m["loss_ref"]) <= LOSS_RTOL * m["loss_ref"], (what, m)
    assert m["g_idx_equal"], (what, m)
