"""GPU parity of the quantized-weight linear (gptq_dequantize_weight, gptq_quantized_linear)
against the oracle: Y = X round16(W_hat)^T with W_hat[o, c] = s16[g_idx[c], o] (q - z).

Inputs are synthetic checkpoint parts (random codes, zero points, fp16 scales, monotone or
act-order group indices) packed by the oracle; activations are the configs' laws.

Bars: the dequantized weight is bit-exact (scale * (code - zero) is exact in fp32 and is
rounded once, to nearest even, on both sides).  Y: with integer activations and
power-of-two scales every fp32 partial sum is exact, so Y must equal the oracle's exact
product rounded to the output type, bit for bit.  Otherwise the kernel's only errors are
the fp32 accumulation of exact products and the final rounding to the output type:
|Y - Y_ref| <= u_out |Y_ref| + 2^-16 S, with u_out the output type's unit roundoff (2^-8
bfloat16, 2^-11 float16) and S = |X| |round16(W_hat)|^T; the second term is about 2^8
times the typical fp32 accumulation error and far below the change that one wrong
weight makes (about S / n_in).
"""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import synth
from tests.gpu_util import device

pytestmark = pytest.mark.gpu

U_OUT = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}
NAME = {torch.bfloat16: "bfloat16", torch.float16: "float16"}


def _checkpoint(n_out, n_in, bits, g, seed, act_order, scale_range=(0.002, 0.02)):
    codes, zeros, scales, g_idx = synth.checkpoint_parts(n_out, n_in, bits, g, seed, act_order, scale_range)
    S16, qz = O.export_tensors(scales.float().numpy(), zeros.numpy(), bits)
    qw = O.pack(codes.numpy(), bits)
    dev = device()
    ck = {"qweight": torch.from_numpy(qw).to(dev), "qzeros": torch.from_numpy(qz).to(dev),
          "scales": torch.from_numpy(S16).to(dev), "g_idx": g_idx.to(dev)}
    W = O.dequantize_checkpoint(qw, qz, S16, g_idx.numpy(), bits)
    return ck, W


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("bits,g,act_order", [(4, 128, False), (4, 128, True), (2, 32, True), (8, -1, False),
                                              (4, 64, True)])
def test_dequantize_weight_bit_exact(dtype, bits, g, act_order):
    ck, W = _checkpoint(272, 512, bits, g, 10 + bits, act_order)
    Wg = gq.dequantize_weight(ck, bits, dtype)
    torch.cuda.synchronize()
    ref = O.round16(W, NAME[dtype])
    assert np.array_equal(Wg.double().cpu().numpy(), ref)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M", [1, 3, 4, 5, 130, 384])
def test_linear_integer_inputs_exact(dtype, M):
    """Integer activations in [-3, 3] and scales 2^-4: every partial sum is exact in fp32,
    so Y is the exact product rounded once to the output type (GEMV path for M <= 4, the
    tensor-core path above)."""
    n_out, n_in, bits = 520, 1024, 4
    ck, W = _checkpoint(n_out, n_in, bits, 128, 77, True, scale_range=(0.0625, 0.0625))
    gen = torch.Generator().manual_seed(M)
    X = torch.randint(-3, 4, (M, n_in), generator=gen).to(dtype)
    Y = gq.quantized_linear(X.to(device()), ck, bits)
    torch.cuda.synchronize()
    ref = O.round16(O.quantized_linear(X.double().numpy(), O.round16(W, NAME[dtype])), NAME[dtype])
    assert np.array_equal(Y.double().cpu().numpy(), ref)


def _tol_check(Y, X, W16, dtype):
    Xn = X.double().cpu().numpy()
    ref = O.quantized_linear(Xn, W16)
    S = np.abs(Xn) @ np.abs(W16).T
    err = np.abs(Y.double().cpu().numpy() - ref)
    bound = U_OUT[dtype] * np.abs(ref) + 2.0 ** -16 * S
    assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("M", [1, 4, 333, 2048])
@pytest.mark.parametrize("n_in,n_out", [(4096, 4096), (4096, 11008), (11008, 4096), (8192, 1024)])
def test_linear_llama_shapes(M, n_in, n_out):
    """bf16 heavy-tailed activations (the Llama-shaped configs' law), 4-bit, group 128,
    act-order groups."""
    dtype = torch.bfloat16
    ck, W = _checkpoint(n_out, n_in, 4, 128, n_in + n_out, True)
    X = synth.StudentTActs(n_in, M, 5 + M, dtype=dtype).full()
    Y = gq.quantized_linear(X.to(device()), ck, 4)
    torch.cuda.synchronize()
    _tol_check(Y, X, O.round16(W, "bfloat16"), dtype)


@pytest.mark.parametrize("bits,g", [(2, 32), (8, 128), (4, -1)])
@pytest.mark.parametrize("M", [2, 200])
def test_linear_other_widths_fp16(bits, g, M):
    dtype = torch.float16
    ck, W = _checkpoint(768, 3072, bits, g, bits * 31 + M, False)
    X = synth.HeavyChannelActs(3072, M, 9, 0.02, 30.0, dtype).full()
    Y = gq.quantized_linear(X.to(device()), ck, bits)
    torch.cuda.synchronize()
    _tol_check(Y, X, O.round16(W, "float16"), dtype)


def test_linear_zero_rows_and_determinism():
    dev = device()
    ck, _ = _checkpoint(256, 512, 4, 128, 3, True)
    Y0 = gq.quantized_linear(torch.zeros(0, 512, dtype=torch.float16, device=dev), ck, 4)
    assert Y0.shape == (0, 256)
    X = synth.StudentTActs(512, 700, 2, dtype=torch.bfloat16).full().to(dev)
    a = gq.quantized_linear(X, ck, 4)
    b = gq.quantized_linear(X, ck, 4)
    x1 = X[:3].contiguous()
    c = gq.quantized_linear(x1, ck, 4)
    d = gq.quantized_linear(x1, ck, 4)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(c, d)
    assert gq.device_status() == 0


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("bits,g", [(4, 128), (2, 32), (8, 64)])
@pytest.mark.parametrize("M", [1, 3, 130])
def test_reordered_act_order_checkpoint(dtype, bits, g, M):
    """gptq_reorder_act_order: the inputs sorted stably by (g_idx, index), the codes and g_idx
    carried along (index work: exact); the dequantized weight is the original's columns in that
    order (bit-exact); the linear on it is the same product (same bound) on both paths."""
    n_out, n_in = 272, 1024
    ck, W = _checkpoint(n_out, n_in, bits, g, 40 + bits + M, True)
    ck2 = gq.reorder_act_order(ck, bits)
    torch.cuda.synchronize()
    gi = ck["g_idx"].cpu().numpy()
    xp = ck2["x_perm"].cpu().numpy()
    assert np.array_equal(xp, np.lexsort((np.arange(n_in), gi)))
    assert np.array_equal(ck2["g_idx"].cpu().numpy(), gi[xp])
    assert np.all(np.diff(ck2["g_idx"].cpu().numpy()) >= 0)
    W16 = O.round16(W, NAME[dtype])
    Wd = gq.dequantize_weight(ck2, bits, dtype)
    torch.cuda.synchronize()
    assert np.array_equal(Wd.double().cpu().numpy(), W16[:, xp])
    X = synth.StudentTActs(n_in, M, 70 + M, dtype=dtype).full()
    Y = gq.quantized_linear(X.to(device()), ck2, bits)
    torch.cuda.synchronize()
    _tol_check(Y, X, W16, dtype)


def test_reordered_checkpoint_llama_decode():
    """A Llama-shaped act-order checkpoint (4096 -> 11008): the reordered decode agrees with the
    original checkpoint's decode within the fp32 accumulation bound."""
    dtype = torch.bfloat16
    ck, W = _checkpoint(11008, 4096, 4, 128, 91, True)
    ck2 = gq.reorder_act_order(ck, 4)
    X = synth.StudentTActs(4096, 1, 92, dtype=dtype).full()
    Y = gq.quantized_linear(X.to(device()), ck2, 4)
    torch.cuda.synchronize()
    _tol_check(Y, X, O.round16(W, "bfloat16"), dtype)
    with pytest.raises(ValueError):
        gq.reorder_act_order(ck2, 4)
