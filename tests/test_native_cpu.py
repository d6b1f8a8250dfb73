"""CPU-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments on the host before touching the GPU.

Only rejection paths are exercised here: a call whose arguments pass host
validation would enqueue GPU work.  Pointer arguments are fake but non-null
and 16-byte aligned, so only the argument under test decides the outcome.
"""

import ctypes
import math

import pytest

from post_weight_quantization_layer_b200 import _native
from post_weight_quantization_layer_b200.build import build
from tests.conftest import read_golden

INVALID, UNSUPPORTED = 1, 2
FAKE = ctypes.c_void_p(0x10000)
MISALIGNED = ctypes.c_void_p(0x10004)
FAKE2 = ctypes.c_void_p(0x20000)  # a second distinct (never dereferenced) pointer


@pytest.fixture(scope="module")
def L():
    build()
    return _native.lib()


def test_exports_every_declared_symbol(L):
    names = _native.declared_symbols()
    assert set(names) >= {"gptq_accumulate_hessian", "gptq_quantize_layer", "gptq_status_string"}
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    for st in range(7):
        assert L.gptq_status_string(st)
    assert L.gptq_status_string(99) == b"unknown status"
    assert L.gptq_version() >= 100


def _quant(L, bits=4, g=128, damp=0.01, bs=128, n_out=64, n_in=256, dtype=1, W=FAKE, H=FAKE, out=FAKE):
    return L.gptq_quantize_layer(W, dtype, n_out, n_in, H, bits, g, damp, 1, 0, 0, bs, out, out, out, out,
                                 None, None)


def test_validation_table_through_c_abi(L):
    for ln in read_golden("validation.txt"):
        bits, g, damp, bs, n_in, expect = ln.split()
        if expect != "reject":
            continue
        st = _quant(L, int(bits), int(g), float(damp), int(bs), 64, int(n_in))
        assert st == INVALID, ln


def test_other_rejections(L):
    assert _quant(L, W=None) == INVALID
    assert _quant(L, H=None) == INVALID
    assert _quant(L, out=None) == INVALID
    assert _quant(L, dtype=7) == INVALID
    assert _quant(L, n_out=0) == INVALID
    assert _quant(L, n_in=-8) == INVALID
    assert _quant(L, damp=math.nan) == INVALID
    assert _quant(L, n_in=260, g=-1) == UNSUPPORTED          # n_in % 8
    assert _quant(L, bits=3, n_in=264, g=-1) == UNSUPPORTED  # n_in*bits % 32
    assert _quant(L, W=MISALIGNED) == UNSUPPORTED
    assert _quant(L, n_in=70000, g=-1) == UNSUPPORTED


def test_hessian_rejections(L):
    acc = L.gptq_accumulate_hessian
    assert acc(None, 1, 16, 64, FAKE, None) == INVALID
    assert acc(FAKE, 1, 16, 64, None, None) == INVALID
    assert acc(FAKE, 1, -1, 64, FAKE, None) == INVALID
    assert acc(FAKE, 1, 16, 0, FAKE, None) == INVALID
    assert acc(FAKE, 0, 16, 64, FAKE, None) == UNSUPPORTED   # fp32 activations
    assert acc(FAKE, 5, 16, 64, FAKE, None) == INVALID
    assert acc(FAKE, 2, 16, 60, FAKE, None) == UNSUPPORTED   # n_in % 8
    assert acc(MISALIGNED, 2, 16, 64, FAKE, None) == UNSUPPORTED
    assert acc(FAKE, 2, 0, 64, FAKE, None) == 0              # zero tokens: no-op, no GPU touched


def test_factor_rejections(L):
    f = L.gptq_factor_hessian
    assert f(None, 64, 0.01, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, 64, 0.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, 64, 1.0, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, 64, math.nan, 0, FAKE, FAKE, None) == INVALID
    assert f(FAKE, 60, 0.01, 0, FAKE, FAKE, None) == UNSUPPORTED
    q = L.gptq_quantize_layer_factored
    assert q(FAKE, 1, 64, 256, None, FAKE, 4, 128, 1, 0, 128, FAKE, FAKE, FAKE, FAKE, None, None) == INVALID
    assert q(FAKE, 1, 64, 256, FAKE, FAKE, 6, 128, 1, 0, 128, FAKE, FAKE, FAKE, FAKE, None, None) == INVALID


def test_batched_factor_rejections(L):
    f = L.gptq_factor_hessians
    P = ctypes.c_void_p * 2
    ptrs = P(FAKE, FAKE)
    ns = (ctypes.c_int64 * 2)(64, 128)
    st = (ctypes.c_int * 2)()
    assert f(0, ptrs, ns, 0.01, 0, ptrs, ptrs, None, st) == INVALID
    assert f(-1, ptrs, ns, 0.01, 0, ptrs, ptrs, None, st) == INVALID
    assert f(2, None, ns, 0.01, 0, ptrs, ptrs, None, st) == INVALID
    assert f(2, ptrs, None, 0.01, 0, ptrs, ptrs, None, st) == INVALID
    assert f(2, ptrs, ns, 0.0, 0, ptrs, ptrs, None, st) == INVALID
    assert f(2, ptrs, ns, math.nan, 0, ptrs, ptrs, None, st) == INVALID
    assert f(2, P(FAKE, None), ns, 0.01, 0, ptrs, ptrs, None, st) == INVALID
    assert f(2, ptrs, (ctypes.c_int64 * 2)(64, 0), 0.01, 0, ptrs, ptrs, None, st) == INVALID
    assert f(2, ptrs, (ctypes.c_int64 * 2)(64, 60), 0.01, 0, ptrs, ptrs, None, st) == UNSUPPORTED
    assert f(2, P(FAKE, MISALIGNED), ns, 0.01, 0, ptrs, ptrs, None, st) == UNSUPPORTED


def test_python_binding_fails_loudly_without_cuda_tensors():
    import torch

    import post_weight_quantization_layer_b200 as gq
    with pytest.raises(ValueError):
        gq.quantize_layer(torch.zeros(4, 8), torch.zeros(8, 8))



def test_python_binding_rejects_mismatched_tensors():
    """Every wrapper checks dtype, shape and layout of its tensors (and of `out=`) before
    the native call, so a mismatched tensor can never reach a kernel as a raw pointer."""
    import torch

    import post_weight_quantization_layer_b200 as gq
    W = torch.zeros(4, 64)
    H = torch.zeros(64, 64)
    cases = [
        (lambda: gq.quantize_layer(W, H.half()), "H must have dtype"),
        (lambda: gq.quantize_layer(W, torch.zeros(64, 32)), "H must have shape"),
        (lambda: gq.quantize_layer(W.int(), H), "W must be float32"),
        (lambda: gq.quantize_layer(torch.zeros(64), H), "2-D"),
        (lambda: gq.quantize_layer(W.t(), torch.zeros(4, 4)), "contiguous"),
        (lambda: gq.quantize_layer(W, H, 4, 32, out=(1, 2, 3)), "out must be a tuple"),
        (lambda: gq.quantize_layer(W, H, 4, 32, out=(torch.zeros(4, 8, dtype=torch.int32),
                                                     torch.zeros(2, 4), torch.zeros(2, 4, dtype=torch.int32),
                                                     torch.zeros(64, dtype=torch.int32))), "out qweight"),
        (lambda: gq.quantize_layer(W, H, 4, 32, out=(torch.zeros(8, 4, dtype=torch.int32),
                                                     torch.zeros(1, 4), torch.zeros(2, 4, dtype=torch.int32),
                                                     torch.zeros(64, dtype=torch.int32))), "out scales"),
        (lambda: gq.quantize_layer(W, H, 4, 32, out=(torch.zeros(8, 4, dtype=torch.int32),
                                                     torch.zeros(2, 4), torch.zeros(2, 4),
                                                     torch.zeros(64, dtype=torch.int32))), "out zeros"),
        (lambda: gq.factor_hessian(torch.zeros(64, 32)), "H must have shape"),
        (lambda: gq.factor_hessian(H.double()), "H must have dtype"),
        (lambda: gq.factor_hessians([]), "at least one"),
        (lambda: gq.factor_hessians([H, H.half()]), r"H\[1\] must have dtype"),
        (lambda: gq.quantize_layer_factored(W, H, torch.zeros(64, dtype=torch.int32)), "U must have dtype"),
        (lambda: gq.quantize_layer_factored(W, H.double()[:32], torch.zeros(64, dtype=torch.int32)),
         "U must have shape"),
        (lambda: gq.quantize_layer_factored(W, H.double(), torch.zeros(64, dtype=torch.int64)), "perm must have dtype"),
        (lambda: gq.quantize_layer_factored(W, H.double(), torch.zeros(60, dtype=torch.int32)), "perm must have shape"),
        (lambda: gq.accumulate_hessian(torch.zeros(16, 64), H), "X must have dtype"),
        (lambda: gq.accumulate_hessian(torch.zeros(16, 64, dtype=torch.bfloat16), torch.zeros(32, 32)),
         "H must have shape"),
        (lambda: gq.quantize_layer(W, H), "CUDA tensors"),
    ]
    for fn, msg in cases:
        with pytest.raises(ValueError, match=msg):
            fn()


def test_checkpoint_and_forward_rejections(L):
    """Host-side rejections of the export, quantized-linear and layer-forward entry points
    (nothing reaches the GPU)."""
    ex = L.gptq_export_layer
    assert ex(None, FAKE, 4, 64, 4, FAKE, FAKE, None) == INVALID
    assert ex(FAKE, FAKE, 0, 64, 4, FAKE, FAKE, None) == INVALID
    assert ex(FAKE, FAKE, 4, 64, 5, FAKE, FAKE, None) == INVALID
    assert ex(FAKE, FAKE, 4, 36, 4, FAKE, FAKE, None) == UNSUPPORTED       # 36*4 % 32
    assert ex(MISALIGNED, FAKE, 4, 64, 4, FAKE, FAKE, None) == UNSUPPORTED
    dq = L.gptq_dequantize_weight
    assert dq(None, FAKE, FAKE, FAKE, 4, 512, 64, 4, 1, FAKE, None) == INVALID
    assert dq(FAKE, FAKE, FAKE, FAKE, 4, 512, 64, 5, 1, FAKE, None) == INVALID
    assert dq(FAKE, FAKE, FAKE, FAKE, 4, 512, 64, 3, 1, FAKE, None) == UNSUPPORTED   # 3-bit
    assert dq(FAKE, FAKE, FAKE, FAKE, 4, 500, 64, 4, 1, FAKE, None) == UNSUPPORTED   # n_in % 64
    assert dq(FAKE, FAKE, FAKE, FAKE, 4, 512, 72, 2, 1, FAKE, None) == UNSUPPORTED   # 72*2 % 32
    assert dq(FAKE, FAKE, FAKE, FAKE, 4, 512, 64, 4, 0, FAKE, None) == INVALID       # fp32 output
    ql = L.gptq_quantized_linear
    assert ql(FAKE, 2, 8, 512, FAKE, FAKE, FAKE, FAKE, None, 4, 64, 4, None, None) == INVALID
    assert ql(FAKE, 0, 8, 512, FAKE, FAKE, FAKE, FAKE, None, 4, 64, 4, FAKE, None) == INVALID   # fp32 X
    assert ql(FAKE, 2, -1, 512, FAKE, FAKE, FAKE, FAKE, None, 4, 64, 4, FAKE, None) == INVALID
    assert ql(FAKE, 2, 0, 512, FAKE, FAKE, FAKE, FAKE, None, 4, 64, 4, FAKE, None) == 0         # no rows: no-op
    assert ql(None, 2, 0, 512, FAKE, FAKE, FAKE, FAKE, None, 4, 64, 4, None, None) == 0         # ... even NULL X, Y
    assert ql(MISALIGNED, 2, 8, 512, FAKE, FAKE, FAKE, FAKE, None, 4, 64, 4, FAKE, None) == UNSUPPORTED
    assert ql(FAKE, 2, 8, 512, FAKE, FAKE, FAKE, FAKE, MISALIGNED, 4, 64, 4, FAKE, None) == UNSUPPORTED
    ro = L.gptq_reorder_act_order
    assert ro(None, FAKE, 4, 512, 64, 4, FAKE2, FAKE2, FAKE2, None) == INVALID
    assert ro(FAKE, FAKE, 4, 512, 64, 5, FAKE2, FAKE2, FAKE2, None) == INVALID
    assert ro(FAKE, FAKE, 4, 512, 64, 3, FAKE2, FAKE2, FAKE2, None) == UNSUPPORTED   # 3-bit
    assert ro(FAKE, FAKE, 4, 500, 64, 4, FAKE2, FAKE2, FAKE2, None) == UNSUPPORTED   # n_in % 64
    assert ro(FAKE, FAKE, 4, 512, 64, 4, FAKE, FAKE2, FAKE2, None) == INVALID        # in place
    assert ro(FAKE, FAKE, 40000, 65536, 64, 4, FAKE2, FAKE2, FAKE2, None) == UNSUPPORTED  # > 32768 groups
    assert L.gptq_rmsnorm(FAKE, 0, 4, 64, FAKE, 1e-6, FAKE, None) == INVALID
    assert L.gptq_rmsnorm(FAKE, 2, 4, 64, None, 1e-6, FAKE, None) == INVALID
    assert L.gptq_rope(FAKE, 2, 16, 4, 63, 8, 10000.0, None) == INVALID   # odd head_dim
    assert L.gptq_attention(FAKE, FAKE, FAKE, 2, 100, 4, 64, 32, FAKE, None) == INVALID  # ragged sequences
    assert L.gptq_attention(FAKE, FAKE, FAKE, 2, 64, 1, 256, 32, FAKE, None) == UNSUPPORTED  # head_dim > 128
    assert L.gptq_silu_mul(FAKE, None, 2, 8, FAKE, None) == INVALID
    assert L.gptq_add(FAKE, FAKE, 1, -1, FAKE, None) == INVALID
    assert L.gptq_test_wait_expiry(1, 0) == INVALID


def test_pipelined_linears_rejections(L):
    """gptq_quantize_linears rejects bad arguments before any device work."""
    f = L.gptq_quantize_linears
    P2 = ctypes.c_void_p * 2
    hp = P2(FAKE, FAKE)
    ns = (ctypes.c_int64 * 2)(256, 512)
    wp = P2(FAKE, FAKE)
    no = (ctypes.c_int64 * 2)(64, 64)
    hof = (ctypes.c_int * 2)(0, 1)
    st = (ctypes.c_int * 2)()

    def call(nh=2, H=hp, n_in=ns, damp=0.01, nl=2, W=wp, n_out=no, hidx=hof, bits=4, g=128, bs=128):
        return f(nh, H, n_in, damp, 1, hp, hp, nl, W, 1, n_out, hidx, bits, g, 1, 0, bs, wp, wp, wp, wp, None, None,
                 st)
    assert call(nh=0) == INVALID
    assert call(nl=0) == INVALID
    assert call(H=None) == INVALID
    assert call(damp=0.0) == INVALID
    assert call(damp=math.nan) == INVALID
    assert call(hidx=(ctypes.c_int * 2)(0, 2)) == INVALID                     # Hessian index out of range
    assert call(hidx=(ctypes.c_int * 2)(0, -1)) == INVALID
    assert call(n_in=(ctypes.c_int64 * 2)(256, 500)) == UNSUPPORTED           # n_in % 8
    assert call(bits=5) == INVALID                                            # a config rule per linear
    assert call(H=P2(FAKE, MISALIGNED)) == UNSUPPORTED
    assert call(W=P2(FAKE, None)) == INVALID


def test_pipelined_and_reorder_binding_rejections():
    import torch

    import post_weight_quantization_layer_b200 as gq
    H = torch.zeros(64, 64)
    W = torch.zeros(8, 64, dtype=torch.float16)
    ck = {"qweight": torch.zeros(8, 16, dtype=torch.int32), "qzeros": torch.zeros(1, 2, dtype=torch.int32),
          "scales": torch.zeros(1, 16, dtype=torch.float16), "g_idx": torch.zeros(64, dtype=torch.int32)}
    cases = [
        (lambda: gq.quantize_linears([], [(W, 0)]), "at least one"),
        (lambda: gq.quantize_linears([H], []), "at least one"),
        (lambda: gq.quantize_linears([H], [(W, 1)]), "out of range"),
        (lambda: gq.quantize_linears([H], [(torch.zeros(8, 32, dtype=torch.float16), 0)]), "does not match"),
        (lambda: gq.quantize_linears([H], [(W, 0), (W.float(), 0)]), "same weight dtype"),
        (lambda: gq.quantize_linears([H.half()], [(W, 0)]), r"H\[0\] must have dtype"),
        (lambda: gq.quantize_linears([H], [(W, 0)], ready=[None, None]), "one entry"),
        (lambda: gq.quantize_linears([H], [(W, 0)]), "CUDA tensors"),
        (lambda: gq.reorder_act_order(dict(ck, x_perm=torch.zeros(64, dtype=torch.int32))), "already reordered"),
        (lambda: gq.reorder_act_order(dict(ck, x_perm=torch.zeros(32, dtype=torch.int32))), "x_perm must have shape"),
        (lambda: gq.quantized_linear(torch.zeros(1, 64, dtype=torch.float16),
                                     dict(ck, x_perm=torch.zeros(64, dtype=torch.int64))), "x_perm must have dtype"),
        (lambda: gq.reorder_act_order(ck), "CUDA tensors"),
    ]
    for fn, msg in cases:
        with pytest.raises(ValueError, match=msg):
            fn()
