"""The allocation-free factor entry point (gptq_factor_hessian_noalloc).

Callers that cannot allocate device memory (a runtime with a fixed arena, a loop
that must not touch the allocator) use this variant; its scratch is a fixed
array inside the library.  It must give the same factor and order as
gptq_factor_hessian, bit for bit (both run the same deterministic kernels), on
repeated calls (the shared scratch keeps the previous call's contents); once
the library's code is loaded on the device, a call must not change the device's
free memory; and sizes above its capacity are rejected.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_layer_b200 import _native, synth

pytestmark = pytest.mark.gpu

U_RTOL = 1e-7  # the factor tolerance of the other GPU tests


def _fn():
    L = _native.lib()
    f = L.gptq_factor_hessian_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    return L, f


def _call(fn, H, damp, desc_act, U, perm):
    st = fn(ctypes.c_void_p(H.data_ptr()), H.shape[0], damp, desc_act, ctypes.c_void_p(U.data_ptr()),
            ctypes.c_void_p(perm.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st


def _hessian(n, T, seed):
    X = synth.StudentTActs(n, T, seed, dtype=torch.bfloat16).full()
    return torch.from_numpy(O.hessian(X.double().numpy())).float()


@pytest.mark.parametrize("n,desc_act", [(1024, 1), (520, 0)])
def test_matches_pooled_entry_point_on_two_calls(n, desc_act):
    assert torch.cuda.is_available()
    dev = torch.device("cuda:0")
    L, f = _fn()
    Hs = [_hessian(n, 2 * n, 11 + n), _hessian(n, 2 * n, 12 + n)]
    for H in Hs:  # two calls in a row, different inputs, same shared scratch
        Hd = H.to(dev)
        U_ref = torch.empty(n, n, dtype=torch.float64, device=dev)
        p_ref = torch.empty(n, dtype=torch.int32, device=dev)
        st = L.gptq_factor_hessian(ctypes.c_void_p(Hd.data_ptr()), n, ctypes.c_float(0.01), desc_act,
                                   ctypes.c_void_p(U_ref.data_ptr()), ctypes.c_void_p(p_ref.data_ptr()),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0
        U = torch.full((n, n), float("nan"), dtype=torch.float64, device=dev)
        perm = torch.full((n,), -1, dtype=torch.int32, device=dev)
        assert _call(f, Hd, 0.01, desc_act, U, perm) == 0
        assert torch.equal(perm, p_ref)
        a, b = U.cpu().numpy(), U_ref.cpu().numpy()
        err = np.abs(a - b).max(axis=1) / np.abs(b).max(axis=1)
        assert err.max() <= U_RTOL
        assert torch.equal(U, U_ref)  # same kernels, deterministic: identical bits
        assert np.all(np.tril(a, -1) == 0)


def test_a_call_allocates_no_device_memory():
    """After a first call (which may load the library's code, and with it the fixed array,
    onto the device), further calls leave the device's free memory unchanged."""
    dev = torch.device("cuda:0")
    L, f = _fn()
    n = 512
    Hd = _hessian(n, 2 * n, 77).to(dev)
    U = torch.empty(n, n, dtype=torch.float64, device=dev)
    perm = torch.empty(n, dtype=torch.int32, device=dev)
    assert _call(f, Hd, 0.01, 1, U, perm) == 0  # warm-up: module load
    free0, _ = torch.cuda.mem_get_info(dev)
    for desc_act in (1, 0):
        assert _call(f, Hd, 0.01, desc_act, U, perm) == 0
    free1, _ = torch.cuda.mem_get_info(dev)
    assert free1 == free0, (free0, free1)


def test_rejects_sizes_beyond_capacity():
    dev = torch.device("cuda:0")
    L, f = _fn()
    n = 1032
    H = torch.eye(n, device=dev)
    U = torch.empty(n, n, dtype=torch.float64, device=dev)
    perm = torch.empty(n, dtype=torch.int32, device=dev)
    assert _call(f, H, 0.01, 0, U, perm) == 2  # GPTQ_ERR_UNSUPPORTED
