"""GPU parity of gptq_accumulate_hessian against the oracle (H = 2 X^T X)."""

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import synth
from tests.gpu_util import H_REL_FROB, device, rel_frob

pytestmark = pytest.mark.gpu


def _gpu_h(X, n, chunks=1):
    dev = device()
    H = torch.zeros(n, n, dtype=torch.float32, device=dev)
    Xd = X.to(dev)
    T = X.shape[0]
    step = (T + chunks - 1) // chunks
    for t0 in range(0, T, step):
        gq.accumulate_hessian(Xd[t0:t0 + step], H)
    torch.cuda.synchronize()
    assert gq.device_status() == 0
    return H.cpu().double().numpy()


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("T,n", [(777, 264), (64, 8), (130, 392), (1500, 520), (777, 4104), (5000, 1032)])
def test_integer_valued_x_is_bit_exact(dtype, T, n):
    """Entries in {-3..3} are exact in fp16/bf16 and every partial sum stays below
    2^24, so the fp32 result must equal the integer SYRK exactly (both triangles)."""
    g = torch.Generator().manual_seed(T * 7 + n)
    X = torch.randint(-3, 4, (T, n), generator=g).to(dtype)
    H = _gpu_h(X, n)
    ref = O.hessian(X.double().numpy())
    assert np.array_equal(H, ref)


def test_one_hot_rows():
    n, T = 136, 1000
    g = torch.Generator().manual_seed(5)
    idx = torch.randint(0, n, (T,), generator=g)
    X = torch.zeros(T, n, dtype=torch.float16)
    X[torch.arange(T), idx] = 1
    H = _gpu_h(X, n)
    assert np.array_equal(H, np.diag(2.0 * np.bincount(idx.numpy(), minlength=n)))


def test_tiny_config():
    cfg = synth.CONFIGS["tiny"]
    X = synth.acts_for(cfg, 0).full()
    H = _gpu_h(X, 256)
    assert rel_frob(H, O.hessian(X.double().numpy())) <= H_REL_FROB
    assert np.allclose(H, H.T, rtol=1e-6, atol=0)


@pytest.mark.parametrize("chunks", [1, 3, 7])
def test_streaming_chunks_accumulate(chunks):
    X = synth.HeavyChannelActs(384, 5000, 17, 0.02, 30.0, torch.bfloat16).full()
    H = _gpu_h(X, 384, chunks)
    assert rel_frob(H, O.hessian(X.double().numpy())) <= H_REL_FROB


def test_zero_tokens_is_noop():
    dev = device()
    H = torch.full((64, 64), 3.0, device=dev)
    gq.accumulate_hessian(torch.zeros(0, 64, dtype=torch.float16, device=dev), H)
    torch.cuda.synchronize()
    assert torch.all(H == 3.0)


def test_bounded_wait_expiry_reports_timeout_and_context_survives():
    """The expiry path of the kernel's bounded waits: with the test switch the producer
    issues no loads, the other warps' waits run out after a short limit, the launch ends
    with GPTQ_ERR_TIMEOUT recorded (H untouched), and the next normal call succeeds."""
    from post_weight_quantization_layer_b200 import _native
    L = _native.lib()
    dev = device()
    X = synth.HeavyChannelActs(256, 4096, 21, 0.02, 30.0, torch.bfloat16).full()
    H = torch.full((256, 256), 7.0, device=dev)
    assert gq.device_status(clear=True) == 0
    assert L.gptq_test_wait_expiry(1, 0) == 1  # a skipped load needs a short limit
    assert L.gptq_test_wait_expiry(1, 1 << 12) == 0
    try:
        gq.accumulate_hessian(X.to(dev), H)
        torch.cuda.synchronize()
        assert gq.device_status(clear=True) == gq.api.TIMEOUT
        assert torch.all(H == 7.0)
    finally:
        assert L.gptq_test_wait_expiry(0, 0) == 0
    H.zero_()
    gq.accumulate_hessian(X.to(dev), H)
    torch.cuda.synchronize()
    assert gq.device_status(clear=True) == 0
    assert rel_frob(H.cpu().double().numpy(), O.hessian(X.double().numpy())) <= H_REL_FROB
