"""GPU side of the checkpoint export (AutoGPTQ examples guide §1.4; OLMo quick-start §四
step 4): gptq_export_layer against the oracle's checkpoint form, bit for bit, and a
save_quantized / load_quantized round trip of a quantized decoder layer."""

import os

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_layer_b200 as gq
from post_weight_quantization_layer_b200 import export as E
from post_weight_quantization_layer_b200 import synth
from tests.gpu_util import device

pytestmark = pytest.mark.gpu


def _quantized(n_out, n_in, bits, g, seed):
    dev = device()
    W = synth.outlier_weight(n_out, n_in, seed)
    X = synth.StudentTActs(n_in, 2 * n_in, seed + 1, dtype=torch.bfloat16).full()
    H = torch.from_numpy(O.hessian(X.double().numpy())).float()
    res = gq.quantize_layer(W.to(dev), H.to(dev), bits, g, 0.01, bits != 3, False, False, 128)
    torch.cuda.synchronize()
    return res


@pytest.mark.parametrize("bits,g,n_out", [(4, 128, 96), (3, 64, 64), (2, 32, 160), (8, -1, 40)])
def test_export_layer_matches_oracle(bits, g, n_out):
    res = _quantized(n_out, 512, bits, g, 40 + bits)
    t = E.export_layer(res, bits)
    torch.cuda.synchronize()
    S, qz = O.export_tensors(res.scales.cpu().numpy(), res.zeros.cpu().numpy(), bits)
    assert np.array_equal(t["scales"].cpu().numpy().view(np.uint16), S.view(np.uint16))
    assert np.array_equal(t["qzeros"].cpu().numpy(), qz)
    assert t["qweight"] is res.qweight and t["g_idx"] is res.g_idx


def test_export_layer_half_rounding_edges():
    """Scales at fp16 rounding ties, subnormal and overflow range: conversion equals the
    oracle's IEEE round to nearest even bit for bit."""
    dev = device()
    vals = np.array([1.00048828125, 1.00146484375, 6.1e-5, 3.0e-8, 1.0e-9, 65504.0, 65520.0, 7e4, 2.0 ** -24,
                     2.0 ** -25, 1.5 * 2.0 ** -24, 0.1], dtype=np.float32)
    n_out = 32
    S = np.resize(vals, (2, n_out)).astype(np.float32)
    Z = np.resize(np.arange(16), (2, n_out)).astype(np.int32)
    res = gq.QuantResult(None, torch.from_numpy(S).to(dev), torch.from_numpy(Z).to(dev), None)
    t = E.export_layer(res, 4)
    torch.cuda.synchronize()
    S16, qz = O.export_tensors(S, Z, 4)
    assert np.array_equal(t["scales"].cpu().numpy().view(np.uint16), S16.view(np.uint16))
    assert np.array_equal(t["qzeros"].cpu().numpy(), qz)


@pytest.mark.parametrize("use_safetensors", [True, False])
def test_save_and_load_decoder_layer(tmp_path, use_safetensors):
    cfg = E.QuantizeConfig(bits=4, group_size=128, desc_act=True, static_groups=True,
                           model_name_or_path="synthetic-llama-like")
    layers = {f"model.layers.0.self_attn.{k}_proj": _quantized(256, 512, 4, 128, 7 + i)
              for i, k in enumerate("qkvo")}
    path = E.save_quantized(str(tmp_path), layers, cfg, use_safetensors=use_safetensors)
    assert os.path.basename(path) == "gptq_model-4bit-128g" + (".safetensors" if use_safetensors else ".bin")
    assert os.path.exists(os.path.join(tmp_path, "quantize_config.json"))
    cfg2, loaded = E.load_quantized(str(tmp_path), device=device())
    assert cfg2 == cfg
    assert set(loaded) == set(layers)
    for name, res in layers.items():
        t = loaded[name]
        assert torch.equal(t["qweight"], res.qweight) and torch.equal(t["g_idx"], res.g_idx)
        S, qz = O.export_tensors(res.scales.cpu().numpy(), res.zeros.cpu().numpy(), 4)
        assert np.array_equal(t["scales"].cpu().numpy().view(np.uint16), S.view(np.uint16))
        assert np.array_equal(t["qzeros"].cpu().numpy(), qz)
        # the checkpoint dequantizes to the layer's weights with half-precision scales
        zeros = O.unpack(t["qzeros"].cpu().numpy().T, 4, 256)  # [G, n_out]
        What = O.dequantize(t["qweight"].cpu().numpy(), S.astype(np.float32), zeros, t["g_idx"].cpu().numpy(), 4,
                            512)
        ref = O.dequantize(res.qweight.cpu().numpy(), res.scales.cpu().numpy().astype(np.float16).astype(np.float32),
                           res.zeros.cpu().numpy(), res.g_idx.cpu().numpy(), 4, 512)
        assert np.array_equal(What, ref)
