"""Host side of the checkpoint export: the safetensors container, quantize_config.json and
the loader's file lookup (the AutoGPTQ examples guide §1.4; OLMo quick-start §四 steps 4-5).
Tensors here come from the oracle; the GPU conversion is tested in test_gpu_export.py."""

import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from post_weight_quantization_layer_b200 import export as E


def _tensors():
    g = torch.Generator().manual_seed(3)
    return {"a.qweight": torch.randint(-2**31, 2**31 - 1, (16, 8), generator=g, dtype=torch.int64).to(torch.int32),
            "a.scales": torch.rand(4, 8, generator=g).half(),
            "b.x": torch.randn(3, 5, generator=g),
            "b.empty": torch.zeros(0, 4, dtype=torch.int32)}


def test_safetensors_roundtrip(tmp_path):
    t = _tensors()
    p = os.path.join(tmp_path, "w.safetensors")
    E.write_safetensors(p, t, {"format": "pt"})
    back, meta = E.read_safetensors(p)
    assert meta == {"format": "pt"}
    assert set(back) == set(t)
    for k in t:
        assert back[k].dtype == t[k].dtype and torch.equal(back[k], t[k]), k
    with open(p, "rb") as f:
        hlen = int.from_bytes(f.read(8), "little")
    assert (8 + hlen) % 8 == 0  # the byte buffer starts 8-byte aligned


def test_safetensors_matches_reference_reader(tmp_path):
    st = pytest.importorskip("safetensors.torch")
    t = {k: v for k, v in _tensors().items() if v.numel()}
    p = os.path.join(tmp_path, "w.safetensors")
    E.write_safetensors(p, t)
    lib_read = st.load_file(p)
    for k in t:
        assert torch.equal(lib_read[k], t[k]), k
    q = os.path.join(tmp_path, "lib.safetensors")
    st.save_file(t, q)
    ours, _ = E.read_safetensors(q)
    for k in t:
        assert torch.equal(ours[k], t[k]), k


@pytest.mark.parametrize("use_safetensors", [True, False])
def test_load_quantized_reads_config_then_weights(tmp_path, use_safetensors):
    """The loader reads quantize_config.json first and finds gptq_model-{bits}bit-{g}g."""
    rng = np.random.default_rng(1)
    cfg = E.QuantizeConfig(bits=3, group_size=64, desc_act=True, model_name_or_path="synthetic")
    zeros = rng.integers(0, 8, size=(4, 64))
    S, qz = O.export_tensors(rng.random((4, 64)), zeros, 3)
    t = {"layer.q.qzeros": torch.from_numpy(qz), "layer.q.scales": torch.from_numpy(S),
         "layer.q.g_idx": torch.arange(256, dtype=torch.int32) // 64,
         "layer.q.qweight": torch.from_numpy(O.pack(rng.integers(0, 8, size=(64, 256)), 3))}
    base = os.path.join(tmp_path, "gptq_model-3bit-64g")
    if use_safetensors:
        E.write_safetensors(base + ".safetensors", t)
    else:
        torch.save(t, base + ".bin")
    with open(os.path.join(tmp_path, "quantize_config.json"), "w") as f:
        json.dump(E.asdict(cfg), f)
    cfg2, layers = E.load_quantized(str(tmp_path))
    assert cfg2 == cfg
    assert set(layers) == {"layer.q"}
    for k, v in t.items():
        assert torch.equal(layers["layer.q"][k.rsplit(".", 1)[1]], v)
    assert np.array_equal(O.unpack(layers["layer.q"]["qzeros"].numpy().T, 3, 64), zeros)


def test_load_quantized_missing_weights(tmp_path):
    with open(os.path.join(tmp_path, "quantize_config.json"), "w") as f:
        json.dump(E.asdict(E.QuantizeConfig(model_file_base_name="custom")), f)
    with pytest.raises(FileNotFoundError, match="custom"):
        E.load_quantized(str(tmp_path))
