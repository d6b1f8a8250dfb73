"""Checkpoint export of quantized linears (save_quantized / load_quantized).

The AutoGPTQ examples guide (§1.4) and the OLMo quick-start (§四 step 4) describe what a
quantization run saves: one weights file named ``gptq_model-{bits}bit-{group_size}g`` --
``.bin`` by default, ``.safetensors`` with ``use_safetensors=True`` -- and beside it
``quantize_config.json``, the BaseQuantizeConfig fields (bits, group_size, damp_percent,
desc_act, static_groups, sym, true_sequential, model_name_or_path, model_file_base_name)
that the loader reads first to find and interpret the weights (OLMo quick-start §三 and
§四 step 5).

Per linear ``name`` the weights file holds ``name.qweight`` (int32, the sweep's packed
codes), ``name.qzeros`` (int32, packed zero points), ``name.scales`` (fp16) and
``name.g_idx`` (int32); the conversion of scales and zero points runs in the native
library (gptq_export_layer).  Serialization is host code: the safetensors container is a
little-endian 8-byte header length, a JSON header of dtype / shape / byte range per
tensor, then the raw bytes.
"""

from __future__ import annotations

import json
import os
import struct
from dataclasses import asdict, dataclass

import torch

from . import api
from ._native import lib

CONFIG_NAME = "quantize_config.json"


@dataclass
class QuantizeConfig:
    """The BaseQuantizeConfig fields that quantize_config.json records."""

    bits: int = 4
    group_size: int = 128
    damp_percent: float = 0.01
    desc_act: bool = False
    static_groups: bool = False
    sym: bool = True
    true_sequential: bool = True
    model_name_or_path: str | None = None
    model_file_base_name: str | None = None


def weights_basename(cfg: QuantizeConfig) -> str:
    """gptq_model-{bits}bit-{group_size}g, unless the config names its own base name."""
    return cfg.model_file_base_name or f"gptq_model-{cfg.bits}bit-{cfg.group_size}g"


def export_layer(res: api.QuantResult, bits: int, stream=None) -> dict:
    """Checkpoint tensors of one quantized linear (on its device): qweight and g_idx as
    produced, scales in fp16, zero points packed into int32 words along n_out."""
    G, n_out = res.scales.shape
    if res.zeros.shape != (G, n_out) or res.zeros.dtype != torch.int32 or res.scales.dtype != torch.float32:
        raise ValueError("scales must be float32 and zeros int32, both [G, n_out]")
    api._need_cuda(res.scales, res.zeros)
    scales16 = torch.empty(G, n_out, dtype=torch.float16, device=res.scales.device)
    qzeros = torch.empty(G, n_out * bits // 32, dtype=torch.int32, device=res.scales.device)
    st = lib().gptq_export_layer(api._ptr(res.scales), api._ptr(res.zeros), G, n_out, bits, api._ptr(scales16),
                                 api._ptr(qzeros), api._stream(stream))
    api._check(st, "gptq_export_layer")
    return {"qweight": res.qweight, "qzeros": qzeros, "scales": scales16, "g_idx": res.g_idx}


# ------------------------------------------------------------------ safetensors container
_ST_DTYPES = {torch.int32: "I32", torch.float16: "F16", torch.float32: "F32", torch.bfloat16: "BF16",
              torch.int64: "I64", torch.uint8: "U8"}
_ST_BACK = {v: k for k, v in _ST_DTYPES.items()}


def write_safetensors(path: str, tensors: dict, metadata: dict | None = None) -> None:
    """Write CPU copies of `tensors` (name -> tensor) in the safetensors layout."""
    header, blobs, off = {}, [], 0
    for name in sorted(tensors):
        t = tensors[name].detach().to("cpu").contiguous()
        b = t.view(torch.uint8).numpy().tobytes() if t.numel() else b""
        header[name] = {"dtype": _ST_DTYPES[t.dtype], "shape": list(t.shape), "data_offsets": [off, off + len(b)]}
        blobs.append(b)
        off += len(b)
    if metadata:
        header["__metadata__"] = {str(k): str(v) for k, v in metadata.items()}
    h = json.dumps(header, separators=(",", ":")).encode()
    h += b" " * (-len(h) % 8)  # the byte buffer starts 8-byte aligned
    with open(path, "wb") as f:
        f.write(struct.pack("<Q", len(h)))
        f.write(h)
        for b in blobs:
            f.write(b)


def read_safetensors(path: str) -> tuple[dict, dict]:
    """(tensors on the CPU, metadata) of a safetensors file."""
    with open(path, "rb") as f:
        (hlen,) = struct.unpack("<Q", f.read(8))
        header = json.loads(f.read(hlen))
        data = f.read()
    meta = header.pop("__metadata__", {})
    out = {}
    for name, e in header.items():
        a, b = e["data_offsets"]
        dt = _ST_BACK[e["dtype"]]
        buf = bytearray(data[a:b])
        t = torch.frombuffer(buf, dtype=dt) if b > a else torch.empty(0, dtype=dt)
        out[name] = t.reshape(e["shape"]).clone()
    return out, meta


# ------------------------------------------------------------------ save / load
def save_quantized(save_dir: str, layers: dict, cfg: QuantizeConfig, use_safetensors: bool = False,
                   stream=None) -> str:
    """Save quantized linears ({name: QuantResult}) and quantize_config.json into
    `save_dir`.  Returns the weights file's path."""
    os.makedirs(save_dir, exist_ok=True)
    tensors = {}
    for name, res in layers.items():
        for k, t in export_layer(res, cfg.bits, stream).items():
            tensors[f"{name}.{k}"] = t
    if stream is not None:
        stream.synchronize()
    else:
        torch.cuda.current_stream().synchronize()
    base = weights_basename(cfg)
    if use_safetensors:
        path = os.path.join(save_dir, base + ".safetensors")
        write_safetensors(path, tensors, {"format": "pt", "quantize_config": json.dumps(asdict(cfg))})
    else:
        path = os.path.join(save_dir, base + ".bin")
        torch.save({k: v.cpu() for k, v in tensors.items()}, path)
    with open(os.path.join(save_dir, CONFIG_NAME), "w") as f:
        json.dump(asdict(cfg), f, indent=2)
    return path


def load_quantized(save_dir: str, device=None) -> tuple[QuantizeConfig, dict]:
    """Read quantize_config.json, then the weights file it names (safetensors if present,
    else .bin).  Returns (config, {name: {"qweight", "qzeros", "scales", "g_idx"}})."""
    with open(os.path.join(save_dir, CONFIG_NAME)) as f:
        cfg = QuantizeConfig(**json.load(f))
    base = os.path.join(save_dir, weights_basename(cfg))
    if os.path.exists(base + ".safetensors"):
        flat, _ = read_safetensors(base + ".safetensors")
    elif os.path.exists(base + ".bin"):
        flat = torch.load(base + ".bin", map_location="cpu", weights_only=True)
    else:
        raise FileNotFoundError(f"no {weights_basename(cfg)}.safetensors or .bin in {save_dir}")
    layers = {}
    for key, t in flat.items():
        name, part = key.rsplit(".", 1)
        layers.setdefault(name, {})[part] = t.to(device) if device is not None else t
    return cfg, layers
