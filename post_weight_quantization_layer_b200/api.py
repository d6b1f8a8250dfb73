"""Torch-facing wrappers of the C ABI (argument marshalling only).

Tensors must already live on a CUDA device; outputs are allocated with torch
(device memory plumbing) and filled by the native kernels.  Every call goes to
``lib/libgptq.so``; nothing here computes any part of the method.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from ._native import GptqStats, lib

OK, INVALID_ARG, UNSUPPORTED, NOT_PD, CUDA_ERR, OOM, TIMEOUT = range(7)
_DTYPE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}


class GPTQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().gptq_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


def _check(st, where):
    if st != OK:
        raise GPTQError(st, where)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts):
    """Every tensor must be a contiguous CUDA tensor on the current device (checked last, so
    that shape and dtype errors are reported first)."""
    for t in ts:
        if not isinstance(t, torch.Tensor):
            raise ValueError("arguments must be torch tensors")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors")
        if t.device.index != torch.cuda.current_device():
            raise ValueError(f"tensor on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")


def _need(t, what, dtypes, shape):
    """Shape and dtype of one argument (raises ValueError before any native call)."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{what} must be a torch tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{what} must have dtype {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _weight(W):
    if not isinstance(W, torch.Tensor) or W.dim() != 2:
        raise ValueError("W must be a 2-D [n_out, n_in] tensor")
    if W.dtype not in _DTYPE:
        raise ValueError(f"W must be float32, float16 or bfloat16, got {W.dtype}")
    return W.shape


def group_count(n_in: int, group_size: int) -> int:
    return 1 if group_size == -1 else n_in // group_size


@dataclass
class QuantResult:
    qweight: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    g_idx: torch.Tensor
    stats: dict | None = None


def accumulate_hessian(X: torch.Tensor, H: torch.Tensor, stream=None) -> torch.Tensor:
    """H += 2 X^T X (asynchronous on the stream).  X [T, n] fp16/bf16, H [n, n] fp32."""
    if not isinstance(X, torch.Tensor) or X.dim() != 2:
        raise ValueError("X must be a 2-D [tokens, n_in] tensor")
    _need(X, "X", (torch.float16, torch.bfloat16), tuple(X.shape))
    _need(H, "H", (torch.float32,), (X.shape[1], X.shape[1]))
    _need_cuda(X, H)
    st = lib().gptq_accumulate_hessian(_ptr(X), _DTYPE.get(X.dtype, 99), X.shape[0], X.shape[1], _ptr(H),
                                       _stream(stream))
    _check(st, "gptq_accumulate_hessian")
    return H


def device_status(clear: bool = True, stream=None) -> int:
    return lib().gptq_device_status(_stream(stream), 1 if clear else 0)


def launch_count() -> int:
    return lib().gptq_launch_count()


def _outputs(n_out, n_in, bits, group_size, device, out):
    """Output tensors (qweight, scales, zeros, g_idx): allocated here, or the caller's
    `out` tuple after checking that every piece has the shape and dtype the call writes."""
    # an invalid group size is rejected by the native call, which then writes nothing
    G = group_count(n_in, group_size) if (group_size == -1 or group_size > 0) else 1
    words = n_in * bits // 32
    if out is None:
        return (torch.empty(words, n_out, dtype=torch.int32, device=device),
                torch.empty(G, n_out, dtype=torch.float32, device=device),
                torch.empty(G, n_out, dtype=torch.int32, device=device),
                torch.empty(n_in, dtype=torch.int32, device=device))
    if not isinstance(out, (tuple, list)) or len(out) != 4:
        raise ValueError("out must be a tuple (qweight, scales, zeros, g_idx)")
    qw, sc, zr, gi = out
    _need(qw, "out qweight", (torch.int32,), (words, n_out))
    _need(sc, "out scales", (torch.float32,), (G, n_out))
    _need(zr, "out zeros", (torch.int32,), (G, n_out))
    _need(gi, "out g_idx", (torch.int32,), (n_in,))
    _need_cuda(qw, sc, zr, gi)
    return tuple(out)


def _stats_dict(s: GptqStats):
    return {k: getattr(s, k) for k, _ in GptqStats._fields_}


def quantize_layer(W, H, bits=4, group_size=128, damp_percent=0.01, sym=True, desc_act=False,
                   static_groups=False, blocksize=128, stats=False, out=None, stream=None) -> QuantResult:
    """GPTQ of one linear layer: W [n_out, n_in] (fp32/fp16/bf16), H [n_in, n_in] fp32."""
    n_out, n_in = _weight(W)
    _need(H, "H", (torch.float32,), (n_in, n_in))
    qw, sc, zr, gi = _outputs(n_out, n_in, bits, group_size, W.device, out)
    _need_cuda(W, H)
    st_obj = GptqStats() if stats else None
    st = lib().gptq_quantize_layer(
        _ptr(W), _DTYPE.get(W.dtype, 99), n_out, n_in, _ptr(H), bits, group_size, float(damp_percent),
        int(bool(sym)), int(bool(desc_act)), int(bool(static_groups)), blocksize, _ptr(qw), _ptr(sc),
        _ptr(zr), _ptr(gi), _stream(stream), ctypes.byref(st_obj) if stats else None)
    _check(st, "gptq_quantize_layer")
    return QuantResult(qw, sc, zr, gi, _stats_dict(st_obj) if stats else None)


def factor_hessian(H, damp_percent=0.01, desc_act=False, stream=None):
    """Returns (U, perm): inverse(H_d) = U^T U in sweep order (fp64), perm = column order."""
    if not isinstance(H, torch.Tensor) or H.dim() != 2:
        raise ValueError("H must be a square 2-D tensor")
    n = H.shape[0]
    _need(H, "H", (torch.float32,), (n, n))
    _need_cuda(H)
    U = torch.empty(n, n, dtype=torch.float64, device=H.device)
    perm = torch.empty(n, dtype=torch.int32, device=H.device)
    st = lib().gptq_factor_hessian(_ptr(H), n, float(damp_percent), int(bool(desc_act)), _ptr(U), _ptr(perm),
                                   _stream(stream))
    _check(st, "gptq_factor_hessian")
    return U, perm


def factor_hessians(Hs, damp_percent=0.01, desc_act=False, stream=None):
    """factor_hessian for several independent Hessians in one call (run concurrently by
    the library).  Returns [(U, perm), ...] in the order of Hs; raises GPTQError naming
    the first item that failed."""
    Hs = list(Hs)
    if not Hs:
        raise ValueError("factor_hessians needs at least one Hessian")
    for i, H in enumerate(Hs):
        if not isinstance(H, torch.Tensor) or H.dim() != 2:
            raise ValueError(f"H[{i}] must be a square 2-D tensor")
        _need(H, f"H[{i}]", (torch.float32,), (H.shape[0], H.shape[0]))
    _need_cuda(*Hs)
    k = len(Hs)
    outs = [(torch.empty(H.shape[0], H.shape[0], dtype=torch.float64, device=H.device),
             torch.empty(H.shape[0], dtype=torch.int32, device=H.device)) for H in Hs]
    arr = ctypes.c_void_p * k
    st_arr = (ctypes.c_int * k)()
    st = lib().gptq_factor_hessians(k, arr(*[H.data_ptr() for H in Hs]),
                                    (ctypes.c_int64 * k)(*[H.shape[0] for H in Hs]), float(damp_percent),
                                    int(bool(desc_act)), arr(*[U.data_ptr() for U, _ in outs]),
                                    arr(*[p.data_ptr() for _, p in outs]), _stream(stream), st_arr)
    if st != OK:
        bad = next((i for i in range(k) if st_arr[i] != OK), None)
        _check(st, "gptq_factor_hessians" + (f" (item {bad})" if bad is not None else ""))
    return outs


def quantize_layer_factored(W, U, perm, bits=4, group_size=128, sym=True, static_groups=False, blocksize=128,
                            stats=False, out=None, stream=None) -> QuantResult:
    n_out, n_in = _weight(W)
    _need(U, "U", (torch.float64,), (n_in, n_in))
    _need(perm, "perm", (torch.int32,), (n_in,))
    qw, sc, zr, gi = _outputs(n_out, n_in, bits, group_size, W.device, out)
    _need_cuda(W, U, perm)
    st_obj = GptqStats() if stats else None
    st = lib().gptq_quantize_layer_factored(
        _ptr(W), _DTYPE.get(W.dtype, 99), n_out, n_in, _ptr(U), _ptr(perm), bits, group_size, int(bool(sym)),
        int(bool(static_groups)), blocksize, _ptr(qw), _ptr(sc), _ptr(zr), _ptr(gi), _stream(stream),
        ctypes.byref(st_obj) if stats else None)
    _check(st, "gptq_quantize_layer_factored")
    return QuantResult(qw, sc, zr, gi, _stats_dict(st_obj) if stats else None)


def quantize_linears(Hs, linears, bits=4, group_size=128, damp_percent=0.01, sym=True, desc_act=False,
                      static_groups=False, blocksize=128, stream=None, ready=None):
    """Factor every Hessian in Hs and quantize every linear in one pipelined call.

    Hs:      list of [n, n] float32 Hessians.
    linears: list of (W, h) pairs: W [n_out, n_in] weight (all of one dtype) whose input has
             Hessian Hs[h].
    ready:   optional list (one per Hessian) of recorded torch.cuda.Event or None: Hessian i's
             factor also waits for ready[i] (for Hessians accumulated on another stream).
    Returns ([(U, perm) per Hessian], [QuantResult per linear]): bit-identical to
    factor_hessians followed by quantize_layer_factored per linear.  Raises GPTQError naming
    the first linear that failed."""
    Hs, linears = list(Hs), list(linears)
    if not Hs or not linears:
        raise ValueError("quantize_linears needs at least one Hessian and one linear")
    for i, H in enumerate(Hs):
        if not isinstance(H, torch.Tensor) or H.dim() != 2:
            raise ValueError(f"H[{i}] must be a square 2-D tensor")
        _need(H, f"H[{i}]", (torch.float32,), (H.shape[0], H.shape[0]))
    dtypes = {W.dtype for W, _ in linears if isinstance(W, torch.Tensor)}
    if len(dtypes) > 1:
        raise ValueError("every linear must have the same weight dtype")
    outs, hidx = [], []
    for j, (W, h) in enumerate(linears):
        if not isinstance(h, int) or not 0 <= h < len(Hs):
            raise ValueError(f"linear {j}: Hessian index {h!r} out of range")
        n_out, n_in = _weight(W)
        if n_in != Hs[h].shape[0]:
            raise ValueError(f"linear {j}: n_in {n_in} does not match its Hessian's order {Hs[h].shape[0]}")
        outs.append(_outputs(n_out, n_in, bits, group_size, W.device, None))
        hidx.append(h)
    if ready is not None and len(ready) != len(Hs):
        raise ValueError("ready needs one entry (an event or None) per Hessian")
    _need_cuda(*Hs, *[W for W, _ in linears])
    factors = [(torch.empty(H.shape[0], H.shape[0], dtype=torch.float64, device=H.device),
                torch.empty(H.shape[0], dtype=torch.int32, device=H.device)) for H in Hs]
    kh, kl = len(Hs), len(linears)
    ah, al = ctypes.c_void_p * kh, ctypes.c_void_p * kl
    st_arr = (ctypes.c_int * kl)()
    st = lib().gptq_quantize_linears(
        kh, ah(*[H.data_ptr() for H in Hs]), (ctypes.c_int64 * kh)(*[H.shape[0] for H in Hs]), float(damp_percent),
        int(bool(desc_act)), ah(*[U.data_ptr() for U, _ in factors]), ah(*[p.data_ptr() for _, p in factors]), kl,
        al(*[W.data_ptr() for W, _ in linears]), _DTYPE.get(linears[0][0].dtype, 99),
        (ctypes.c_int64 * kl)(*[W.shape[0] for W, _ in linears]), (ctypes.c_int * kl)(*hidx), bits, group_size,
        int(bool(sym)), int(bool(static_groups)), blocksize, al(*[o[0].data_ptr() for o in outs]),
        al(*[o[1].data_ptr() for o in outs]), al(*[o[2].data_ptr() for o in outs]),
        al(*[o[3].data_ptr() for o in outs]),
        None if ready is None else ah(*[None if e is None else e.cuda_event for e in ready]), _stream(stream), st_arr)
    if st != OK:
        bad = next((j for j in range(kl) if st_arr[j] != OK), None)
        _check(st, "gptq_quantize_linears" + (f" (linear {bad})" if bad is not None else ""))
    return factors, [QuantResult(*o, None) for o in outs]


def _checkpoint(ck, bits):
    """(qweight, qzeros, scales, g_idx, groups, n_in, n_out) of a checkpoint-form linear
    (the dict of export.export_layer / export.load_quantized), checked."""
    try:
        qw, qz, sc, gi = ck["qweight"], ck["qzeros"], ck["scales"], ck["g_idx"]
    except (KeyError, TypeError):
        raise ValueError("checkpoint linear needs qweight, qzeros, scales and g_idx") from None
    if not isinstance(gi, torch.Tensor) or gi.dim() != 1:
        raise ValueError("g_idx must be a 1-D int32 tensor")
    n_in = gi.shape[0]
    if not isinstance(sc, torch.Tensor) or sc.dim() != 2:
        raise ValueError("scales must be a 2-D [groups, n_out] float16 tensor")
    G, n_out = sc.shape
    _need(qw, "qweight", (torch.int32,), (n_in * bits // 32, n_out))
    _need(qz, "qzeros", (torch.int32,), (G, n_out * bits // 32))
    _need(sc, "scales", (torch.float16,), (G, n_out))
    _need(gi, "g_idx", (torch.int32,), (n_in,))
    xp = ck.get("x_perm") if isinstance(ck, dict) else None
    if xp is not None:
        _need(xp, "x_perm", (torch.int32,), (n_in,))
    return qw, qz, sc, gi, G, n_in, n_out


def dequantize_weight(ck, bits=4, dtype=torch.float16, stream=None):
    """Dense [n_out, n_in] weight of a checkpoint-form linear, each value rounded once to
    `dtype` (float16 or bfloat16)."""
    qw, qz, sc, gi, G, n_in, n_out = _checkpoint(ck, bits)
    if dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("dtype must be float16 or bfloat16")
    _need_cuda(qw, qz, sc, gi)
    W = torch.empty(n_out, n_in, dtype=dtype, device=qw.device)
    st = lib().gptq_dequantize_weight(_ptr(qw), _ptr(qz), _ptr(sc), _ptr(gi), G, n_in, n_out, bits, _DTYPE[dtype],
                                      _ptr(W), _stream(stream))
    _check(st, "gptq_dequantize_weight")
    return W


def quantized_linear(X, ck, bits=4, out=None, stream=None):
    """Y = X W_hat^T for X [M, n_in] (float16 or bfloat16) and a checkpoint-form linear."""
    qw, qz, sc, gi, G, n_in, n_out = _checkpoint(ck, bits)
    if not isinstance(X, torch.Tensor) or X.dim() != 2:
        raise ValueError("X must be a 2-D [M, n_in] tensor")
    _need(X, "X", (torch.float16, torch.bfloat16), (X.shape[0], n_in))
    M = X.shape[0]
    if out is None:
        out = torch.empty(M, n_out, dtype=X.dtype, device=X.device)
    _need(out, "out", (X.dtype,), (M, n_out))
    xp = ck.get("x_perm")
    _need_cuda(X, out, qw, qz, sc, gi, *([xp] if xp is not None else []))
    st = lib().gptq_quantized_linear(_ptr(X), _DTYPE[X.dtype], M, n_in, _ptr(qw), _ptr(qz), _ptr(sc), _ptr(gi),
                                     None if xp is None else _ptr(xp), G, n_out, bits, _ptr(out), _stream(stream))
    _check(st, "gptq_quantized_linear")
    return out


def reorder_act_order(ck, bits=4, stream=None):
    """An act-order checkpoint with its inputs sorted by group (gptq_reorder_act_order): a new
    dict with qweight and g_idx reordered, qzeros and scales shared, and x_perm (row k of the
    codes belongs to input x_perm[k]).  quantized_linear gives the same product on it, with
    every word of codes in one group."""
    qw, qz, sc, gi, G, n_in, n_out = _checkpoint(ck, bits)
    if ck.get("x_perm") is not None:
        raise ValueError("checkpoint is already reordered")
    _need_cuda(qw, gi)
    qw2, gi2, xp = torch.empty_like(qw), torch.empty_like(gi), torch.empty_like(gi)
    st = lib().gptq_reorder_act_order(_ptr(qw), _ptr(gi), G, n_in, n_out, bits, _ptr(qw2), _ptr(gi2), _ptr(xp),
                                      _stream(stream))
    _check(st, "gptq_reorder_act_order")
    out = dict(ck)
    out.update(qweight=qw2, g_idx=gi2, x_perm=xp)
    return out


# ------------------------------------------------------------------ decoder-layer forward pieces
def _act(x, what):
    if not isinstance(x, torch.Tensor) or x.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError(f"{what} must be a float16 or bfloat16 tensor")
    return x


def rmsnorm(x, gamma, eps=1e-5, stream=None):
    """x / sqrt(mean(x^2) + eps) * gamma over the last dimension of x [rows, dim]."""
    _act(x, "x")
    if x.dim() != 2:
        raise ValueError("x must be [rows, dim]")
    _need(gamma, "gamma", (x.dtype,), (x.shape[1],))
    y = torch.empty_like(x)
    _need_cuda(x, gamma, y)
    _check(lib().gptq_rmsnorm(_ptr(x), _DTYPE[x.dtype], x.shape[0], x.shape[1], _ptr(gamma), float(eps), _ptr(y),
                              _stream(stream)), "gptq_rmsnorm")
    return y


def rope_(x, heads, seq_len, base=10000.0, stream=None):
    """Rotary embedding in place on x [tokens, heads * head_dim] (tokens = whole sequences)."""
    _act(x, "x")
    if x.dim() != 2 or x.shape[1] % heads:
        raise ValueError("x must be [tokens, heads * head_dim]")
    _need_cuda(x)
    _check(lib().gptq_rope(_ptr(x), _DTYPE[x.dtype], x.shape[0], heads, x.shape[1] // heads, seq_len, float(base),
                           _stream(stream)), "gptq_rope")
    return x


def attention(q, k, v, heads, seq_len, stream=None):
    """Causal softmax attention per sequence and head; q, k, v [tokens, heads * head_dim]."""
    _act(q, "q")
    if q.dim() != 2 or q.shape[1] % heads:
        raise ValueError("q must be [tokens, heads * head_dim]")
    _need(k, "k", (q.dtype,), tuple(q.shape))
    _need(v, "v", (q.dtype,), tuple(q.shape))
    out = torch.empty_like(q)
    _need_cuda(q, k, v, out)
    _check(lib().gptq_attention(_ptr(q), _ptr(k), _ptr(v), _DTYPE[q.dtype], q.shape[0], heads, q.shape[1] // heads,
                                seq_len, _ptr(out), _stream(stream)), "gptq_attention")
    return out


def silu_mul(gate, up, stream=None):
    """gate / (1 + exp(-gate)) * up, elementwise."""
    _act(gate, "gate")
    _need(up, "up", (gate.dtype,), tuple(gate.shape))
    out = torch.empty_like(gate)
    _need_cuda(gate, up, out)
    _check(lib().gptq_silu_mul(_ptr(gate), _ptr(up), _DTYPE[gate.dtype], gate.numel(), _ptr(out), _stream(stream)),
           "gptq_silu_mul")
    return out


def add(a, b, stream=None):
    """a + b, elementwise (the residual connection)."""
    _act(a, "a")
    _need(b, "b", (a.dtype,), tuple(a.shape))
    out = torch.empty_like(a)
    _need_cuda(a, b, out)
    _check(lib().gptq_add(_ptr(a), _ptr(b), _DTYPE[a.dtype], a.numel(), _ptr(out), _stream(stream)), "gptq_add")
    return out
