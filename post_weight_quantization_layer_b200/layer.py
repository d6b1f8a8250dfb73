"""Decoder-layer driver: quantize every linear of one transformer block.

The modules that read the same input share one calibration Hessian (q/k/v the
attention input, gate/up the MLP input; the OLMo quick-start's fused att_proj,
§六 6.1).  Each distinct Hessian is accumulated once and factored once, and every
module that reads it is swept against that factor.  By default the factors and
sweeps are one pipelined native call (gptq_quantize_linears: each linear's sweep
starts as soon as its own Hessian is factored, while the larger factors are still
running); pipelined=False runs them as two phases (gptq_factor_hessians, then one
gptq_quantize_layer_factored per module), which gives bit-identical results and
separate factor and sweep times.  All arithmetic runs in the native library; this
module only sequences the calls and records per-phase CUDA-event times on the
stream.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import api


@dataclass
class LayerTimes:
    hessian_ms: float = 0.0  # start until every Hessian is accumulated
    factor_ms: float = 0.0  # two-phase route only
    sweep_ms: float = 0.0  # two-phase route only
    # two-phase: factors and sweeps; pipelined: from the largest Hessian's completion (where
    # its factor starts) to the end, overlapping the other Hessians' accumulation
    factor_sweep_ms: float = 0.0
    total_ms: float = 0.0
    hessian_launch_ms: list = field(default_factory=list)


_side_streams = {}


def _side_stream(device):
    """A library-side torch stream per device for the smaller Hessians of a pipelined layer."""
    key = torch.device(device).index
    if key not in _side_streams:
        _side_streams[key] = torch.cuda.Stream(device=device)
    return _side_streams[key]


def quantize_decoder_layer(acts, weights, modules, qcfg, hessians=None, timing=False, stream=None,
                           hessians_given=False, pipelined=True):
    """Quantize the linears of one decoder layer.

    acts:     {h_index: X [tokens, n] fp16/bf16 CUDA tensor, or a list of token chunks}
    weights:  {module name: W [n_out, n_in] CUDA tensor}
    modules:  iterable of objects with .name and .h_index
    qcfg:     object with bits, group_size, damp_percent, sym, desc_act, static_groups, blocksize
    hessians: optional {h_index: preallocated [n, n] fp32 CUDA tensor} (zeroed here)
    hessians_given: the `hessians` already hold the layer's Hessians (accumulated earlier,
              e.g. streamed chunk by chunk); `acts` is then ignored and nothing is
              accumulated.
    pipelined: factors and sweeps in one overlapped call (default) or as two phases.
    Returns ({module name: QuantResult}, LayerTimes or None).
    """
    stream = stream or torch.cuda.current_stream()
    ev = (lambda: torch.cuda.Event(enable_timing=True)) if timing else None
    times = LayerTimes() if timing else None
    marks = []

    def mark_on(st):
        if timing:
            e = ev()
            e.record(st)
            marks.append(e)
            return e
        return None

    def mark():
        return mark_on(stream)

    with torch.cuda.stream(stream):
        m0 = mark()
        Hs = {}
        launch_marks = []
        ready = None
        m_first = None
        if hessians_given:
            if not hessians:
                raise ValueError("hessians_given needs the layer's Hessians in `hessians`")
            Hs = dict(hessians)
        else:
            def width(X):
                return (X[0] if isinstance(X, (list, tuple)) else X).shape[1]

            for h, X in acts.items():
                n = width(X)
                chunks = X if isinstance(X, (list, tuple)) else [X]
                Hs[h] = hessians[h] if hessians is not None else torch.empty(n, n, dtype=torch.float32,
                                                                             device=chunks[0].device)

            def accumulate(h, st):
                X = acts[h]
                chunks = X if isinstance(X, (list, tuple)) else [X]
                with torch.cuda.stream(st):
                    Hs[h].zero_()
                    a = mark_on(st)
                    for c in chunks:
                        api.accumulate_hessian(c, Hs[h], stream=st)
                    launch_marks.append((h, a, mark_on(st)))

            # the largest Hessian first: with the pipelined route its factor (the layer's
            # critical path) starts while the others are still being accumulated
            order = sorted(acts, key=lambda h: -width(acts[h]))
            accumulate(order[0], stream)
            m_first = mark()
            if pipelined and len(order) > 1:
                side = _side_stream(stream.device)
                side.wait_stream(stream)
                for h in order[1:]:
                    accumulate(h, side)
                side_done = torch.cuda.Event(enable_timing=timing)
                side_done.record(side)
                ready = [None if h == order[0] else side_done for h in Hs]
                m_h = side_done if timing else None
            else:
                for h in order[1:]:
                    accumulate(h, stream)
        if ready is None:
            m_h = mark()
        if m_first is None:
            m_first = m_h
        keys = list(Hs)
        m_f = None
        if pipelined:
            hpos = {h: i for i, h in enumerate(keys)}
            mods = list(modules)
            _, res = api.quantize_linears([Hs[h] for h in keys], [(weights[m.name], hpos[m.h_index]) for m in mods],
                                          qcfg.bits, qcfg.group_size, qcfg.damp_percent, qcfg.sym, qcfg.desc_act,
                                          qcfg.static_groups, qcfg.blocksize, stream=stream, ready=ready)
            results = {m.name: r for m, r in zip(mods, res)}
        else:
            # every distinct Hessian factored in one call: the library runs them concurrently
            factors = dict(zip(keys, api.factor_hessians([Hs[h] for h in keys], qcfg.damp_percent, qcfg.desc_act,
                                                         stream=stream)))
            m_f = mark()
            results = {}
            for mod in modules:
                U, perm = factors[mod.h_index]
                results[mod.name] = api.quantize_layer_factored(
                    weights[mod.name], U, perm, qcfg.bits, qcfg.group_size, qcfg.sym, qcfg.static_groups,
                    qcfg.blocksize, stream=stream)
        m_s = mark()
    if timing:
        m_s.synchronize()
        times.hessian_ms = m0.elapsed_time(m_h)
        times.factor_sweep_ms = (m_h if ready is None else m_first).elapsed_time(m_s)
        times.total_ms = m0.elapsed_time(m_s)
        if m_f is not None:
            times.factor_ms = m_h.elapsed_time(m_f)
            times.sweep_ms = m_f.elapsed_time(m_s)
        by_h = {h: a.elapsed_time(b) for h, a, b in launch_marks}
        times.hessian_launch_ms = [by_h[h] for h in sorted(by_h)]
    return results, times
