"""Float64 CPU oracle of GPTQ layer quantization (test infrastructure only).

This module is test infrastructure: only the tests, the smoke check and the
CPU-baseline leg of the benchmark call it.  It shares no code with the CUDA
path.  It restates, step by step and in plain NumPy float64, what the pages
describe:

1. calibration Hessian H = 2 X^T X                    [ch5 §5.1.7]
2. act-order permutation by descending diag(H)        [examples §1.4: desc_act]
3. damping H + damp * mean(diag H) * I                [ch5 §5.1.8, key point 2]
4. upper Cholesky factor U of inverse(H_d)            [ch5 §5.1.8, key point 1]
5. uniform quantizer with scale and zero point        [ch5 §5.1.1; skill card 分组量化]
6. per-group parameters, fixed once computed          [ch5 §5.1.10; pseudo-code "fixed scale"]
7. column sweep with normalised error and compensation,
   eager or lazy-blocked                              [ch5 §5.1.8 pseudo-code]
8. un-permute and pack codes into int32 words         (layout is this library's; the pages give none)

Where a floating-point value decides an integer code, the decision is taken in
float32, the precision the GPU kernels use; every other step is float64.

Readings taken where the pages are silent:
* rounding is round-half-to-even; division is IEEE x / s, never x * (1/s);
* sym: s = 2*max|x| / maxq, zero = 2^(bits-1);
* asym: range [min(0, min x), max(0, max x)], s = (hi-lo)/maxq, zero = rint(-lo/s);
* a degenerate group (all zero) uses the range [-1, 1];
* group_size = -1 means one group per output row, taken from the row before
  any update; group_size > 0 must divide n_in;
* non-static groups take their parameters from the current, already
  error-updated weights when the sweep reaches the group's first column;
* static_groups takes every group's parameters from the original, unpermuted
  weights before any update, and column c always uses group c // group_size;
* act-order ties keep ascending original index (stable sort).
"""

from __future__ import annotations

import numpy as np
from scipy.linalg import lapack as _lapack

__all__ = [
    "NotPositiveDefinite",
    "validate_config",
    "hessian",
    "accumulate_hessian",
    "act_order_perm",
    "dampen",
    "inverse_cholesky_upper",
    "quant_params",
    "quantize",
    "gptq_quantize",
    "gptq_sweep",
    "rtn_quantize",
    "obq_quantize",
    "pack",
    "unpack",
    "dequantize",
    "export_tensors",
    "dequantize_checkpoint",
    "round16",
    "quantized_linear",
    "layer_loss",
    "layer_loss_h",
    "brute_force_min_loss",
    "group_count",
]

VALID_BITS = (2, 3, 4, 8)


class NotPositiveDefinite(ValueError):
    """The damped Hessian has a non-positive or non-finite pivot.

    Counterpart of the Cholesky LinAlgError that one page reports when the
    damping is too small (dpshk practitioner account, §2.2).
    """


# --------------------------------------------------------------------------- config
def validate_config(bits, group_size, damp_percent, blocksize=128, n_in=None):
    """Reject configurations the pages forbid, raising ValueError.

    [examples §1.4; OLMo §三]: bits must be one of 2/3/4/8; group_size is -1
    (no grouping) or > 0; damp_percent lies strictly inside (0, 1).
    Readings: blocksize must be > 0, and group_size must divide n_in
    (the skill card's group-count example, 分组量化, divides exactly).
    """
    if bits not in VALID_BITS:
        raise ValueError(f"bits must be one of {VALID_BITS}, got {bits}")
    if not (group_size == -1 or group_size > 0):
        raise ValueError(f"group_size must be -1 or > 0, got {group_size}")
    d = float(damp_percent)
    if not (0.0 < d < 1.0):  # also rejects NaN
        raise ValueError(f"damp_percent must lie in (0, 1), got {damp_percent}")
    if blocksize <= 0:
        raise ValueError(f"blocksize must be > 0, got {blocksize}")
    if n_in is not None:
        if n_in <= 0:
            raise ValueError("n_in must be > 0")
        if group_size > 0 and n_in % group_size != 0:
            raise ValueError(f"group_size {group_size} must divide n_in {n_in}")


def group_count(n_in, group_size):
    """Groups per output row: n_in / group_size, or 1 without grouping.

    [skill card, 分组量化]: a [1024, 4096] matrix at group size 128 has
    4.2M / 128 = 32,768 groups in total, i.e. 32 per row of 4096 inputs.
    """
    return 1 if group_size == -1 else n_in // group_size


# --------------------------------------------------------------------------- Hessian
def hessian(X):
    """H = 2 * X^T X in float64, X = [tokens, n_in].

    [ch5 §5.1.7]: the reconstruction objective ||(W - W_q) X||^2 is a quadratic
    form whose Hessian is X X^T up to a constant; with tokens as rows that is
    X^T X, and the constant here is 2 (the Hessian of the squared error).
    """
    X = np.asarray(X, dtype=np.float64)
    return 2.0 * (X.T @ X)


def accumulate_hessian(H, X):
    """Streaming form: H + 2 * X^T X for one more chunk of calibration tokens."""
    return np.asarray(H, dtype=np.float64) + hessian(X)


# --------------------------------------------------------------------------- ordering / damping / factor
def act_order_perm(H):
    """Column order for desc_act: descending diag(H), ties by ascending index.

    [examples §1.4: desc_act reorders columns by activation]; the sort key is
    diag(H) (the energy of each input channel over the calibration data).
    """
    d = np.diag(np.asarray(H, dtype=np.float64))
    return np.argsort(-d, kind="stable")


def dampen(H, damp_percent):
    """H + damp_percent * mean(diag H) * I   [ch5 §5.1.8, key point 2]."""
    H = np.array(H, dtype=np.float64, copy=True)
    n = H.shape[0]
    H[np.arange(n), np.arange(n)] += damp_percent * np.mean(np.diag(H))
    return H


def inverse_cholesky_upper(Hd):
    """Upper-triangular U with inverse(Hd) = U^T U and positive diagonal.

    Literal route of [ch5 §5.1.8, key point 1 and the pseudo-code's factor
    step]: invert the damped Hessian once, then take its Cholesky factor; the
    rows of the factor are the compensation coefficients of the sweep.
    Raises NotPositiveDefinite if Hd is not positive definite.
    """
    Hd = np.asarray(Hd, dtype=np.float64)
    if not np.all(np.isfinite(Hd)):
        raise NotPositiveDefinite("non-finite entries in the damped Hessian")
    # inverse(Hd) of a symmetric positive definite matrix, formed from its own Cholesky
    # factor (LAPACK potrf, then potri, upper triangles); potrf's failure is the
    # not-positive-definite case
    C, info = _lapack.dpotrf(Hd, lower=0, clean=1)
    if info != 0:
        raise NotPositiveDefinite(f"Cholesky of the damped Hessian failed (potrf info {info})")
    Hinv, info = _lapack.dpotri(C, lower=0)  # upper triangle of inverse(Hd)
    if info != 0:
        raise NotPositiveDefinite(f"inverse of the damped Hessian failed (potri info {info})")
    # Cholesky factor of the inverse: upper U with inverse(Hd) = U^T U (potrf reads the
    # upper triangle only)
    U, info = _lapack.dpotrf(Hinv, lower=0, clean=1)
    if info != 0:
        raise NotPositiveDefinite(f"Cholesky of the inverse failed (potrf info {info})")
    return np.ascontiguousarray(U)  # LAPACK returns column-major storage


# --------------------------------------------------------------------------- quantizer
def quant_params(x, bits, sym):
    """Scale and zero point of a group, computed in float32.

    x is [rows, group] (float64 current weights).  [ch5 §5.1.1]: x_q =
    round(x / s), x_hat = s * x_q; [skill card, 分组量化]: each group has its
    own scale and zero point.  Readings (pages silent): sym uses s = 2*max|x|
    / maxq with zero 2^(bits-1); asym uses [min(0,min x), max(0,max x)] with
    zero = rint(-lo / s); an all-zero group uses the range [-1, 1].
    Returns (scale float32 [rows], zero int64 [rows]).
    """
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    if x32.ndim == 1:
        x32 = x32[:, None]
    maxq = np.float32(2**bits - 1)
    if sym:
        a = np.max(np.abs(x32), axis=1)
        a = np.where(a == np.float32(0), np.float32(1), a).astype(np.float32)
        s = (np.float32(2) * a) / maxq
        z = np.full(a.shape, 2 ** (bits - 1), dtype=np.int64)
    else:
        lo = np.minimum(np.float32(0), np.min(x32, axis=1)).astype(np.float32)
        hi = np.maximum(np.float32(0), np.max(x32, axis=1)).astype(np.float32)
        deg = hi == lo
        lo = np.where(deg, np.float32(-1), lo).astype(np.float32)
        hi = np.where(deg, np.float32(1), hi).astype(np.float32)
        s = (hi - lo).astype(np.float32) / maxq
        z = np.rint((-lo).astype(np.float32) / s).astype(np.int64)
        z = np.clip(z, 0, int(maxq))
    return s.astype(np.float32), z


def quantize(x, scale, zero, bits):
    """Codes and dequantized values of one column (or any array).

    q = clamp(rint(x / s) + z, 0, maxq), decided in float32;
    x_hat = s * (q - z) in float64.  [ch5 §5.1.1]
    """
    maxq = 2**bits - 1
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    s = np.asarray(scale, dtype=np.float32)
    r = np.rint(x32 / s).astype(np.int64)
    q = np.clip(r + np.asarray(zero, dtype=np.int64), 0, maxq)
    xhat = s.astype(np.float64) * (q - np.asarray(zero, dtype=np.int64)).astype(np.float64)
    return q, xhat


# --------------------------------------------------------------------------- sweep
def _params_source(W_orig, bits, sym, group_size, static_groups):
    """Parameters that are fixed before the sweep starts, or None.

    g = -1: one group per row from the row before any update.
    static_groups: every group from the original (unpermuted) weights.
    """
    n_out, n_in = W_orig.shape
    if group_size == -1:
        s, z = quant_params(W_orig, bits, sym)
        return s[None, :], z[None, :]
    if static_groups:
        G = n_in // group_size
        S = np.empty((G, n_out), np.float32)
        Z = np.empty((G, n_out), np.int64)
        for k in range(G):
            S[k], Z[k] = quant_params(W_orig[:, k * group_size:(k + 1) * group_size], bits, sym)
        return S, Z
    return None


def gptq_sweep(Wp, U, bits, sym, group_size, perm, static_groups, W_orig, blocksize=None):
    """Quantize-and-compensate column sweep over the permuted weights.

    [ch5 §5.1.8 pseudo-code]: for each column q: quantize it with the fixed
    group scale, form the normalised error err = (w - q_int) / U[q, q], and
    subtract err (outer) U[q, later columns] from the columns not yet
    quantized.  With ``blocksize`` None the compensation is eager (every later
    column at once); with a block size it is lazy: within a block only the
    block's later columns are updated, and after the block the accumulated
    block errors hit all later columns in one matrix product (the lazy batch
    update, key point 3).  Both orders give the same result in exact
    arithmetic.

    Wp: [n_out, n_in] float64 weights in sweep order (columns W[:, perm]).
    Returns dict(codes, xhat, err, scales, zeros, gsweep) all in sweep order,
    where gsweep[j] is the group index used by sweep position j.
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    n_out, n_in = W.shape
    G = group_count(n_in, group_size)
    fixed = _params_source(W_orig, bits, sym, group_size, static_groups)
    if fixed is not None:
        S, Z = fixed
    else:
        S = np.zeros((G, n_out), np.float32)
        Z = np.zeros((G, n_out), np.int64)
    codes = np.zeros((n_out, n_in), np.int64)
    xhat = np.zeros((n_out, n_in), np.float64)
    err = np.zeros((n_out, n_in), np.float64)
    gsweep = np.zeros(n_in, np.int64)

    B = n_in if blocksize is None else int(blocksize)
    if blocksize is not None and group_size > 0 and not static_groups:
        if not (B % group_size == 0 or group_size % B == 0):
            raise ValueError("lazy blocks must align with group boundaries")

    for b0 in range(0, n_in, B):
        b1 = min(b0 + B, n_in)
        for j in range(b0, b1):
            if group_size == -1:
                gi = 0
            elif static_groups:
                gi = int(perm[j]) // group_size
            else:
                gi = j // group_size
                if j % group_size == 0:
                    S[gi], Z[gi] = quant_params(W[:, j:j + group_size], bits, sym)
            gsweep[j] = gi
            q, xh = quantize(W[:, j], S[gi], Z[gi], bits)
            e = (W[:, j] - xh) / U[j, j]
            hi = b1 if blocksize is not None else n_in
            W[:, j + 1:hi] -= np.outer(e, U[j, j + 1:hi])
            codes[:, j] = q
            xhat[:, j] = xh
            err[:, j] = e
        if blocksize is not None and b1 < n_in:
            W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
    return dict(codes=codes, xhat=xhat, err=err, scales=S, zeros=Z, gsweep=gsweep)


def gptq_quantize(W, H, bits, group_size, damp_percent, sym=True, desc_act=False,
                  static_groups=False, blocksize=None):
    """GPTQ on one linear layer, end to end (the oracle of the whole path).

    W: [n_out, n_in] weights; H: [n_in, n_in] calibration Hessian.
    Steps: [examples §1.4] validate; [examples §1.4: desc_act] permute;
    [ch5 §5.1.8] damp, factor, sweep; then un-permute and pack.
    Returns a dict with the packed outputs (qweight, scales, zeros, g_idx) and
    intermediates (perm, U, codes in original order, What, err, damped_loss).
    """
    W = np.asarray(W, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    n_out, n_in = W.shape
    validate_config(bits, group_size, damp_percent, 128 if blocksize is None else blocksize, n_in)
    perm = act_order_perm(H) if desc_act else np.arange(n_in)
    Hp = H[np.ix_(perm, perm)]
    Hd = dampen(Hp, damp_percent)
    U = inverse_cholesky_upper(Hd)
    r = gptq_sweep(W[:, perm], U, bits, sym, group_size, perm, static_groups, W, blocksize)

    codes = np.empty_like(r["codes"])
    codes[:, perm] = r["codes"]
    What = np.empty_like(r["xhat"])
    What[:, perm] = r["xhat"]
    g_idx = np.empty(n_in, np.int64)
    g_idx[perm] = r["gsweep"]
    return dict(
        qweight=pack(codes, bits) if (n_in * bits) % 32 == 0 else None,
        scales=r["scales"].astype(np.float32),
        zeros=r["zeros"].astype(np.int32),
        g_idx=g_idx.astype(np.int32),
        codes=codes,
        What=What,
        err=r["err"],
        perm=perm,
        U=U,
        Hd=Hd,
        damped_loss=float(np.sum(r["err"] ** 2)),
    )


def rtn_quantize(W, bits, group_size, sym):
    """Round-to-nearest baseline: same quantizer and groups, no compensation.

    [ch5 §5.1.3] contrasts GPTQ with rounding every weight on its own.
    Groups are consecutive original columns.  Returns (codes, What).
    """
    W = np.asarray(W, dtype=np.float64)
    n_out, n_in = W.shape
    g = n_in if group_size == -1 else group_size
    codes = np.empty((n_out, n_in), np.int64)
    What = np.empty((n_out, n_in), np.float64)
    for k in range(0, n_in, g):
        s, z = quant_params(W[:, k:k + g], bits, sym)
        for c in range(k, k + g):
            codes[:, c], What[:, c] = quantize(W[:, c], s, z, bits)
    return codes, What


# --------------------------------------------------------------------------- OBS / OBQ route
def obq_quantize(W, Hd, bits, group_size, sym):
    """Cross-route through the OBS closed form with explicit inverse updates.

    [ch5 §5.1.8, "OBS 闭式解"]: quantizing weight q gives the error e_q =
    w_q - quant(w_q); the optimal change of the remaining weights is
    delta = -e_q / [H^-1]_qq * (H^-1)_{:,q}, and the loss grows by
    e_q^2 / [H^-1]_qq.  After each step the inverse is updated by Gaussian
    elimination of row/column q (the slow naive scheme the page describes).
    Columns in natural order, non-static groups.  For tiny n only.
    Returns (codes, What, delta_E per column summed over rows).
    """
    W = np.array(W, dtype=np.float64, copy=True)
    n_out, n_in = W.shape
    Hinv = np.linalg.inv(np.asarray(Hd, dtype=np.float64))
    G = group_count(n_in, group_size)
    fixed = _params_source(W, bits, sym, group_size, False) if group_size == -1 else None
    S = fixed[0] if fixed else np.zeros((G, n_out), np.float32)
    Z = fixed[1] if fixed else np.zeros((G, n_out), np.int64)
    codes = np.zeros((n_out, n_in), np.int64)
    What = np.zeros((n_out, n_in))
    dE = np.zeros(n_in)
    for q in range(n_in):
        gi = 0 if group_size == -1 else q // group_size
        if group_size > 0 and q % group_size == 0:
            S[gi], Z[gi] = quant_params(W[:, q:q + group_size], bits, sym)
        cq, xh = quantize(W[:, q], S[gi], Z[gi], bits)
        e = W[:, q] - xh
        d = Hinv[q, q]
        W[:, q + 1:] += -np.outer(e / d, Hinv[q + 1:, q])
        W[:, q] = xh
        codes[:, q] = cq
        What[:, q] = xh
        dE[q] = np.sum(e * e) / d
        Hinv = Hinv - np.outer(Hinv[:, q], Hinv[q, :]) / d
    return codes, What, dE


# --------------------------------------------------------------------------- packing
def pack(codes, bits):
    """Pack [n_out, n_in] codes into int32 words, shape [n_in*bits/32, n_out].

    Layout of this library (the pages name only "INT4 + scale + zero_point"):
    for each output channel the codes along n_in form a least-significant-bit
    first stream of ``bits``-bit fields cut into 32-bit words; a field may
    straddle two words (3-bit).
    """
    codes = np.asarray(codes, dtype=np.int64)
    n_out, n_in = codes.shape
    if (n_in * bits) % 32:
        raise ValueError("n_in * bits must be a multiple of 32")
    nw = n_in * bits // 32
    out = np.zeros((nw, n_out), dtype=np.uint64)
    mask = (1 << bits) - 1
    for c in range(n_in):
        v = (codes[:, c] & mask).astype(np.uint64)
        pos = c * bits
        w, off = divmod(pos, 32)
        out[w] |= (v << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            out[w + 1] |= v >> np.uint64(32 - off)
    return out.astype(np.uint32).view(np.int32)


def unpack(qweight, bits, n_in):
    """Inverse of :func:`pack`: [n_in*bits/32, n_out] int32 -> [n_out, n_in] codes."""
    q = np.asarray(qweight).view(np.uint32).astype(np.uint64)
    n_out = q.shape[1]
    codes = np.zeros((n_out, n_in), dtype=np.int64)
    mask = np.uint64((1 << bits) - 1)
    for c in range(n_in):
        pos = c * bits
        w, off = divmod(pos, 32)
        v = q[w] >> np.uint64(off)
        if off + bits > 32:
            v |= q[w + 1] << np.uint64(32 - off)
        codes[:, c] = (v & mask).astype(np.int64)
    return codes


def export_tensors(scales, zeros, bits):
    """Checkpoint form of a linear's group parameters: (fp16 scales, packed zero points).

    [examples §1.4; OLMo §四 step 4]: save_quantized stores the quantized weights with
    their scale and zero point; the pages give no tensor layout.  Layout of this library:
    scales rounded to IEEE half precision (round to nearest even), and for each group
    the zero points of the output channels packed as :func:`pack` packs codes, along
    n_out: qzeros [G, n_out*bits/32].
    """
    S = np.asarray(scales, dtype=np.float32).astype(np.float16)
    Z = np.asarray(zeros, dtype=np.int64)
    return S, pack(Z, bits).T.copy()


def dequantize_checkpoint(qweight, qzeros, scales16, g_idx, bits):
    """Exact dequantized weight [n_out, n_in] of the checkpoint form (float64).

    [ch5 §5.1.1]: x_hat = s * (q - z), per weight with its group's half-precision scale
    and packed zero point (the layout of :func:`export_tensors`):
    W_hat[o, c] = scales16[g_idx[c], o] * (code[o, c] - zero[g_idx[c], o]).
    """
    g = np.asarray(g_idx, dtype=np.int64)
    n_in = g.shape[0]
    S = np.asarray(scales16, dtype=np.float16).astype(np.float64)
    n_out = S.shape[1]
    Z = unpack(np.asarray(qzeros).T, bits, n_out)  # [G, n_out]
    codes = unpack(qweight, bits, n_in)
    return S[g, :].T * (codes - Z[g, :].T)


def round16(A, dtype):
    """Round to the nearest 16-bit value ("float16" or "bfloat16"), ties to even; returned
    as float64.  The operand precision of a 16-bit tensor-core multiply."""
    A = np.asarray(A, dtype=np.float64)
    if dtype == "float16":
        return A.astype(np.float16).astype(np.float64)
    import torch  # the bfloat16 conversion of plain PyTorch on the CPU
    return torch.from_numpy(A).to(torch.bfloat16).to(torch.float64).numpy()


def quantized_linear(X, What16):
    """Y = X W^T in float64 (X [M, n_in] 16-bit values, What16 the rounded weight)."""
    return np.asarray(X, np.float64) @ np.asarray(What16, np.float64).T


def dequantize(qweight, scales, zeros, g_idx, bits, n_in):
    """W_hat[o, c] = scales[g_idx[c], o] * (code[o, c] - zeros[g_idx[c], o])."""
    codes = unpack(qweight, bits, n_in)
    g = np.asarray(g_idx, dtype=np.int64)
    S = np.asarray(scales, dtype=np.float32).astype(np.float64)
    Z = np.asarray(zeros, dtype=np.int64)
    return S[g, :].T * (codes - Z[g, :].T)


# --------------------------------------------------------------------------- losses
def layer_loss(W, What, X):
    """||(W - W_hat) X||^2 with X = [tokens, n_in]   [ch5 §5.1.4]."""
    D = np.asarray(W, np.float64) - np.asarray(What, np.float64)
    Y = D @ np.asarray(X, np.float64).T
    return float(np.sum(Y * Y))


def layer_loss_h(W, What, H):
    """The same loss through H = 2 X^T X: 1/2 * sum_rows D H D^T."""
    D = np.asarray(W, np.float64) - np.asarray(What, np.float64)
    return float(0.5 * np.einsum("ri,ij,rj->", D, np.asarray(H, np.float64), D))


def brute_force_min_loss(w, H, scale, zero, bits):
    """Minimum of 1/2 d H d^T over every code vector of one row on a fixed grid.

    [ch5 §5.1.8]: the exact problem is a quadratic over integer grid points
    (16^n choices at 4 bits), which GPTQ solves greedily; enumeration is
    possible only for tiny n.  Returns (min loss, argmin codes).
    """
    w = np.asarray(w, np.float64)
    n = w.shape[0]
    levels = 2**bits
    grid = np.stack(np.meshgrid(*([np.arange(levels)] * n), indexing="ij"), -1).reshape(-1, n)
    vals = float(np.float32(scale)) * (grid - int(zero)).astype(np.float64)
    D = w[None, :] - vals
    loss = 0.5 * np.einsum("ki,ij,kj->k", D, np.asarray(H, np.float64), D)
    k = int(np.argmin(loss))
    return float(loss[k]), grid[k]
