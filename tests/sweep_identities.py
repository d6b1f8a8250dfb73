"""Per-decision check of a GPTQ sweep's outputs against the identities that define it.

Given the factor U (upper, inverse(H_d) = U^T U, sweep order) and a row's weights W, the
sweep of ch5 §5.1.8 is fully characterised column by column: with the normalised errors
err defined by W - W_hat = err U (the compensation identity, solved as a triangular
system), the current value of column j when the sweep reaches it is
    w_cur_j = W_j - sum_{k<j} err_k U_kj = W_hat_j + err_j U_jj,
and every code must be the quantizer's code of w_cur_j under its group's parameters;
every non-static group's parameters must be the quantizer's parameters of that group's
current weights at its first column, W[:, group] - err[:, :j0] U[:j0, group].  By
induction over the columns, outputs that pass every decision are exactly the sweep's
outputs under U; a decision that fails is counted where it happens, without cascading
into the later columns (those are checked against the outputs' own history).

Used where the oracle cannot afford its own factor (order 28672); tests/test_oracle_pins.py
pins it on the oracle's outputs and on a mistake planted in the oracle.
"""

import numpy as np
from scipy.linalg import solve_triangular

import oracle as O


def sweep_decisions(W, What, codes, scales, zeros, U, bits, sym, group_size):
    """Fractions of (group parameters, codes) consistent with the sweep under U.

    W, What, codes: [rows, n] in sweep order (no act order); scales, zeros: [G, rows]
    (non-static groups of group_size consecutive columns)."""
    W = np.asarray(W, np.float64)
    What = np.asarray(What, np.float64)
    n = W.shape[1]
    g = group_size
    err = solve_triangular(U, (W - What).T, trans="T", lower=False).T
    p_ok = []
    for k in range(n // g):
        j0 = k * g
        cur = W[:, j0:j0 + g] - err[:, :j0] @ U[:j0, j0:j0 + g]
        s, z = O.quant_params(cur, bits, sym)
        p_ok.append((np.abs(scales[k] - s) <= 1e-3 * np.abs(s)) & (zeros[k] == z))
    cur_all = What + err * np.diag(U)[None, :]
    q_ref = np.empty_like(codes)
    for k in range(n // g):
        cols = slice(k * g, (k + 1) * g)
        q_ref[:, cols], _ = O.quantize(cur_all[:, cols], np.asarray(scales[k])[:, None],
                                       np.asarray(zeros[k], np.int64)[:, None], bits)
    return float(np.mean(p_ok)), float(np.mean(codes == q_ref))
