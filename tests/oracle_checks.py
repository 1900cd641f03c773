"""Checks of a GPU result against the CPU oracle on every row of a layer, in
row chunks so that the fp64 references of a full-size layer never sit in host
memory at once.  Expected values come only from the oracle."""
import numpy as np

import oracle

import helpers


def linear_all_rows(y_bits, inp, skip=False, act=None, rows=None, chunk=512):
    """Compare Y (bf16 bits [M,N], or only `rows` of it) with the oracle's
    Y = S(X) W^T + bias + (X A^T) B^T (act: None or "gelu_tanh").

    Returns (worst, fro): the largest ratio of |dY| to the elementwise bound
    2e-2 * ||S(X)_m||_2 * ||W_n||_2, and the relative Frobenius error, both over
    all compared rows (with GELU, the bound and the Frobenius norm of the
    pre-activation reference are scaled by GELU's largest slope, 1.13)."""
    X, W = inp["X"], inp["W"]
    M = X.shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    w = helpers.f32(W).astype(np.float64)
    wn = np.linalg.norm(w, axis=1)
    slope = 1.13 if act == "gelu_tanh" else 1.0
    worst, err2, ref2 = 0.0, 0.0, 0.0
    for c0 in range(0, len(rows), chunk):
        rr = rows[c0:c0 + chunk]
        y_pre, _, sx = oracle.linear(X[rr], W, inp["bias"], inp["A"], inp["B"], skip=skip,
                                     want_sx=True)
        y_ref = oracle.gelu_tanh(y_pre) if act == "gelu_tanh" else y_pre
        y = helpers.f32(y_bits[rr] if y_bits.shape[0] == M else y_bits[c0:c0 + chunk]) \
            .astype(np.float64)
        bound = slope * 2e-2 * np.outer(np.linalg.norm(sx, axis=1), wn)
        d = np.abs(y - y_ref)
        worst = max(worst, float((d / np.maximum(bound, 1e-30)).max()))
        err2 += float(np.sum(d * d))
        ref2 += float(np.sum(y_pre * y_pre))
    fro = np.sqrt(err2) / max(np.sqrt(ref2), 1e-30) / slope
    return worst, fro
