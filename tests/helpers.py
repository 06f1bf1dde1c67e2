"""Shared test helpers: inputs to torch, and the tolerance bounds the parity
tests use (each derived from the arithmetic the kernels do in fp32)."""
import numpy as np

import oracle
from clustered_sparse_attention_b200 import synth

U32 = 2.0 ** -24   # fp32 unit roundoff


def to_torch(x_f32, dtype, device="cuda"):
    """float32 numpy (values already on the bf16 grid for bf16) -> torch."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x_f32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)   # exact: the values are on the bf16 grid
    return t.to(device)


def workload_tensors(w, heads=None, step=0):
    return {n: synth.layer_tensor(w, n, step=step, heads=heads) for n in ("q", "k", "v")}


def np64(t):
    import torch
    return t.detach().to("cpu", torch.float64).numpy()


def check_assign(X, cent, labels_gpu):
    """Labels must equal the fp64 argmin (lowest index on ties) except where
    the GPU's choice is within the fp32 rounding band of the best distance:
    |c|^2 - 2x.c in fp32 errs by at most ~d*u*(|x|^2 + |c|^2) per candidate.
    Returns the number of accepted near-tie flips."""
    X = np.asarray(X, np.float64)
    cent = np.asarray(cent, np.float64)
    lab_o, _, best, _ = oracle.assign(X, cent)
    bad = np.nonzero(lab_o != labels_gpu)[0]
    d = X.shape[1]
    for t in bad:
        g = int(labels_gpu[t])
        assert 0 <= g < cent.shape[0], "label out of range at token %d" % t
        dg = float(((X[t] - cent[g]) ** 2).sum())
        band = 8 * d * U32 * (float(X[t] @ X[t]) + float(cent[lab_o[t]] @ cent[lab_o[t]])
                              + float(cent[g] @ cent[g]))
        assert dg - best[t] <= band, (
            "token %d: gpu label %d (dist %.9g) vs oracle %d (dist %.9g), band %.3g"
            % (t, g, dg, lab_o[t], best[t], band))
    return len(bad)


def update_tolerance(X, labels, C):
    """Per-element bound for fp32 segment means: (n/R + R) u * mean|x| with
    R = 8 row groups, plus one rounding of the quotient."""
    X = np.asarray(X, np.float64)
    n = np.bincount(labels, minlength=C).astype(np.float64)
    sabs = np.zeros((C, X.shape[1]))
    np.add.at(sabs, labels, np.abs(X))
    mean_abs = sabs / np.maximum(n, 1)[:, None]
    return (n[:, None] / 8 + 40) * U32 * mean_abs * 2 + 1e-30


def probe_tolerance(qbar, Kp, E, S, scale, P=None):
    """|dE| <= 2.5 k sqrt(E S) + k^2 S + 1e-5 P, with k the relative error of
    the fp32 weights e^{s-m}: twice the dot-product bound d u scale |q||k|_max
    plus the exp rounding.  The last term bounds the fp32 evaluation and
    summation of the per-key terms: the kernel evaluates each term expanded
    around v_t - vbar_c, whose parts can differ in sign, so the bound is on
    the sum of their magnitudes P (>= E); with all terms non-negative (the
    value-free error) P = E."""
    qbar = np.asarray(qbar, np.float64)
    kmax = float(np.sqrt((np.asarray(Kp, np.float64) ** 2).sum(1).max()))
    d = qbar.shape[1]
    kappa = 2 * d * U32 * scale * np.sqrt((qbar ** 2).sum(1)) * kmax + 4e-7
    kappa = kappa[:, None]
    P = E if P is None else P
    return 2.5 * kappa * np.sqrt(E * S) + kappa ** 2 * S + 1e-5 * P + 1e-37
