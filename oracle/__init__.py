"""CPU oracle for the clustered sparse attention layer -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It never touches the CUDA library and shares
no code with it.  Every routine is plain fp64 C (``svgear_oracle.c``), each
citing the passage of the pages it follows; this module only marshals numpy
arrays and composes the steps in the pages' order:

  k-means++ seeding -> iters x (assign, update) -> stable sort by label
  (permutation + segment offsets) -> value centroids -> compensation-error
  probe -> greedy error-to-cost routing -> exact blocks + centroid
  compensation, written back in the original token order.

Parity status of each routine is pinned by ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, u64, f64, f32 = (ctypes.c_int64, ctypes.c_int, ctypes.c_uint64,
                                   ctypes.c_double, ctypes.c_float)
        L.orc_philox4x64_10.argtypes = [P, P, P]
        L.orc_uniform.argtypes = [u64, u64, u64]
        L.orc_uniform.restype = f64
        L.orc_kmeanspp.argtypes = [P, i64, i32, i32, u64, u64, P, P, P]
        L.orc_assign.argtypes = [P, i64, i32, P, i32, P, P, P, P]
        L.orc_update.argtypes = [P, i64, i32, P, i32, P, P]
        L.orc_stable_sort.argtypes = [P, i64, i32, P, P]
        L.orc_segment_mean.argtypes = [P, i32, P, i32, P, P]
        L.orc_probe.argtypes = [P, i32, P, P, i64, i32, P, P, P, i32, f64, P, P, P]
        L.orc_route.argtypes = [P, P, i32, P, i32, i64, f32, P, P]
        L.orc_route_budgets.argtypes = [P, P, i32, P, i32, P, P, P]
        L.orc_topp_budget.argtypes = [P, i32, P, i32, i32, P, P, f64, f64, P, P]
        L.orc_attend.argtypes = [P, i64, P, P, i32, P, i32, P, i32, P, P, P, P,
                                 P, f64, P, i64, P, P, P, f64]
        L.orc_segment_var.argtypes = [P, i32, P, i32, P]
        L.orc_probe_value_free.argtypes = [P, i32, P, i64, i32, P, P, i32, f64, P]
        L.orc_diagnostics.argtypes = [P, P, P, i64, i32, P, i32, P, i32, P, P, P, P, f64, P,
                                      i64, P, P, P]
        L.orc_num_threads.restype = i32
        _lib = L
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def philox4x64_10(counter, key) -> np.ndarray:
    c = np.ascontiguousarray(counter, dtype=np.uint64)
    k = np.ascontiguousarray(key, dtype=np.uint64)
    out = np.zeros(4, dtype=np.uint64)
    lib().orc_philox4x64_10(_p(c), _p(k), _p(out))
    return out


def uniform(seed: int, stream: int, j: int) -> float:
    return float(lib().orc_uniform(seed, stream, j))


def kmeanspp(X, C: int, seed: int, stream: int, follow=None):
    """k-means++ seed token indices [C]; with ``follow`` also the margins."""
    X = _f64(X)
    N, d = X.shape
    idx = np.zeros(C, dtype=np.int32)
    margin = np.zeros(C, dtype=np.float64)
    fol = None if follow is None else _i32(follow)
    lib().orc_kmeanspp(_p(X), N, d, C, seed, stream, _p(fol), _p(idx), _p(margin))
    return idx, margin


def assign(X, cent):
    """labels, runner-up, best distance, gap (fp64 direct form)."""
    X, cent = _f64(X), _f64(cent)
    N, d = X.shape
    C = cent.shape[0]
    labels = np.zeros(N, dtype=np.int32)
    second = np.zeros(N, dtype=np.int32)
    best = np.zeros(N)
    gap = np.zeros(N)
    lib().orc_assign(_p(X), N, d, _p(cent), C, _p(labels), _p(second), _p(best), _p(gap))
    return labels, second, best, gap


def update(X, labels, prev):
    X, prev = _f64(X), _f64(prev)
    labels = _i32(labels)
    N, d = X.shape
    C = prev.shape[0]
    out = np.zeros((C, d))
    lib().orc_update(_p(X), N, d, _p(labels), C, _p(prev), _p(out))
    return out


def stable_sort(labels, C: int):
    labels = _i32(labels)
    N = labels.shape[0]
    perm = np.zeros(N, dtype=np.int32)
    off = np.zeros(C + 1, dtype=np.int32)
    lib().orc_stable_sort(_p(labels), N, C, _p(perm), _p(off))
    return perm, off


def segment_mean(Xp, offsets, prev=None):
    Xp = _f64(Xp)
    off = _i32(offsets)
    C = off.shape[0] - 1
    d = Xp.shape[1]
    out = np.zeros((C, d))
    pv = None if prev is None else _f64(prev)
    lib().orc_segment_mean(_p(Xp), d, _p(off), C, _p(pv), _p(out))
    return out


def probe(qbar, Kp, Vp, kbar, vbar, k_off, scale: float, with_scale=False, with_parts=False):
    """Probe errors E [Cq, Ck]; with_scale adds the error scale S, with_parts
    also P (the bound on the terms of the error expanded around v_t - vbar_c);
    S and P serve tolerance bounds only."""
    qbar, Kp, Vp, kbar, vbar = map(_f64, (qbar, Kp, Vp, kbar, vbar))
    k_off = _i32(k_off)
    Cq, d = qbar.shape
    Ck = kbar.shape[0]
    E = np.zeros((Cq, Ck))
    S = np.zeros((Cq, Ck)) if (with_scale or with_parts) else None
    P = np.zeros((Cq, Ck)) if with_parts else None
    lib().orc_probe(_p(qbar), Cq, _p(Kp), _p(Vp), Kp.shape[0], d, _p(kbar), _p(vbar),
                    _p(k_off), Ck, float(scale), _p(E), _p(S), _p(P))
    if with_parts:
        return E, S, P
    return (E, S) if with_scale else E


def probe_value_free(qbar, Kp, kbar, k_off, scale: float):
    """Value-free probe error Ehat [Cq, Ck] (the probe without the values)."""
    qbar, Kp, kbar = map(_f64, (qbar, Kp, kbar))
    k_off = _i32(k_off)
    Cq, d = qbar.shape
    Ck = kbar.shape[0]
    E = np.zeros((Cq, Ck))
    lib().orc_probe_value_free(_p(qbar), Cq, _p(Kp), Kp.shape[0], d, _p(kbar), _p(k_off), Ck,
                               float(scale), _p(E))
    return E


def diagnostics(Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, O_sparse, q_perm, scale: float,
                rows):
    """Attention recall, |O_sparse - O_dense|^2 and |O_dense|^2 of the query
    rows ``rows`` (permuted positions); O_sparse in the original order."""
    Qp, Kp, Vp, O_sparse = map(_f64, (Qp, Kp, Vp, O_sparse))
    q_off, k_off, pair_off, q_perm = map(_i32, (q_off, k_off, pair_off, q_perm))
    pair_kc = _i32(pair_kc if len(pair_kc) else np.zeros(1, np.int32))
    r = np.ascontiguousarray(rows, dtype=np.int64)
    n = r.shape[0]
    recall, err2, ref2 = np.zeros(n), np.zeros(n), np.zeros(n)
    lib().orc_diagnostics(_p(Qp), _p(Kp), _p(Vp), Kp.shape[0], Qp.shape[1], _p(q_off),
                          q_off.shape[0] - 1, _p(k_off), k_off.shape[0] - 1, _p(pair_off),
                          _p(pair_kc), _p(O_sparse), _p(q_perm), float(scale), _p(r), n,
                          _p(recall), _p(err2), _p(ref2))
    return recall, err2, ref2


def route(E, q_off, k_off, Nk: int, density: float, budgets=None):
    """pair_off [Cq+1], pair_kc [nnz] from fp32 errors E [Cq, Ck]; the budget
    is floor(density * Nk) keys per query cluster, or budgets[i] when given."""
    E = np.ascontiguousarray(E, dtype=np.float32)
    q_off, k_off = _i32(q_off), _i32(k_off)
    Cq, Ck = E.shape
    pair_off = np.zeros(Cq + 1, dtype=np.int32)
    pair_kc = np.zeros(max(1, Cq * Ck), dtype=np.int32)
    if budgets is None:
        lib().orc_route(_p(E), _p(q_off), Cq, _p(k_off), Ck, int(Nk),
                        ctypes.c_float(density), _p(pair_off), _p(pair_kc))
    else:
        b = np.ascontiguousarray(budgets, dtype=np.int64)
        assert b.shape == (Cq,)
        lib().orc_route_budgets(_p(E), _p(q_off), Cq, _p(k_off), Ck, _p(b), _p(pair_off),
                                _p(pair_kc))
    return pair_off, pair_kc[:pair_off[-1]].copy()


def topp_budget(qbar, kbar, q_off, k_off, p: float, scale: float):
    """Per query cluster: keys of the key clusters holding p of the estimated
    weight P' (budget int64 [Cq]) and the distance of the crossing from p
    (margin float64 [Cq])."""
    qbar, kbar = _f64(qbar), _f64(kbar)
    q_off, k_off = _i32(q_off), _i32(k_off)
    Cq, d = qbar.shape
    Ck = kbar.shape[0]
    budget = np.zeros(Cq, dtype=np.int64)
    margin = np.zeros(Cq)
    lib().orc_topp_budget(_p(qbar), Cq, _p(kbar), Ck, d, _p(q_off), _p(k_off), float(p),
                          float(scale), _p(budget), _p(margin))
    return budget, margin


def segment_var(Xp, offsets):
    """Per-coordinate population variance of every segment [C, d] (0 if empty)."""
    Xp = _f64(Xp)
    offsets = _i32(offsets)
    C = offsets.shape[0] - 1
    out = np.zeros((C, Xp.shape[1]))
    lib().orc_segment_var(_p(Xp), Xp.shape[1], _p(offsets), C, _p(out))
    return out


def attend(Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, kbar, vbar, q_perm,
           scale: float, rows=None, kvar=None, lam: float = 0.0):
    """O (original token order) and lse; with ``rows`` (permuted positions),
    only those rows, in the order given.  With ``kvar`` (per-coordinate key
    variance of every key cluster) a skipped cluster's log-weight gains
    lam * scale^2 / 2 * sum_k q_k^2 kvar[c][k]."""
    Qp, Kp, Vp, kbar, vbar = map(_f64, (Qp, Kp, Vp, kbar, vbar))
    kv = None if kvar is None else _f64(kvar)
    q_off, k_off, pair_off, q_perm = map(_i32, (q_off, k_off, pair_off, q_perm))
    pair_kc = _i32(pair_kc if len(pair_kc) else np.zeros(1, np.int32))
    Nq, d = Qp.shape
    Cq, Ck = q_off.shape[0] - 1, k_off.shape[0] - 1
    if rows is None:
        O = np.zeros((Nq, d))
        lse = np.zeros(Nq)
        r, nr = None, 0
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        nr = r.shape[0]
        O = np.zeros((nr, d))
        lse = np.zeros(nr)
    lib().orc_attend(_p(Qp), Nq, _p(Kp), _p(Vp), d, _p(q_off), Cq, _p(k_off), Ck,
                     _p(pair_off), _p(pair_kc), _p(kbar), _p(vbar), _p(q_perm),
                     float(scale), _p(r), nr, _p(O), _p(lse), _p(kv), float(lam))
    return O, lse


# -------------------------------------------------------------------------
# Composition of the steps, in the pages' order.
# -------------------------------------------------------------------------
def cluster(X, C: int, iters: int, seed: int, stream: int, warm=None):
    """k-means (k-means++ or warm centroids, then ``iters`` rounds of assign +
    update), then the stable sort by final label.  The last round's labels
    are the final labels and its update gives the returned centroids, so
    every non-empty centroid is the mean of its final members."""
    X = _f64(X)
    if iters < 1:
        raise ValueError("iters must be >= 1")
    if warm is None:
        idx, _ = kmeanspp(X, C, seed, stream)
        cent = X[idx].copy()
    else:
        cent = _f64(warm).copy()
    labels = None
    for _ in range(iters):
        labels, _, _, _ = assign(X, cent)
        cent = update(X, labels, cent)
    perm, off = stable_sort(labels, C)
    return {"labels": labels, "perm": perm, "offsets": off, "centroids": cent,
            "Xp": X[perm]}


def layer(Q, K, V, Cq: int, Ck: int, iters: int, density: float, scale: float,
          seed_q: int, seed_k: int, stream: int, warm_q=None, warm_k=None, topp=None):
    """One head of the layer, every intermediate returned; with topp=p the
    routing budget per query cluster is topp_budget's (density unused)."""
    cq = cluster(Q, Cq, iters, seed_q, stream, warm_q)
    ck = cluster(K, Ck, iters, seed_k, stream, warm_k)
    Vp = _f64(V)[ck["perm"]]
    vbar = segment_mean(Vp, ck["offsets"])
    E = probe(cq["centroids"], ck["Xp"], Vp, ck["centroids"], vbar, ck["offsets"], scale)
    budgets = None
    if topp is not None:
        budgets, _ = topp_budget(cq["centroids"], ck["centroids"], cq["offsets"], ck["offsets"],
                                 topp, scale)
    pair_off, pair_kc = route(E.astype(np.float32), cq["offsets"], ck["offsets"],
                              K.shape[0], density if topp is None else 1.0, budgets=budgets)
    O, lse = attend(cq["Xp"], ck["Xp"], Vp, cq["offsets"], ck["offsets"], pair_off,
                    pair_kc, ck["centroids"], vbar, cq["perm"], scale)
    return {"q": cq, "k": ck, "Vp": Vp, "vbar": vbar, "E": E, "pair_off": pair_off,
            "pair_kc": pair_kc, "O": O, "lse": lse, "budgets": budgets}
