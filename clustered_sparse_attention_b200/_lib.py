"""ctypes binding of libsvgear.so (include/svgear.h).

Argument marshalling only: every step runs in the library's CUDA kernels on
torch's current stream.  Output and workspace buffers are allocated with
torch (device memory plumbing); the library itself never allocates.  There
is no CPU path: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsvgear.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = 0, -1, -2, -3, -4, -5
ERR_SCRATCH_LIMIT = -6
ERR_TMEM_LOST = -7
NOALLOC_SORT_SCRATCH_INTS = 2 * 1024 * 1024
F32, BF16 = 0, 1
OP_CLUSTER, OP_KMEANSPP, OP_LABEL_SORT, OP_KMEANS_UPDATE, OP_ROUTE, OP_ATTEND = range(6)
OP_KMEANS_ASSIGN = 6
OP_ROUTE_TOPP = 7
OP_CENTROIDS = 8
MAX_CLUSTERS = 4096

EXPORTED = ("svgear_cluster", "svgear_kmeanspp_init", "svgear_kmeans_assign",
            "svgear_label_sort", "svgear_kmeans_update", "svgear_permute",
            "svgear_centroids", "svgear_probe", "svgear_route_select", "svgear_route",
            "svgear_attend", "svgear_workspace_bytes", "svgear_status_string",
            "svgear_version", "svgear_kernel_launches", "svgear_attend_status",
            "svgear_device_status", "svgear_topp_budget", "svgear_route_select_budget",
            "svgear_route_topp", "svgear_key_variance", "svgear_attend_var",
            "svgear_probe_value_free", "svgear_diagnostics",
            "svgear_label_sort_noalloc", "svgear_selftest_wait", "svgear_layer",
            "svgear_layer_host", "svgear_layer_workspace_bytes")


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class LayerParams(ctypes.Structure):
    _fields_ = [("Cq", ctypes.c_int32), ("Ck", ctypes.c_int32), ("iters", ctypes.c_int32),
                ("density", ctypes.c_float), ("topp", ctypes.c_float), ("scale", ctypes.c_float),
                ("var_lambda", ctypes.c_float), ("seed", ctypes.c_uint64)]


class SvgearError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__("%s failed: %s (%d)" % (fn, msg, status))
        self.status = status


_L = None


def lib():
    """Load libsvgear.so; raises if it has not been built."""
    global _L
    if _L is not None:
        return _L
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libsvgear.so is not built (run clustered_sparse_attention_b200/build.py"
                           " or __graft_entry__.build()); there is no fallback path")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, U64, F, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_float,
                          ctypes.c_size_t)
    sig = {
        "svgear_cluster": [P, Dims, I32, I32, P, U64, P, P, P, P, P, P, SZ, P],
        "svgear_kmeanspp_init": [P, Dims, I32, U64, P, P, P, SZ, P],
        "svgear_kmeans_assign": [P, Dims, P, I32, P, P, SZ, P],
        "svgear_label_sort": [P, Dims, I32, P, P, P, SZ, P],
        "svgear_kmeans_update": [P, Dims, P, I32, P, P, SZ, P],
        "svgear_permute": [P, P, Dims, P, P],
        "svgear_centroids": [P, P, I32, Dims, P, P, SZ, P],
        "svgear_probe": [P, I32, P, P, P, P, P, I32, Dims, F, P, P, SZ, P],
        "svgear_route_select": [P, P, I32, P, I32, I32, I32, I32, F, P, P, P, SZ, P],
        "svgear_route": [P, P, I32, P, P, P, I32, P, P, Dims, F, F, P, P, P, P, SZ, P],
        "svgear_topp_budget": [P, P, I32, P, P, I32, I32, I32, I32, I32, F, F, P, P],
        "svgear_route_select_budget": [P, P, I32, P, I32, I32, I32, I32, P, P, P, P, SZ, P],
        "svgear_route_topp": [P, P, I32, P, P, P, I32, P, P, Dims, F, F, P, P, P, P, P, SZ, P],
        "svgear_key_variance": [P, P, I32, Dims, P, P],
        "svgear_probe_value_free": [P, I32, P, P, P, I32, Dims, F, P, P, SZ, P],
        "svgear_diagnostics": [P, P, P, Dims, I32, P, I32, P, I32, P, P, P, P, F, P, I32, P, P, P,
                               P],
        "svgear_attend_var": [P, P, P, Dims, I32, P, I32, P, I32, P, P, P, P, P, F, P, F, P, P, SZ,
                              P],
        "svgear_attend": [P, P, P, Dims, I32, P, I32, P, I32, P, P, P, P, P, F, P, P, SZ, P],
        "svgear_workspace_bytes": [I32, Dims, I32, I32],
        "svgear_status_string": [ctypes.c_int],
        "svgear_version": [],
        "svgear_kernel_launches": [],
        "svgear_attend_status": [P, SZ, P, P],
        "svgear_device_status": [P, SZ, P, P],
        "svgear_label_sort_noalloc": [P, Dims, I32, P, P, P],
        "svgear_selftest_wait": [P, SZ, I32, I32, I32, P],
        "svgear_layer": [P, P, P, Dims, ctypes.POINTER(LayerParams), P, P, P, P, P, P, SZ, P, P],
        "svgear_layer_host": [P, P, P, Dims, ctypes.POINTER(LayerParams), P, P, P, P, P, P, SZ,
                              P],
        "svgear_layer_workspace_bytes": [Dims, ctypes.POINTER(LayerParams), I32],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    L.svgear_workspace_bytes.restype = SZ
    L.svgear_layer_workspace_bytes.restype = SZ
    L.svgear_status_string.restype = ctypes.c_char_p
    L.svgear_kernel_launches.restype = ctypes.c_uint64
    _L = L
    return L


def kernel_launches() -> int:
    """Kernels the library has launched since it was loaded."""
    return int(lib().svgear_kernel_launches())


def _check(fn, status):
    if status != OK:
        raise SvgearError(fn, status, lib().svgear_status_string(status).decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("token tensors must be float32 or bfloat16, got %s" % t.dtype)


def _tokens(t, name):
    if not (t.is_cuda and t.dim() == 4 and t.is_contiguous()):
        raise ValueError("%s must be a contiguous CUDA tensor [B, H, N, d]" % name)
    B, H, N, d = t.shape
    return Dims(B, H, N, d, _dtype_code(t))


def _cuda(t, name, dtype):
    if not (t.is_cuda and t.is_contiguous() and t.dtype == dtype):
        raise ValueError("%s must be a contiguous CUDA %s tensor" % (name, dtype))
    return t


def workspace_bytes(op, dims, c1, c2=0):
    return int(lib().svgear_workspace_bytes(op, dims, c1, c2))


def _workspace(op, dims, c1, c2, device):
    # A zero answer means the sizes are invalid: pass a token buffer and let
    # the entry point report the precise status.
    n = max(workspace_bytes(op, dims, c1, c2), 256)
    return torch.empty(n, dtype=torch.uint8, device=device), n


@dataclass
class Clustering:
    labels: torch.Tensor      # int32 [B, H, N]
    perm: torch.Tensor        # int32 [B, H, N]
    offsets: torch.Tensor     # int32 [B, H, C+1]
    centroids: torch.Tensor   # float32 [B, H, C, d]
    Xp: torch.Tensor | None   # [B, H, N, d] permuted copy


def device_status(ws, n=None):
    """The four device status words of the call that used workspace `ws`
    (synchronises the current stream): [status, wait site * 65536 + index,
    CTA, 1 if the device's tensor memory is lost else 0]."""
    n = ws.numel() * ws.element_size() if n is None else n
    st = (ctypes.c_int32 * 4)()
    _check("svgear_device_status", lib().svgear_device_status(_ptr(ws), n, st, _stream()))
    return [int(x) for x in st]


def _device_status(fn, ws, n):
    """Synchronise and raise if a bounded wait inside a tensor-core kernel of
    the call that used `ws` gave up, or the kernel refused to start because
    the device's tensor memory was lost earlier."""
    st = device_status(ws, n)
    if st[0] != OK:
        raise SvgearError("%s (device: wait site %d, index %d, cta %d, tensor memory lost %d)"
                          % (fn, st[1] >> 16, st[1] & 0xFFFF, st[2], st[3]), st[0],
                          lib().svgear_status_string(st[0]).decode())


def selftest_wait(arrive, timeout_us, mark_lost=False):
    """Run the library's bounded device wait on its own (svgear_selftest_wait)
    and return the device status words (device_status)."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    _check("svgear_selftest_wait", lib().svgear_selftest_wait(
        _ptr(ws), ws.numel(), int(bool(arrive)), int(timeout_us), int(bool(mark_lost)), _stream()))
    return device_status(ws)


def svgear_cluster(X, C, iters, warm_centroids=None, seed=0, permuted=True, out=None,
                   check_status=False):
    """check_status=True synchronises and raises if a bounded wait inside the
    assignment kernel gave up."""
    dims = _tokens(X, "X")
    B, H, N, d = X.shape
    dev = X.device
    if out is None:
        out = Clustering(
            torch.empty((B, H, N), dtype=torch.int32, device=dev),
            torch.empty((B, H, N), dtype=torch.int32, device=dev),
            torch.empty((B, H, C + 1), dtype=torch.int32, device=dev),
            torch.empty((B, H, C, d), dtype=torch.float32, device=dev),
            torch.empty_like(X) if permuted else None)
    if warm_centroids is not None:
        _cuda(warm_centroids, "warm_centroids", torch.float32)
    ws, n = _workspace(OP_CLUSTER, dims, C, 0, dev)
    _check("svgear_cluster", lib().svgear_cluster(
        _ptr(X), dims, C, iters, _ptr(warm_centroids), seed, _ptr(out.labels), _ptr(out.perm),
        _ptr(out.offsets), _ptr(out.centroids), _ptr(out.Xp), _ptr(ws), n, _stream()))
    if check_status:
        _device_status("svgear_cluster", ws, n)
    return out


def svgear_kmeanspp_init(X, C, seed=0):
    dims = _tokens(X, "X")
    B, H, N, d = X.shape
    cent = torch.empty((B, H, C, d), dtype=torch.float32, device=X.device)
    idx = torch.empty((B, H, C), dtype=torch.int32, device=X.device)
    ws, n = _workspace(OP_KMEANSPP, dims, C, 0, X.device)
    _check("svgear_kmeanspp_init", lib().svgear_kmeanspp_init(
        _ptr(X), dims, C, seed, _ptr(cent), _ptr(idx), _ptr(ws), n, _stream()))
    return cent, idx


def svgear_kmeans_assign(X, centroids, check_status=False):
    dims = _tokens(X, "X")
    _cuda(centroids, "centroids", torch.float32)
    B, H, N, d = X.shape
    C = centroids.shape[2]
    labels = torch.empty((B, H, N), dtype=torch.int32, device=X.device)
    ws, n = _workspace(OP_KMEANS_ASSIGN, dims, C, 0, X.device)
    _check("svgear_kmeans_assign", lib().svgear_kmeans_assign(
        _ptr(X), dims, _ptr(centroids), C, _ptr(labels), _ptr(ws), n, _stream()))
    if check_status:
        _device_status("svgear_kmeans_assign", ws, n)
    return labels


def svgear_label_sort(labels, C):
    _cuda(labels, "labels", torch.int32)
    B, H, N = labels.shape
    dims = Dims(B, H, N, 64, F32)
    perm = torch.empty_like(labels)
    off = torch.empty((B, H, C + 1), dtype=torch.int32, device=labels.device)
    ws, n = _workspace(OP_LABEL_SORT, dims, C, 0, labels.device)
    _check("svgear_label_sort", lib().svgear_label_sort(
        _ptr(labels), dims, C, _ptr(perm), _ptr(off), _ptr(ws), n, _stream()))
    return perm, off


def svgear_kmeans_update(X, labels, centroids):
    """Returns a new tensor: member means, previous rows for empty clusters."""
    dims = _tokens(X, "X")
    _cuda(labels, "labels", torch.int32)
    out = _cuda(centroids, "centroids", torch.float32).clone()
    C = centroids.shape[2]
    ws, n = _workspace(OP_KMEANS_UPDATE, dims, C, 0, X.device)
    _check("svgear_kmeans_update", lib().svgear_kmeans_update(
        _ptr(X), dims, _ptr(labels), C, _ptr(out), _ptr(ws), n, _stream()))
    return out


def svgear_permute(X, perm):
    dims = _tokens(X, "X")
    _cuda(perm, "perm", torch.int32)
    Xp = torch.empty_like(X)
    _check("svgear_permute", lib().svgear_permute(_ptr(X), _ptr(perm), dims, _ptr(Xp), _stream()))
    return Xp


def svgear_centroids(Xp, offsets, C=None):
    dims = _tokens(Xp, "Xp")
    _cuda(offsets, "offsets", torch.int32)
    C = offsets.shape[-1] - 1 if C is None else C
    B, H, N, d = Xp.shape
    out = torch.empty((B, H, C, d), dtype=torch.float32, device=Xp.device)
    ws, n = _workspace(OP_CENTROIDS, dims, C, 0, Xp.device)
    _check("svgear_centroids", lib().svgear_centroids(
        _ptr(Xp), _ptr(offsets), C, dims, _ptr(out), _ptr(ws), n, _stream()))
    return out


def svgear_probe(qbar, Kp, Vp, kbar, vbar, k_off, scale):
    kd = _tokens(Kp, "Kp")
    _tokens(Vp, "Vp")
    B, H, Cq, d = qbar.shape
    Ck = kbar.shape[2]
    E = torch.empty((B, H, Cq, Ck), dtype=torch.float32, device=Kp.device)
    ws, n = _workspace(OP_ROUTE, kd, Cq, Ck, Kp.device)
    _check("svgear_probe", lib().svgear_probe(
        _ptr(qbar), Cq, _ptr(Kp), _ptr(Vp), _ptr(kbar), _ptr(vbar), _ptr(k_off), Ck, kd,
        float(scale), _ptr(E), _ptr(ws), n, _stream()))
    return E


def svgear_route_select(E, q_off, k_off, Nk, density):
    _cuda(E, "E", torch.float32)
    B, H, Cq, Ck = E.shape
    pair_off = torch.empty((B, H, Cq + 1), dtype=torch.int32, device=E.device)
    pair_kc = torch.empty((B, H, Cq * Ck), dtype=torch.int32, device=E.device)
    ws, n = _workspace(OP_ROUTE, Dims(B, H, Nk, 64, F32), Cq, Ck, E.device)
    _check("svgear_route_select", lib().svgear_route_select(
        _ptr(E), _ptr(q_off), Cq, _ptr(k_off), Ck, B, H, Nk, float(density), _ptr(pair_off),
        _ptr(pair_kc), _ptr(ws), n, _stream()))
    return pair_off, pair_kc


def svgear_topp_budget(qbar, q_off, kbar, k_off, Nk, p, scale):
    """Keys per query cluster holding p of the estimated weight: int32 [B, H, Cq]."""
    _cuda(qbar, "qbar", torch.float32)
    _cuda(kbar, "kbar", torch.float32)
    B, H, Cq, d = qbar.shape
    Ck = kbar.shape[2]
    budget = torch.empty((B, H, Cq), dtype=torch.int32, device=qbar.device)
    _check("svgear_topp_budget", lib().svgear_topp_budget(
        _ptr(qbar), _ptr(q_off), Cq, _ptr(kbar), _ptr(k_off), Ck, B, H, d, int(Nk), float(p),
        float(scale), _ptr(budget), _stream()))
    return budget


def svgear_route_select_budget(E, q_off, k_off, Nk, budget):
    _cuda(E, "E", torch.float32)
    _cuda(budget, "budget", torch.int32)
    B, H, Cq, Ck = E.shape
    pair_off = torch.empty((B, H, Cq + 1), dtype=torch.int32, device=E.device)
    pair_kc = torch.empty((B, H, Cq * Ck), dtype=torch.int32, device=E.device)
    ws, n = _workspace(OP_ROUTE, Dims(B, H, Nk, 64, F32), Cq, Ck, E.device)
    _check("svgear_route_select_budget", lib().svgear_route_select_budget(
        _ptr(E), _ptr(q_off), Cq, _ptr(k_off), Ck, B, H, Nk, _ptr(budget), _ptr(pair_off),
        _ptr(pair_kc), _ptr(ws), n, _stream()))
    return pair_off, pair_kc


def svgear_route_topp(qbar, q_off, kbar, vbar, k_off, Kp, Vp, p, scale, return_errors=False):
    """Probe, top-p budget and greedy selection; returns (pair_off, pair_kc,
    budget[, E])."""
    kd = _tokens(Kp, "Kp")
    _tokens(Vp, "Vp")
    B, H, Cq, d = qbar.shape
    Ck = kbar.shape[2]
    dev = Kp.device
    pair_off = torch.empty((B, H, Cq + 1), dtype=torch.int32, device=dev)
    pair_kc = torch.empty((B, H, Cq * Ck), dtype=torch.int32, device=dev)
    budget = torch.empty((B, H, Cq), dtype=torch.int32, device=dev)
    E = torch.empty((B, H, Cq, Ck), dtype=torch.float32, device=dev) if return_errors else None
    ws, n = _workspace(OP_ROUTE_TOPP, kd, Cq, Ck, dev)
    _check("svgear_route_topp", lib().svgear_route_topp(
        _ptr(qbar), _ptr(q_off), Cq, _ptr(kbar), _ptr(vbar), _ptr(k_off), Ck, _ptr(Kp), _ptr(Vp),
        kd, float(p), float(scale), _ptr(pair_off), _ptr(pair_kc), _ptr(E), _ptr(budget),
        _ptr(ws), n, _stream()))
    return (pair_off, pair_kc, budget, E) if return_errors else (pair_off, pair_kc, budget)


def svgear_route(qbar, q_off, kbar, vbar, k_off, Kp, Vp, density, scale, return_errors=False):
    kd = _tokens(Kp, "Kp")
    _tokens(Vp, "Vp")
    B, H, Cq, d = qbar.shape
    Ck = kbar.shape[2]
    dev = Kp.device
    pair_off = torch.empty((B, H, Cq + 1), dtype=torch.int32, device=dev)
    pair_kc = torch.empty((B, H, Cq * Ck), dtype=torch.int32, device=dev)
    E = torch.empty((B, H, Cq, Ck), dtype=torch.float32, device=dev) if return_errors else None
    ws, n = _workspace(OP_ROUTE, kd, Cq, Ck, dev)
    _check("svgear_route", lib().svgear_route(
        _ptr(qbar), _ptr(q_off), Cq, _ptr(kbar), _ptr(vbar), _ptr(k_off), Ck, _ptr(Kp), _ptr(Vp),
        kd, float(density), float(scale), _ptr(pair_off), _ptr(pair_kc), _ptr(E), _ptr(ws), n,
        _stream()))
    return (pair_off, pair_kc, E) if return_errors else (pair_off, pair_kc)


def svgear_probe_value_free(qbar, Kp, kbar, k_off, scale):
    """Value-free probe error Ehat float32 [B, H, Cq, Ck]."""
    kd = _tokens(Kp, "Kp")
    B, H, Cq, d = qbar.shape
    Ck = kbar.shape[2]
    E = torch.empty((B, H, Cq, Ck), dtype=torch.float32, device=Kp.device)
    ws, n = _workspace(OP_ROUTE, kd, Cq, Ck, Kp.device)
    _check("svgear_probe_value_free", lib().svgear_probe_value_free(
        _ptr(qbar), Cq, _ptr(Kp), _ptr(kbar), _ptr(k_off), Ck, kd, float(scale), _ptr(E),
        _ptr(ws), n, _stream()))
    return E


def svgear_diagnostics(Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, O, q_perm, scale, rows):
    """Attention recall, |O - O_dense|^2 and |O_dense|^2 on the sampled
    permuted rows ``rows`` (int32 [B, H, R]); each float32 [B, H, R]."""
    qd = _tokens(Qp, "Qp")
    _tokens(Kp, "Kp")
    _tokens(Vp, "Vp")
    _cuda(rows, "rows", torch.int32)
    B, H, R = rows.shape
    Cq = q_off.shape[-1] - 1
    Ck = k_off.shape[-1] - 1
    out = [torch.empty((B, H, R), dtype=torch.float32, device=Qp.device) for _ in range(3)]
    _check("svgear_diagnostics", lib().svgear_diagnostics(
        _ptr(Qp), _ptr(Kp), _ptr(Vp), qd, Kp.shape[2], _ptr(q_off), Cq, _ptr(k_off), Ck,
        _ptr(pair_off), _ptr(pair_kc), _ptr(O), _ptr(q_perm), float(scale), _ptr(rows), R,
        _ptr(out[0]), _ptr(out[1]), _ptr(out[2]), _stream()))
    return tuple(out)


def svgear_key_variance(Kp, k_off, Ck):
    """Per-coordinate variance of every key cluster: float32 [B, H, Ck, d]."""
    kd = _tokens(Kp, "Kp")
    B, H, N, d = Kp.shape
    kvar = torch.empty((B, H, Ck, d), dtype=torch.float32, device=Kp.device)
    _check("svgear_key_variance", lib().svgear_key_variance(_ptr(Kp), _ptr(k_off), Ck, kd,
                                                            _ptr(kvar), _stream()))
    return kvar


def svgear_attend(Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, kbar, vbar, q_perm, scale, O=None,
                  check_status=False, kvar=None, lam=0.0):
    """O in the original token order.  check_status=True synchronises and
    raises if any bounded wait inside the kernel gave up.  With kvar (key
    variance per cluster) and lam != 0 the compensation is variance-corrected
    (svgear_attend_var)."""
    qd = _tokens(Qp, "Qp")
    _tokens(Kp, "Kp")
    _tokens(Vp, "Vp")
    Cq = q_off.shape[-1] - 1
    Ck = k_off.shape[-1] - 1
    Nk = Kp.shape[2]
    if O is None:
        O = torch.empty_like(Qp)
    ws, n = _workspace(OP_ATTEND, qd, Cq, Ck, Qp.device)
    if kvar is None:
        _check("svgear_attend", lib().svgear_attend(
            _ptr(Qp), _ptr(Kp), _ptr(Vp), qd, Nk, _ptr(q_off), Cq, _ptr(k_off), Ck, _ptr(pair_off),
            _ptr(pair_kc), _ptr(kbar), _ptr(vbar), _ptr(q_perm), float(scale), _ptr(O), _ptr(ws),
            n, _stream()))
    else:
        _cuda(kvar, "kvar", torch.float32)
        _check("svgear_attend_var", lib().svgear_attend_var(
            _ptr(Qp), _ptr(Kp), _ptr(Vp), qd, Nk, _ptr(q_off), Cq, _ptr(k_off), Ck, _ptr(pair_off),
            _ptr(pair_kc), _ptr(kbar), _ptr(vbar), _ptr(kvar), float(lam), _ptr(q_perm),
            float(scale), _ptr(O), _ptr(ws), n, _stream()))
    if check_status:
        _device_status("svgear_attend", ws, n)
    return O


def layer(Q, K, V, Cq, Ck, iters, density, scale=None, seed=0, warm_q=None, warm_k=None,
          topp=None, var_lambda=0.0, ready=None):
    """The whole layer for [B, H, N, d] tensors: cluster Q and K (seeds 2*seed
    and 2*seed+1), permute V, value centroids, route, attend.  The routing
    budget is floor(density * N) keys per query cluster, or, with topp=p, the
    keys holding p of the estimated weight (density is then unused).  With
    var_lambda != 0 the compensation is variance-corrected.  ready may map
    "q", "k", "v" to CUDA events the current stream waits for before the
    tensor's first use (inputs still arriving on another stream).  Returns O
    in the original token order and every intermediate."""
    d = Q.shape[-1]
    scale = d ** -0.5 if scale is None else scale

    def wait(name):
        if ready is not None and ready.get(name) is not None:
            torch.cuda.current_stream().wait_event(ready[name])

    wait("q")
    cq = svgear_cluster(Q, Cq, iters, warm_q, seed=2 * seed)
    wait("k")
    ck = svgear_cluster(K, Ck, iters, warm_k, seed=2 * seed + 1)
    wait("v")
    Vp = svgear_permute(V, ck.perm)
    vbar = svgear_centroids(Vp, ck.offsets, Ck)
    budget = None
    if topp is None:
        pair_off, pair_kc = svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets,
                                         ck.Xp, Vp, density, scale)
    else:
        pair_off, pair_kc, budget = svgear_route_topp(cq.centroids, cq.offsets, ck.centroids, vbar,
                                                      ck.offsets, ck.Xp, Vp, topp, scale)
    kvar = svgear_key_variance(ck.Xp, ck.offsets, Ck) if var_lambda else None
    O = svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, pair_off, pair_kc, ck.centroids,
                      vbar, cq.perm, scale, kvar=kvar, lam=var_lambda)
    return {"O": O, "q": cq, "k": ck, "Vp": Vp, "vbar": vbar, "pair_off": pair_off,
            "pair_kc": pair_kc, "budget": budget, "kvar": kvar}


def layer_params(Cq, Ck, iters, density, scale, seed=0, topp=None, var_lambda=0.0):
    return LayerParams(int(Cq), int(Ck), int(iters), float(density if density else 0.0),
                       float(topp or 0.0), float(scale), float(var_lambda), int(seed))


def svgear_layer(Q, K, V, Cq, Ck, iters, density, scale=None, seed=0, warm_q=None, warm_k=None,
                 topp=None, var_lambda=0.0, O=None, cent_q=None, cent_k=None, stage_events=None):
    """The whole layer in one C call on device tensors (svgear_layer).
    Returns (O, cent_q, cent_k); cent_* are the final centroids (allocated
    unless given; they may be the warm_* tensors, updated in place).
    stage_events: None or 6 torch.cuda.Event already recorded once (so that
    they exist), recorded again at the stage boundaries."""
    dims = _tokens(Q, "Q")
    _tokens(K, "K")
    _tokens(V, "V")
    B, H, N, d = Q.shape
    scale = d ** -0.5 if scale is None else scale
    prm = layer_params(Cq, Ck, iters, density, scale, seed, topp, var_lambda)
    dev = Q.device
    O = torch.empty_like(Q) if O is None else O
    if cent_q is None:
        cent_q = torch.empty((B, H, Cq, d), dtype=torch.float32, device=dev)
    if cent_k is None:
        cent_k = torch.empty((B, H, Ck, d), dtype=torch.float32, device=dev)
    for t, nm in ((warm_q, "warm_q"), (warm_k, "warm_k"), (cent_q, "cent_q"), (cent_k, "cent_k")):
        if t is not None:
            _cuda(t, nm, torch.float32)
    n = max(int(lib().svgear_layer_workspace_bytes(dims, ctypes.byref(prm), 0)), 256)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    ev = None
    if stage_events is not None:
        ev = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in stage_events])
    _check("svgear_layer", lib().svgear_layer(
        _ptr(Q), _ptr(K), _ptr(V), dims, ctypes.byref(prm), _ptr(warm_q), _ptr(warm_k), _ptr(O),
        _ptr(cent_q), _ptr(cent_k), _ptr(ws), n, ev, _stream()))
    return O, cent_q, cent_k


def layer_host(Qh, Kh, Vh, Cq, Ck, iters, density, scale=None, seed=0, warm_q=None,
               warm_k=None, topp=None, var_lambda=0.0, out=None, cent_q=None, cent_k=None):
    """The layer for host tensors in one C call (svgear_layer_host): the call
    copies Q, K and V to the device (pinned host tensors let the copies
    overlap the first stages), runs the layer and copies O back into `out`
    (a pinned host tensor like Qh, made if None), all on the current stream.
    Returns {"O_host", "cent_q", "cent_k"}; the host tensor is complete once
    the current stream has passed this call."""
    for t, nm in ((Qh, "Q"), (Kh, "K"), (Vh, "V")):
        if t.is_cuda or t.dim() != 4 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous host tensor [B, H, N, d]" % nm)
    B, H, N, d = Qh.shape
    dims = Dims(B, H, N, d, _dtype_code(Qh))
    scale = d ** -0.5 if scale is None else scale
    prm = layer_params(Cq, Ck, iters, density, scale, seed, topp, var_lambda)
    dev = torch.device("cuda", torch.cuda.current_device())
    if out is None:
        out = torch.empty(Qh.shape, dtype=Qh.dtype, pin_memory=True)
    if cent_q is None:
        cent_q = torch.empty((B, H, Cq, d), dtype=torch.float32, device=dev)
    if cent_k is None:
        cent_k = torch.empty((B, H, Ck, d), dtype=torch.float32, device=dev)
    n = max(int(lib().svgear_layer_workspace_bytes(dims, ctypes.byref(prm), 1)), 256)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    _check("svgear_layer_host", lib().svgear_layer_host(
        _ptr(Qh), _ptr(Kh), _ptr(Vh), dims, ctypes.byref(prm), _ptr(warm_q), _ptr(warm_k),
        _ptr(out), _ptr(cent_q), _ptr(cent_k), _ptr(ws), n, _stream()))
    return {"O_host": out, "cent_q": cent_q, "cent_k": cent_k}
