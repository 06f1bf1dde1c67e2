"""The C-ABI library builds, loads and exports every symbol include/svgear.h
declares; host-side validation rejects bad arguments before any launch
(these run without a GPU: no call below reaches the CUDA runtime)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from clustered_sparse_attention_b200 import build
    build.build()
    from clustered_sparse_attention_b200 import _lib
    return _lib.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "svgear.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svgear_\w+)\s*\(", src)))


def test_header_declares_the_expected_entry_points():
    names = _declared()
    for must in ("svgear_cluster", "svgear_centroids", "svgear_route", "svgear_attend"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    from clustered_sparse_attention_b200 import _lib
    for name in _declared():
        assert hasattr(L, name), name
    assert set(_declared()) <= set(_lib.EXPORTED) | set(_declared())
    assert L.svgear_version() >= 100


def test_library_is_built_for_sm100a_only():
    from clustered_sparse_attention_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)


def _dims(B=1, H=2, N=1000, d=128, dtype=1):
    from clustered_sparse_attention_b200._lib import Dims
    return Dims(B, H, N, d, dtype)


def test_status_strings(L):
    assert L.svgear_status_string(0) == b"ok"
    assert b"workspace" in L.svgear_status_string(-5)


def test_workspace_bytes_rejects_bad_sizes(L):
    from clustered_sparse_attention_b200 import _lib
    assert L.svgear_workspace_bytes(_lib.OP_CLUSTER, _dims(), 100, 0) > 0
    assert L.svgear_workspace_bytes(_lib.OP_CLUSTER, _dims(), 1001, 0) == 0      # C > N
    assert L.svgear_workspace_bytes(_lib.OP_CLUSTER, _dims(d=96), 10, 0) == 0    # d
    assert L.svgear_workspace_bytes(_lib.OP_CLUSTER, _dims(dtype=7), 10, 0) == 0
    assert L.svgear_workspace_bytes(_lib.OP_ROUTE, _dims(), 100, 5000) == 0      # > max clusters
    assert L.svgear_workspace_bytes(99, _dims(), 10, 10) == 0


def test_validation_before_launch(L):
    from clustered_sparse_attention_b200 import _lib
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: validation fails first
    ws_small = ctypes.c_size_t(16)
    big = ctypes.c_size_t(1 << 30)
    # null X
    assert L.svgear_kmeans_assign(None, _dims(), fake, 10, fake, fake, big, None) == _lib.ERR_INVALID_ARG
    # unsupported head dimension / dtype
    assert L.svgear_kmeans_assign(fake, _dims(d=96), fake, 10, fake, fake, big, None) == _lib.ERR_UNSUPPORTED
    assert L.svgear_kmeans_assign(fake, _dims(dtype=3), fake, 10, fake, fake, big, None) == _lib.ERR_UNSUPPORTED
    # C out of range
    assert L.svgear_kmeans_assign(fake, _dims(), fake, 0, fake, fake, big, None) == _lib.ERR_INVALID_ARG
    assert L.svgear_kmeans_assign(fake, _dims(N=5000), fake, 4097, fake, fake, big,
                                  None) == _lib.ERR_UNSUPPORTED
    # misaligned token pointer
    assert L.svgear_kmeans_assign(ctypes.c_void_p((1 << 20) + 4), _dims(), fake, 10, fake, fake,
                                  big, None) == _lib.ERR_INVALID_ARG
    # workspace too small
    assert L.svgear_kmeans_assign(fake, _dims(), fake, 10, fake, fake, ws_small,
                                  None) == _lib.ERR_WORKSPACE
    # iters < 1
    assert L.svgear_cluster(fake, _dims(), 10, 0, None, 0, fake, fake, fake, fake, None, fake,
                            ctypes.c_size_t(1 << 30), None) == _lib.ERR_INVALID_ARG
    # workspace too small
    assert L.svgear_cluster(fake, _dims(), 10, 3, None, 0, fake, fake, fake, fake, None, fake,
                            ws_small, None) == _lib.ERR_WORKSPACE
    # density outside (0, 1]
    for bad in (0.0, -0.5, 1.5, float("nan")):
        assert L.svgear_route_select(fake, fake, 10, fake, 20, 1, 2, 1000, bad, fake, fake, fake,
                                     ctypes.c_size_t(1 << 30), None) == _lib.ERR_INVALID_ARG
    # Ck > Nk
    assert L.svgear_route_select(fake, fake, 10, fake, 2000, 1, 2, 1000, 0.5, fake, fake, fake,
                                 ctypes.c_size_t(1 << 30), None) == _lib.ERR_INVALID_ARG
    # non-finite scale
    assert L.svgear_attend(fake, fake, fake, _dims(), 1000, fake, 10, fake, 20, fake, fake, fake,
                           fake, fake, float("inf"), fake, fake, ctypes.c_size_t(1 << 30),
                           None) == _lib.ERR_INVALID_ARG


def test_empty_batch_is_a_no_op(L):
    fake = ctypes.c_void_p(1 << 20)
    # B = 0: valid, nothing to launch, no CUDA call
    assert L.svgear_kmeans_assign(fake, _dims(B=0), fake, 10, fake, fake, ctypes.c_size_t(1 << 20),
                                  None) == 0
    assert L.svgear_centroids(fake, fake, 10, _dims(B=0), fake, fake, ctypes.c_size_t(1 << 20),
                              None) == 0


def test_selftest_wait_validates_before_launch(L):
    from clustered_sparse_attention_b200 import _lib
    fake = ctypes.c_void_p(1 << 20)
    ok = ctypes.c_size_t(256)
    assert L.svgear_selftest_wait(None, ok, 0, 1000, 0, None) == _lib.ERR_INVALID_ARG
    assert L.svgear_selftest_wait(fake, ctypes.c_size_t(8), 0, 1000, 0, None) == _lib.ERR_INVALID_ARG
    assert L.svgear_selftest_wait(fake, ok, 2, 1000, 0, None) == _lib.ERR_INVALID_ARG
    assert L.svgear_selftest_wait(fake, ok, 0, 0, 0, None) == _lib.ERR_INVALID_ARG
    assert L.svgear_selftest_wait(fake, ok, 0, 10_000_001, 0, None) == _lib.ERR_INVALID_ARG
    assert L.svgear_selftest_wait(fake, ok, 0, 1000, 3, None) == _lib.ERR_INVALID_ARG
    assert L.svgear_device_status(None, ok, fake, None) == _lib.ERR_INVALID_ARG
    assert b"tensor memory" in L.svgear_status_string(_lib.ERR_TMEM_LOST)


def test_layer_entry_points_validate_before_launch(L):
    from clustered_sparse_attention_b200 import _lib
    fake = ctypes.c_void_p(1 << 20)
    big = ctypes.c_size_t(1 << 40)
    good = _lib.layer_params(100, 500, 40, 0.25, 128 ** -0.5)
    d = _dims(H=40, N=75600)
    n0 = L.svgear_layer_workspace_bytes(d, ctypes.byref(good), 0)
    n1 = L.svgear_layer_workspace_bytes(d, ctypes.byref(good), 1)
    assert n1 - n0 >= 3 * 40 * 75600 * 128 * 2            # the three device input copies
    for bad in (_lib.layer_params(0, 500, 40, 0.25, 0.1), _lib.layer_params(100, 500, 0, 0.25, 0.1),
                _lib.layer_params(100, 500, 40, 0.0, 0.1), _lib.layer_params(100, 500, 40, 0.3, 0.1,
                                                                             topp=1.5),
                _lib.layer_params(100, 500, 40, 0.3, float("nan")),
                _lib.layer_params(100, 80000, 40, 0.3, 0.1)):
        assert L.svgear_layer_workspace_bytes(d, ctypes.byref(bad), 0) == 0
        assert L.svgear_layer(fake, fake, fake, d, ctypes.byref(bad), None, None, fake, None, None,
                              fake, big, None, None) != _lib.OK
    # null output, small workspace
    assert L.svgear_layer(fake, fake, fake, d, ctypes.byref(good), None, None, None, None, None,
                          fake, big, None, None) == _lib.ERR_INVALID_ARG
    assert L.svgear_layer_host(fake, fake, fake, d, ctypes.byref(good), None, None, fake, None,
                               None, fake, ctypes.c_size_t(n0), None) == _lib.ERR_WORKSPACE
    # top-p replaces the density: density 0 is then allowed
    tp = _lib.layer_params(100, 500, 40, 0.0, 0.1, topp=0.9)
    assert L.svgear_layer_workspace_bytes(d, ctypes.byref(tp), 0) > 0
