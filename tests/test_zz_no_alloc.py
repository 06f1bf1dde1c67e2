"""The allocation-free label sort, called through the C ABI.

svgear_label_sort_noalloc is for callers that may not allocate device memory
(a framework memory planner that owns every byte, a real-time loop that bans
cudaMalloc, a plugin that only receives its inputs and outputs).  Its scratch
is a fixed array inside the library.  This file runs last on purpose; its
tests pass alone in a fresh process and after every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _call(L, labels, C, perm, off):
    from clustered_sparse_attention_b200 import _lib
    B, H, N = labels.shape
    return L.svgear_label_sort_noalloc(
        ctypes.c_void_p(labels.data_ptr()), _lib.Dims(B, H, N, 64, _lib.F32), C,
        ctypes.c_void_p(perm.data_ptr()), ctypes.c_void_p(off.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_sort_matches_workspace_sort_on_two_calls_in_a_row():
    import clustered_sparse_attention_b200 as csa
    from clustered_sparse_attention_b200 import _lib
    L = _lib.lib()
    g = np.random.default_rng(99)
    # second call: other sizes and fewer clusters, so stale scratch would show
    for (B, H, N, C) in [(1, 3, 5000, 300), (2, 2, 2049, 37)]:
        lab = g.integers(0, C, (B, H, N)).astype(np.int32)
        lab[lab % 5 == 1] = 0                      # some clusters empty
        labels = torch.from_numpy(lab).cuda()
        ref_perm, ref_off = csa.svgear_label_sort(labels, C)
        perm = torch.full((B, H, N), -1, dtype=torch.int32, device="cuda")
        off = torch.full((B, H, C + 1), -1, dtype=torch.int32, device="cuda")
        assert _call(L, labels, C, perm, off) == _lib.OK
        torch.cuda.synchronize()
        assert torch.equal(perm, ref_perm) and torch.equal(off, ref_off)
        p_o, o_o = oracle.stable_sort(lab[0, 0], C)
        assert np.array_equal(perm.cpu().numpy()[0, 0], p_o)
        assert np.array_equal(off.cpu().numpy()[0, 0], o_o)


def test_noalloc_sort_rejects_sizes_beyond_its_scratch():
    from clustered_sparse_attention_b200 import _lib
    L = _lib.lib()
    # 40 heads x 118 blocks of 1024 tokens x 500 clusters > 2 Mi entries
    labels = torch.zeros((1, 40, 120000), dtype=torch.int32, device="cuda")
    perm = torch.empty_like(labels)
    off = torch.empty((1, 40, 501), dtype=torch.int32, device="cuda")
    assert _call(L, labels, 500, perm, off) == _lib.ERR_SCRATCH_LIMIT
