"""The multi-rank host path (one process per GPU) on the CPU with gloo ranks:
the head split of one layer call (each rank owns a contiguous head range,
every head exactly once; O reassembles at the right offsets), the batch split
(each rank draws its own batch element), and the job's time as the slowest
rank's.  No data-path collective exists inside the layer."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from clustered_sparse_attention_b200 import ranks, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, out):
    os.environ.update({"WORLD_SIZE": str(ws), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    got_ws, got_rank, _ = ranks.setup("gloo", timeout_s=60)
    # each rank's own synthetic batch element (a small workload)
    w = synth.custom_workload("ranks", H=1, frames=1, grid_h=8, grid_w=8, d=64, dtype="bf16",
                              Cq=4, Ck=8, iters=1, density=0.5, n_centres=4, sigma=0.5, index=60)
    bits = synth.layer_tensor_bits(w, "k", threads=1, batch_offset=ranks.batch_offset(rank))
    step_ms = 10.0 + 5.0 * rank                       # rank 1 is the slower one
    ranks.barrier(got_ws)
    worst = ranks.max_over_ranks(step_ms, got_ws)
    out[rank] = (got_ws, got_rank, worst, ranks.job_ms_per_call(worst, got_ws, split="batch"),
                 int(bits.astype(np.int64).sum()))
    ranks.teardown(got_ws)


def test_two_gloo_ranks_shard_the_batch_and_time_the_slowest():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][:2] == (2, 0) and res[1][:2] == (2, 1)
    # both ranks see the slowest step; the job runs two layer calls per step
    assert res[0][2] == res[1][2] == 15.0
    assert res[0][3] == 7.5
    # the ranks drew different batch elements, each equal to its own draw
    assert res[0][4] != res[1][4]
    w = synth.custom_workload("ranks", H=1, frames=1, grid_h=8, grid_w=8, d=64, dtype="bf16",
                              Cq=4, Ck=8, iters=1, density=0.5, n_centres=4, sigma=0.5, index=60)
    for r in range(2):
        own = synth.bf16_bits(synth.head_tensor(w, "k", r, 0))
        assert res[r][4] == int(own.astype(np.int64).sum())


def test_single_process_needs_no_process_group():
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        assert ranks.setup() == (1, 0, 0)
        assert ranks.max_over_ranks(3.5, 1) == 3.5
        assert ranks.job_ms_per_call(8.0, 1) == 8.0
        assert ranks.head_range(40, 1, 0) == (0, 40)
        ranks.barrier(1)
        ranks.teardown(1)
    finally:
        os.environ.update(env)


def test_head_ranges_cover_every_head_exactly_once():
    for H in (1, 5, 24, 40, 41):
        for ws in (1, 2, 3, 4, 7, 8, 16, 48):
            seen = []
            prev_hi = 0
            for r in range(ws):
                lo, hi = ranks.head_range(H, ws, r)
                assert lo == prev_hi and lo <= hi           # contiguous, in rank order
                prev_hi = hi
                seen.extend(range(lo, hi))
            assert seen == list(range(H))
            sizes = [ranks.head_range(H, ws, r)[1] - ranks.head_range(H, ws, r)[0]
                     for r in range(ws)]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        ranks.head_range(8, 2, 2)


def _o_value(B, heads, N, d):
    """A host 'output' whose every element names its batch, head, row and
    column, so a misplaced slice cannot go unnoticed."""
    import torch
    b = torch.arange(B, dtype=torch.float64).view(B, 1, 1, 1)
    h = torch.tensor(list(heads), dtype=torch.float64).view(1, -1, 1, 1)
    n = torch.arange(N, dtype=torch.float64).view(1, 1, N, 1)
    k = torch.arange(d, dtype=torch.float64).view(1, 1, 1, d)
    return (b * 1e7 + h * 1e5 + n * 1e2 + k).expand(B, len(list(heads)), N, d).contiguous()


def _head_worker(rank, ws, port, H, out):
    os.environ.update({"WORLD_SIZE": str(ws), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    got_ws, got_rank, _ = ranks.setup("gloo", timeout_s=60)
    lo, hi = ranks.head_range(H, got_ws, got_rank)
    B, N, d = 2, 6, 4
    full = ranks.gather_heads(_o_value(B, range(lo, hi), N, d), H, got_ws, got_rank)
    out[rank] = (lo, hi, bool((full == _o_value(B, range(H), N, d)).all()))
    ranks.teardown(got_ws)


@pytest.mark.parametrize("ws,H", [(2, 5), (3, 40)])
def test_head_split_reassembles_o_at_the_right_offsets(ws, H):
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_head_worker, args=(r, ws, port, H, out)) for r in range(ws)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    covered = sorted(h for r in range(ws) for h in range(res[r][0], res[r][1]))
    assert covered == list(range(H))
    assert all(res[r][2] for r in range(ws))
