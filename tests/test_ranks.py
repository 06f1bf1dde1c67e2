"""The multi-rank host path (one process per GPU, weak scaling) on the CPU:
two gloo ranks join, each draws its own batch element, and the job's time is
the slowest rank's; no data-path collective exists."""
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
    out[rank] = (got_ws, got_rank, worst, ranks.job_ms_per_call(worst, got_ws),
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
        ranks.barrier(1)
        ranks.teardown(1)
    finally:
        os.environ.update(env)
