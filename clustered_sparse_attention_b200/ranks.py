"""One process per GPU: the host-side plumbing of a multi-rank run.

The layer partitions by (batch, head) with no exchange inside it, so ranks run
independent layer calls on their own batch elements (weak scaling); the only
collectives are for timing: a barrier around the timed region and the maximum
of the ranks' step times.  Works with the NCCL backend on GPUs and with gloo on
the CPU (which the tests use).
"""
import datetime
import os

# A rank that waits on the others gives up after this long (the launcher puts
# its own, longer, limit around the whole job).
PG_TIMEOUT_S = 120


def setup(backend=None, timeout_s=PG_TIMEOUT_S):
    """(world_size, rank, local_rank) from the launcher's environment; joins
    the process group when world_size > 1 (NCCL on the local GPU unless
    another backend is named)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        backend = backend or "nccl"
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, **kw)
    return ws, rank, local


def batch_offset(rank):
    """Batch element a rank draws its synthetic inputs for: its own."""
    return rank


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws, device="cpu"):
    """The largest of the ranks' values of x (the job's step time)."""
    if ws == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_call(ms_per_step_max, ws):
    """Whole-job time per layer call: every rank runs one call per step, so
    the job completes ws calls in the slowest rank's step time."""
    return ms_per_step_max / ws


def teardown(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
