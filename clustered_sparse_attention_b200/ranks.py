"""One process per GPU: the host-side plumbing of a multi-rank run.

The layer is independent per (batch, head): clustering, routing and attention
of one head never read another head's data.  So one layer call splits its H
heads over the ranks, rank r taking the contiguous range ``head_range(H, ws,
r)``, and no data moves between ranks inside the layer.  Each rank keeps O for
its own heads; ``gather_heads`` reassembles the full [B, H, N, d] output with
one all-gather when a caller needs it on every rank.  The other collectives
are for timing: a barrier around the timed region and the maximum of the
ranks' step times.  Works with NCCL on GPUs and with gloo on the CPU (which
the tests use).  ``batch_offset`` serves the other split, one independent
batch element per rank.
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


def head_range(H, ws, rank):
    """Heads [lo, hi) of a layer call owned by `rank` of `ws`: contiguous,
    in rank order, sizes differing by at most one, every head exactly once.
    A rank gets no heads (lo == hi) when ws > H."""
    if H < 0 or ws < 1 or not 0 <= rank < ws:
        raise ValueError("bad split: H=%d ws=%d rank=%d" % (H, ws, rank))
    base, extra = divmod(H, ws)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def gather_heads(O_local, H, ws, rank):
    """Reassemble O [B, H, N, d] on every rank from each rank's slice
    O_local [B, hi - lo, N, d] of its head_range (one all-gather; slices are
    padded to the largest range)."""
    import torch
    lo, hi = head_range(H, ws, rank)
    if O_local.shape[1] != hi - lo:
        raise ValueError("rank %d holds %d heads, its range has %d" % (rank, O_local.shape[1],
                                                                      hi - lo))
    if ws == 1:
        return O_local
    import torch.distributed as dist
    B, _, N, d = O_local.shape
    width = max(head_range(H, ws, r)[1] - head_range(H, ws, r)[0] for r in range(ws))
    pad = torch.zeros((B, width, N, d), dtype=O_local.dtype, device=O_local.device)
    pad[:, :hi - lo] = O_local
    parts = [torch.empty_like(pad) for _ in range(ws)]
    dist.all_gather(parts, pad.contiguous())
    out = torch.empty((B, H, N, d), dtype=O_local.dtype, device=O_local.device)
    for r in range(ws):
        a, b = head_range(H, ws, r)
        out[:, a:b] = parts[r][:, :b - a]
    return out


def batch_offset(rank):
    """Batch element a rank draws its synthetic inputs for under the batch
    split: its own."""
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


def job_ms_per_call(ms_per_step_max, ws, split="heads"):
    """Whole-job time per layer call.  Head split: the ranks share one call,
    which ends with the slowest rank.  Batch split: every rank runs one call
    per step, so the job completes ws calls in the slowest rank's step."""
    return ms_per_step_max if split == "heads" else ms_per_step_max / ws


def teardown(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
