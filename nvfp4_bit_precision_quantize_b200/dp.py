"""Data-parallel plumbing for the NVFP4 MLP step: one process per GPU.

Each rank trains on its own token shard (weak scaling: the per-GPU batch is
fixed) and the only exchange is the sum of the weight gradients dW across
ranks (torch.distributed all-reduce; NCCL over NVLink on GPUs, gloo on CPU in
the tests).  Timings are reduced as the maximum over ranks.
"""
import datetime
import os

import torch
import torch.distributed as dist


def world():
    return int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def init(backend="nccl", timeout_s=120):
    """Join the process group if launched under torchrun (WORLD_SIZE > 1)."""
    ws, rank, local = world()
    if ws > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return ws, rank, local


def shard_data_seed(base_seed, rank):
    """Seed of a rank's token shard (its X and dY2; the weights are drawn from
    base_seed on every rank): None on rank 0, which keeps the single-GPU
    workload, base_seed + 1000 * rank elsewhere."""
    return None if rank == 0 else base_seed + 1000 * rank


class GradExchange:
    """Sums each weight gradient over the ranks as soon as the step has queued the
    GEMM that produces it, so the exchange overlaps the rest of the backward pass
    (the down-projection's dW while the up-projection's backward runs).

    ready(name, t) launches an asynchronous all-reduce of t (NCCL runs it on its
    own stream after t's producer; gloo in the background); wait() makes the
    caller's stream (NCCL) or the host (gloo) wait for all of them.  Every rank
    issues the same exchanges in the same order.  On one rank both are no-ops.
    `order` records the names in issue order."""

    def __init__(self):
        self.pending = []
        self.order = []
        self.active = dist.is_initialized() and dist.get_world_size() > 1

    def ready(self, name, t):
        self.order.append(name)
        if self.active:
            self.pending.append(dist.all_reduce(t, op=dist.ReduceOp.SUM, async_op=True))

    def wait(self):
        for w in self.pending:
            w.wait()
        self.pending.clear()


def allreduce_grads(grads):
    """Sum each gradient tensor over all ranks, in place (no-op on one rank)."""
    if dist.is_initialized() and dist.get_world_size() > 1:
        for g in grads:
            dist.all_reduce(g, op=dist.ReduceOp.SUM)
    return grads


def max_over_ranks(value, device="cpu"):
    """Maximum of a float over all ranks (the slowest rank sets the step time)."""
    if dist.is_initialized() and dist.get_world_size() > 1:
        t = torch.tensor([float(value)], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return float(value)


def barrier():
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def finish():
    if dist.is_initialized():
        dist.destroy_process_group()
