"""Multi-GPU orchestration for the attention path: replicas only.

Every (batch, KV head) problem of the path is independent and each workload
fits one GPU, so N GPUs run N independent replicas (weak scaling). No
collective is on the data path; the process group only lines the ranks up
before and after a timed region, takes the slowest rank's time, and reports
the whole job's throughput as N times one replica's work over that time.

One process per GPU, launched by torch.distributed.run (RANK, LOCAL_RANK,
WORLD_SIZE, MASTER_ADDR/PORT from the environment). The backend is NCCL on
GPUs; the same code runs over gloo on CPU for the multi-process tests.
"""

import datetime
import os

import torch


def env():
    """(world, rank, local_rank) from the launcher's environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def setup(backend="nccl", timeout_s=120):
    """Joins the process group when WORLD_SIZE > 1. A short timeout makes ranks
    that wait for a rank which has died end with an error instead of hanging."""
    world, rank, local = env()
    if world > 1:
        import torch.distributed as dist

        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world, device="cuda"):
    """The largest value of x over all ranks (the slowest rank's time)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_replica, world, max_ms):
    """Whole-job throughput: every replica processed units_per_replica in at most max_ms."""
    return world * units_per_replica / (max_ms * 1e-3)


def teardown(world):
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
