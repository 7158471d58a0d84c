"""One process per GPU, each running an independent replica of the workload.

The forward pass has no exchange step between (b, kv head) groups ("DashAttention: Making
Sparse Attention Fully Differentiable with Adaptive Block Selection", section "Core
Mechanism": every group's selection and attention read only its own keys and values), so
several GPUs run replicas side by side (weak scaling) and meet only to time the job: a
barrier on both sides of the timed region and the maximum of the ranks' times.  With CUDA
the process group is NCCL with one device per rank; without it, gloo on the CPU (used by
the multi-process tests).  Rendezvous comes from the torchrun environment (MASTER_ADDR,
MASTER_PORT, RANK, WORLD_SIZE, LOCAL_RANK).
"""
from __future__ import annotations

import datetime
import os


class Replicas:
    def __init__(self, timeout_s: float = 300.0, backend: str | None = None):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.cuda = torch.cuda.is_available()
        self.backend = backend or ("nccl" if self.cuda else "gloo")
        if self.cuda:
            torch.cuda.set_device(self.local if self.world > 1 else 0)
        if self.world > 1:
            import torch.distributed as dist
            kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
            if self.backend == "nccl":
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(self.backend, **kw)

    @property
    def leader(self) -> bool:
        return self.rank == 0

    def barrier(self) -> None:
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float) -> float:
        """Largest value over the ranks (every rank gets it)."""
        if self.world == 1:
            return float(x)
        import torch
        import torch.distributed as dist
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def job_throughput(self, units_per_rank: float, seconds_this_rank: float) -> float:
        """Whole-job rate: the units of all ranks over the slowest rank's time."""
        return self.world * units_per_rank / self.max(seconds_this_rank)

    def close(self) -> None:
        if self.world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()
