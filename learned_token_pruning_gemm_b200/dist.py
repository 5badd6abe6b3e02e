"""Process-group plumbing for running the layer as independent replicas, one
process per GPU (launched by torchrun). The path has no data exchange: sequences
are independent, so each rank runs the whole layer on its own inputs and the only
collectives are a barrier around the timed region and a max over ranks of the
measured time.
"""
from __future__ import annotations

import datetime
import os

import torch


class Replicas:
    def __init__(self, timeout_s: float = 120.0):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.dist = None
        if self.world > 1:
            import torch.distributed as dist
            use_cuda = torch.cuda.is_available()
            if use_cuda:
                local = int(os.environ.get("LOCAL_RANK", "0"))
                torch.cuda.set_device(local)
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=timeout_s),
                                        device_id=torch.device("cuda", local))
            else:
                dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=timeout_s))
            self.dist = dist
            self.rank = dist.get_rank()
            self._device = torch.device("cuda", torch.cuda.current_device()) if use_cuda \
                else torch.device("cpu")

    def barrier(self) -> None:
        if self.dist is not None:
            self.dist.barrier()

    def max(self, value: float) -> float:
        """The largest `value` over all ranks (every rank gets it)."""
        if self.dist is None:
            return value
        t = torch.tensor([value], dtype=torch.float64, device=self._device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self) -> None:
        if self.dist is not None:
            self.dist.destroy_process_group()
            self.dist = None
