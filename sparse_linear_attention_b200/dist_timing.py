"""Multi-process plumbing of the benchmark: one process per GPU, each running
the whole forward on its own batch (the heads of different ranks never
interact, so the data path has no collective).  What the ranks share is the
timing: every interval is measured on the device by each rank and the job's
time is the maximum over ranks.  Runs on any torch.distributed backend (NCCL
on the GPUs, gloo in the CPU tests)."""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist


def world_info() -> tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def distributed() -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1


def max_over_ranks(value: float, device=None) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if not distributed():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    if distributed():
        dist.barrier()


def job_throughput(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job units per second: every rank processes units_per_rank in an
    interval that the slowest rank bounds at ms_max (weak scaling)."""
    if ms_max <= 0.0:
        raise ValueError("interval must be positive")
    return units_per_rank * world / (ms_max * 1e-3)


def reports(rank: int) -> bool:
    """Only rank 0 prints the result line."""
    return rank == 0


def launched() -> bool:
    """True inside a process that a launcher (torchrun) started as one rank."""
    return "WORLD_SIZE" in os.environ


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launcher_argv(script: str, argv: list[str], nproc: int, port: int) -> list[str]:
    """The torchrun command that starts `nproc` ranks of `script argv` on this
    node, rendezvous on 127.0.0.1."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", script, *argv]


def run_ranks(script: str, argv: list[str], nproc: int, timeout_s: float | None = None) -> int:
    """Start `nproc` ranks of `script argv` under torchrun and return its exit
    code (output goes to this process's stdout / stderr)."""
    cmd = launcher_argv(script, argv, nproc, free_port())
    try:
        return subprocess.run(cmd, timeout=timeout_s).returncode
    except subprocess.TimeoutExpired:
        return 124
