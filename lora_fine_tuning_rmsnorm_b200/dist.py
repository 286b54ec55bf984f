"""Data-parallel plumbing for the LoRA-MLP step (host side, torch.distributed).

The path shards along tokens: every rank runs the full sub-block on its own rows
with replicated frozen weights and adapters, and the only exchange is one sum
all-reduce of the six adapter gradients (fp32), packed into one flat buffer so the
collective is a single call.  Y, dX and the saved context stay rank-local.
"""
from __future__ import annotations

GRAD_ORDER = ("dAg", "dBg", "dAu", "dBu", "dAd", "dBd")


def grad_shapes(d: int, f: int, r: int) -> dict:
    return {"dAg": (r, d), "dBg": (f, r), "dAu": (r, d), "dBu": (f, r), "dAd": (r, f), "dBd": (d, r)}


def flat_grads(d: int, f: int, r: int, device=None, dtype=None):
    """One flat fp32 buffer and views into it, one per adapter gradient (16-byte
    aligned views: every size is a multiple of 8 floats when r % 8 == 0)."""
    import torch
    shapes = grad_shapes(d, f, r)
    total = sum(a * b for a, b in shapes.values())
    flat = torch.zeros(total, dtype=dtype or torch.float32, device=device)
    views, off = {}, 0
    for k in GRAD_ORDER:
        n = shapes[k][0] * shapes[k][1]
        views[k] = flat[off:off + n].view(*shapes[k])
        off += n
    return flat, views


def shard_rows(T_global: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous token range [t0, t1) of `rank` (the first T % world ranks get one more)."""
    base, extra = divmod(T_global, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def allreduce_grads(flat, group=None):
    """Sum the packed adapter gradients over all ranks (in place)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat


def max_over_ranks(x: float, device) -> float:
    """The largest value of x over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def torchrun_argv(nproc: int, script: str, argv: list, port: int | None = None) -> list:
    """Command that runs `script argv` as `nproc` ranks on this node (one per GPU),
    rendezvous on 127.0.0.1."""
    import sys
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
            "--master-addr=127.0.0.1", f"--master-port={port or free_port()}", script, *argv]
