"""Data-parallel decomposition, world_size 2 over gloo on the CPU: each rank takes its
token shard, computes its adapter gradients (here with the fp64 oracle standing in for
the GPU step), packs them into the flat buffer and all-reduces; the result must equal
the full-batch gradients, and the row outputs must equal the full-batch rows."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from lora_fine_tuning_rmsnorm_b200 import dist as ldist
from lora_fine_tuning_rmsnorm_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, shape, q):
    from oracle import lora_mlp_ref as ref
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = synth.bits_to_f64(synth.make_inputs_bits(shape))
        t0, t1 = ldist.shard_rows(shape.T, world, rank)
        mine = dict(inp)
        mine["X"], mine["dY"] = inp["X"][t0:t1], inp["dY"][t0:t1]
        out = ref.fwd_bwd(mine, shape.scale, shape.eps, keep=("Y", "dX"))
        flat, views = ldist.flat_grads(shape.d, shape.f, shape.r, dtype=torch.float64)
        for k in ldist.GRAD_ORDER:
            views[k].copy_(torch.from_numpy(out[k]))
        ldist.allreduce_grads(flat)
        q.put((rank, t0, t1, {k: views[k].numpy().copy() for k in ldist.GRAD_ORDER}, out["Y"], out["dX"]))
    finally:
        dist.destroy_process_group()


def test_shard_rows_cover_exactly():
    for T, world in [(64, 2), (65, 2), (7, 4), (8192, 8)]:
        spans = [ldist.shard_rows(T, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == T
        assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))


@pytest.mark.timeout(300)
def test_dp_allreduce_equals_full_batch():
    from oracle import lora_mlp_ref as ref
    shape = synth.Shape(T=45, d=16, f=24, r=8, alpha=16.0)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, shape, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    full = ref.fwd_bwd(synth.bits_to_f64(synth.make_inputs_bits(shape)), shape.scale, shape.eps, keep=("Y", "dX"))
    for rank, t0, t1, grads, Y, dX in res:
        for k in ldist.GRAD_ORDER:
            np.testing.assert_allclose(grads[k], full[k], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(Y, full["Y"][t0:t1], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(dX, full["dX"][t0:t1], rtol=1e-12, atol=1e-14)
