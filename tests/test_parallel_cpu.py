"""World-size-2 gloo tests of the data-parallel exchange, on CPU.

The per-rank adapter gradients come from the oracle (this is a test of the sharding and of the exchange,
not of the kernels); their all-reduced sum must equal the full-batch gradients.  A rank that fails before
the exchange must make the other rank's collective end with an error instead of waiting forever.
"""

import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from qlora_fine_tuning_blockwise_b200.parallel import allreduce_adapter_grads, token_shard


def free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _init(rank, world, port, timeout_s=60):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=timeout_s))


def _dp_worker(rank, world, port, outdir):
    from oracle import linear as L
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    _init(rank, world, port)
    d = I.make_random_linear(37, 24, 64, 8, s=2.0, seed=3)
    f = lambda t: t.float().numpy().astype(np.float64)
    b, e = token_shard(37, world, rank)
    dA, dB = L.lora_grads(f(d["dy"])[b:e], f(d["x"])[b:e], f(d["A"]), f(d["B"]), 2.0)
    tA, tB = torch.from_numpy(dA), torch.from_numpy(dB)
    allreduce_adapter_grads([tA, tB])
    np.save(os.path.join(outdir, f"dA{rank}.npy"), tA.numpy())
    np.save(os.path.join(outdir, f"dB{rank}.npy"), tB.numpy())
    dist.destroy_process_group()


def test_token_shard_covers_batch():
    for M in (0, 1, 7, 37, 2048):
        for world in (1, 2, 3, 8):
            spans = [token_shard(M, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1


def test_dp_adapter_grads_equal_full_batch():
    from oracle import linear as L
    from qlora_fine_tuning_blockwise_b200 import inputs as I
    with tempfile.TemporaryDirectory() as td:
        mp.start_processes(_dp_worker, args=(2, free_port(), td), nprocs=2, join=True, start_method="spawn")
        d = I.make_random_linear(37, 24, 64, 8, s=2.0, seed=3)
        f = lambda t: t.float().numpy().astype(np.float64)
        rA, rB = L.lora_grads(f(d["dy"]), f(d["x"]), f(d["A"]), f(d["B"]), 2.0)
        for r in range(2):
            assert np.allclose(np.load(os.path.join(td, f"dA{r}.npy")), rA, rtol=1e-12, atol=1e-12)
            assert np.allclose(np.load(os.path.join(td, f"dB{r}.npy")), rB, rtol=1e-12, atol=1e-12)


def _failing_worker(rank, world, port, outdir):
    _init(rank, world, port, timeout_s=5)
    if rank == 1:
        # this rank fails before the exchange and leaves
        raise SystemExit(3)
    t = torch.ones(4)
    try:
        allreduce_adapter_grads([t])
        status = "completed"
    except Exception as exc:  # the surviving rank must see an error, not hang
        status = "error: " + type(exc).__name__
    with open(os.path.join(outdir, "rank0.txt"), "w") as fh:
        fh.write(status)


def test_failed_rank_makes_peer_collective_error_not_hang():
    with tempfile.TemporaryDirectory() as td:
        ctx = mp.start_processes(_failing_worker, args=(2, free_port(), td), nprocs=2, join=False,
                                 start_method="spawn")
        for p in ctx.processes:
            p.join(timeout=120)
        alive = [p for p in ctx.processes if p.is_alive()]
        for p in alive:
            p.kill()
        assert not alive, "a rank hung"
        status = open(os.path.join(td, "rank0.txt")).read()
        assert status.startswith("error"), status
