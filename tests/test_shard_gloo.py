"""world_size-2 gloo test of the sharding host logic on CPU: row shards,
and per-tensor scaling from range records combined by an all-reduce MAX.
The per-rank compute is the CPU oracle (no GPU here); the product path runs
the same steps with the library's kernels over NCCL."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synthetic


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(v: torch.Tensor) -> torch.Tensor:
    """f64 range values (exact f32 numbers) -> int64 records of their f32 bits."""
    return torch.from_numpy(v.numpy().astype(np.float32).view(np.uint32).astype(np.int64))


def _unbits(r: torch.Tensor) -> torch.Tensor:
    return torch.from_numpy(r.numpy().astype(np.uint32).view(np.float32).astype(np.float64))


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from dequantize_absmax_reduce_b200.shard import allreduce_ranges_, row_range
        x = synthetic.Stream(42).tensor((37, 96), "bf16", outlier_p=0.02, outlier_factor=30)
        r0, r1 = row_range(37, world, rank)
        xl = x[r0:r1].contiguous()
        out = {}
        for sym, qd in ((True, "s8"), (False, "u8")):
            hi, nlo = oracle.group_range(xl, "tensor")
            rec = torch.stack([_bits(hi), _bits(nlo)], dim=1)
            allreduce_ranges_(rec)
            q, s, z = oracle.quantize(xl, "tensor", qdtype=qd, symmetric=sym,
                                      ranges=(_unbits(rec[:, 0]), _unbits(rec[:, 1])))
            out[qd] = (r0, r1, q, s, z)
        results[rank] = out
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_row_range_partition():
    from dequantize_absmax_reduce_b200.shard import row_range
    for n in (0, 1, 7, 37, 8192):
        for w in (1, 2, 3, 8):
            parts = [row_range(n, w, r) for r in range(w)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(w - 1))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1


def test_sharded_per_tensor_matches_whole_tensor(orc):
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world, join=True,
                       start_method="spawn")
    x = synthetic.Stream(42).tensor((37, 96), "bf16", outlier_p=0.02, outlier_factor=30)
    for sym, qd in ((True, "s8"), (False, "u8")):
        q, s, z = orc.quantize(x, "tensor", qdtype=qd, symmetric=sym)
        got = torch.cat([results[r][qd][2] for r in range(world)])
        assert torch.equal(got, q)
        for r in range(world):
            assert torch.equal(results[r][qd][3], s)
            assert torch.equal(results[r][qd][4], z)
