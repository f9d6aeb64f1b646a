"""The sharded path on CPU ranks (gloo, world size 2): the shard-amax exchange gives every rank the
whole tensor's scale, and the concatenated shard outputs equal the single-process oracle quantize.
The per-shard steps use the oracle here; on GPUs the same exchange drives the CUDA library."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from nvfp4_block_scaled_11_b200 import dist as nvdist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops():
    from oracle import oracle as O

    def amax(x):
        return torch.tensor([O.tensor_amax(x.numpy())], dtype=torch.float32)

    def gs(a):
        return torch.tensor([O.global_scale(a.item())], dtype=torch.float32)

    def quantize(x, f_lo, f_hi, g):
        c, s, _, _, _ = O.quantize(x.numpy(), f_lo, f_hi, gscale_in=float(g.item()))
        return torch.from_numpy(c), torch.from_numpy(s)

    return nvdist.ShardOps(amax=amax, global_scale=gs, quantize=quantize)


def _worker(rank, world, port, x, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lo, hi = nvdist.shard_bounds(x.numel(), world, rank)
        codes, scales, g = nvdist.sharded_quantize(x[lo:hi].contiguous(), -2, 6, ops=_oracle_ops())
        out[rank] = (lo, hi, codes.numpy().copy(), scales.numpy().copy(), float(g.item()))
    finally:
        dist.destroy_process_group()


def test_shard_bounds_cover_and_align():
    for n in (16, 160, 16 * 1001, 16 * 7):
        for world in (1, 2, 3, 8):
            spans = [nvdist.shard_bounds(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c
            assert all(lo % 16 == 0 and hi % 16 == 0 for lo, hi in spans)
    with pytest.raises(ValueError):
        nvdist.shard_bounds(17, 2, 0)


def test_two_rank_sharded_quantize_matches_single_process():
    from oracle import oracle as O
    rng = np.random.default_rng(8)
    x = rng.standard_normal(16 * 4099).astype(np.float32)
    x[16 * 3000 + 5] = 37.0  # the tensor max lives in rank 1's shard
    xt = torch.from_numpy(x)
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), xt, out), nprocs=world, start_method="spawn", join=True)
    rc, rs, rg, _, _ = O.quantize(x, -2, 6)
    gs = {out[r][4] for r in range(world)}
    assert gs == {float(rg)}
    codes = np.concatenate([out[r][2] for r in range(world)])
    scales = np.concatenate([out[r][3] for r in range(world)])
    assert np.array_equal(codes, rc) and np.array_equal(scales, rs)


def _failing_worker(rank, world, port, x, out):
    """Rank 1 fails before the exchange; rank 0 must learn of it on the host through its collective
    (the peer closes its connection, or the short process-group timeout expires), not hang."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    try:
        if rank == 1:
            raise RuntimeError("injected failure before the amax exchange")
        lo, hi = nvdist.shard_bounds(x.numel(), world, rank)
        nvdist.sharded_quantize(x[lo:hi].contiguous(), -2, 6, ops=_oracle_ops())
        out[rank] = "completed"
    except Exception as e:  # recorded for the parent: the failure has to surface as an error
        out[rank] = f"error: {type(e).__name__}: {e}"
    finally:
        if rank == 1:
            dist.destroy_process_group()


def test_failed_rank_is_detected_on_the_host():
    import time
    x = torch.from_numpy(np.random.default_rng(9).standard_normal(16 * 512).astype(np.float32))
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    t = time.monotonic()
    mp.start_processes(_failing_worker, args=(world, _free_port(), x, out), nprocs=world, start_method="spawn",
                       join=True)
    assert time.monotonic() - t < 120
    assert out[1].startswith("error: RuntimeError: injected failure")
    assert out[0].startswith("error:"), out[0]
