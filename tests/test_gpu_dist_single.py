"""The sharded path's CUDA side on hardware: one rank in an NCCL process group (the only multi-process
configuration a single GPU allows: ranks whose collectives wait on each other must not share one GPU).
dist.sharded_quantize with the library's CUDA steps runs the amax, the NCCL all-reduce(MAX) of one
float and the shard quantize; with one rank its result must equal the single-call quantize byte for
byte, and a 2-way split of the tensor quantized with the exchanged scale must concatenate to it too."""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import datetime, os, sys
    import torch, torch.distributed as dist
    sys.path.insert(0, os.environ["NVFP4_ROOT"])
    import nvfp4_block_scaled_11_b200 as nv
    from nvfp4_block_scaled_11_b200 import dist as nvdist, workloads as W
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    x = W.stream_f32("cuda", 2 ** -8).reshape(-1)
    codes, scales, g = nvdist.sharded_quantize(x, -2, 6)
    rc, rs, rg = nv.quantize(x, -2, 6)
    assert torch.equal(g, rg) and torch.equal(codes, rc) and torch.equal(scales, rs)
    # the same exchange over two shards of the tensor (each shard's amax, then one g for both)
    parts = []
    amaxes = []
    for r in range(2):
        lo, hi = nvdist.shard_bounds(x.numel(), 2, r)
        amaxes.append(nv.tensor_amax(x[lo:hi]))
    amax = torch.maximum(amaxes[0], amaxes[1])
    dist.all_reduce(amax, op=dist.ReduceOp.MAX)
    g2 = nv.global_scale(amax)
    for r in range(2):
        lo, hi = nvdist.shard_bounds(x.numel(), 2, r)
        c, s, _, _, _ = nv.quantize_ex(x[lo:hi], -2, 6, gscale_in=g2, want_f=False, want_sse=False)
        parts.append((c, s))
    assert torch.equal(g2, rg)
    assert torch.equal(torch.cat([p[0] for p in parts]), rc) and torch.equal(torch.cat([p[1] for p in parts]), rs)
    dist.barrier()
    dist.destroy_process_group()
    print("ok")
""")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sharded_quantize_over_nccl_one_rank():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), NVFP4_ROOT=ROOT,
               NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-3000:]
