"""Time the ScaleSearch launch shapes against each other on this GPU, to place nvfp4_search_policy's bounds.

    python -m nvfp4_block_scaled_11_b200.tune_policy [--blocks 1024,4096,...] [--dtype f32|bf16]

For each block count and window ([-2, 6] and [-8, 8]) it quantizes N(0, 4) values with an external
tensor scale g = amax / 2688 (the search pass alone) under each launch shape forced through the policy
-- one offset per lane, a few offsets per lane, a thread per block -- and under the default bounds,
and prints microseconds per launch: CUDA events around a CUDA graph of 20 launches, best of 10
replays.  The bounds count threads (blocks x lanes per block: 16 or 32 for one offset per lane, 4 or
8 for a few), so a crossover at B blocks maps to a bound of B x those lanes.  The last lines time one
decode-sized KV append (8 heads x 16 tokens x 128) the same way.  The policy is restored on exit.
"""
from __future__ import annotations

import argparse

import torch

import nvfp4_block_scaled_11_b200 as nv

HUGE = 1 << 40


def graph_us(fn, reps: int = 20, iters: int = 10) -> float:
    """Best per-launch time of `reps` calls of fn captured in one CUDA graph, in microseconds."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            fn()
    graph.replay()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b) * 1e3 / reps)
    return best


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--blocks", default="1024,4096,8192,32768,49152,65536,98304")
    ap.add_argument("--dtype", choices=["f32", "bf16"], default="f32")
    args = ap.parse_args()
    dt = torch.float32 if args.dtype == "f32" else torch.bfloat16
    default = nv.search_policy()
    shapes = (("one/lane", (HUGE, HUGE)), ("few/lane", (0, HUGE)), ("thread/block", (0, 0)), ("default", default))
    try:
        print("blocks  window   " + "  ".join(f"{name:>12s}" for name, _ in shapes) + "   (us per launch)")
        for nb in (int(v) for v in args.blocks.split(",")):
            x = (torch.randn(nb * 16, device="cuda") * 2).to(dt)
            g = (x.float().abs().max() / 2688.0).reshape(1).contiguous()
            codes = torch.empty(nb * 8, dtype=torch.uint8, device="cuda")
            scales = torch.empty(nb, dtype=torch.uint8, device="cuda")
            for win in ((-2, 6), (-8, 8)):
                row = []
                for _, bounds in shapes:
                    nv.search_policy(*bounds)
                    row.append(graph_us(lambda: nv.quantize_ex(x, *win, gscale_in=g, want_f=False, want_sse=False,
                                                               codes=codes, scales=scales)))
                print(f"{nb:7d} {str(win):8s} " + "  ".join(f"{t:12.2f}" for t in row), flush=True)
        k = torch.randn(8, 64, 128, device="cuda").to(torch.bfloat16)
        g = (k.float().abs().max() / 2688.0).reshape(1).contiguous()
        kc = torch.empty(8, 1024, 64, dtype=torch.uint8, device="cuda")
        ks = torch.empty(8, 1024, 8, dtype=torch.uint8, device="cuda")
        for name, bounds in shapes:
            nv.search_policy(*bounds)
            print(f"kv_append 16 tokens x 8 heads x 128 ({name}): "
                  f"{graph_us(lambda: nv.kv_append(k, 16, 16, g, kc, ks, 100)):.2f} us", flush=True)
    finally:
        nv.search_policy(*default)


if __name__ == "__main__":
    main()
