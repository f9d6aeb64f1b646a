"""Format / error study on the synthetic workloads (GPU, through the library's kernels).

    python -m nvfp4_block_scaled_11_b200.error_study [--scale S] [--json PATH]

For every workload tensor (blocks along the innermost dimension) it quantizes and dequantizes with

* MXFP4: 32-element blocks, E8M0 power-of-two scales (the format "NVIDIAのFP4推論が50倍の効率を実現",
  超低精度推論を支えるアーキテクチャ, compares NVFP4 with: NVFP4 is said to reach 88 % lower
  quantization error than such power-of-two scaling);
* NVFP4 max-scaling (offset window {0});
* NVFP4 ScaleSearch with windows [-2, 6] and [-8, 8] ("Search your block floating-point scales!",
  ScaleSearch: search strategy)

and reports the mean squared error, the normalised absolute error mean|x_hat - x| / mean|x| (the
definition of the BEVFormer-on-B200 page, section 7), the reductions against MXFP4 and against
max-scaling, and how often the best offset over [-8, 8] lies outside [-2, 6].
Error sums run in float64 over chunks of the tensor.
"""
from __future__ import annotations

import argparse
import json

import torch

import nvfp4_block_scaled_11_b200 as nv
from nvfp4_block_scaled_11_b200 import workloads as W

CHUNK = 1 << 26


def _errors(x: torch.Tensor, xh: torch.Tensor):
    """(sum (xh - x)^2, sum |xh - x|, sum |x|) in float64."""
    se = ae = ax = 0.0
    xf, hf = x.reshape(-1), xh.reshape(-1)
    for i in range(0, xf.numel(), CHUNK):
        a = xf[i:i + CHUNK].double()
        d = hf[i:i + CHUNK].double() - a
        se += float((d * d).sum())
        ae += float(d.abs().sum())
        ax += float(a.abs().sum())
    return se, ae, ax


def study(name: str, scale: float = 1.0) -> dict:
    x = W.make(name, "cuda", scale).x.contiguous().reshape(-1)
    n = x.numel() - x.numel() % 32
    x = x[:n]
    rows = {}
    c, s = nv.mxfp4_quantize(x)
    xh = nv.mxfp4_dequantize(c, s, torch.float32)
    rows["MXFP4 (32, E8M0)"] = _errors(x, xh)
    del c, s, xh
    out_of_window = None
    for label, (lo, hi) in (("NVFP4 max-scaling {0}", (0, 0)), ("NVFP4 ScaleSearch [-2,6]", (-2, 6)),
                            ("NVFP4 ScaleSearch [-8,8]", (-8, 8))):
        codes, scales, g, bf, _ = nv.quantize_ex(x, lo, hi, want_f=(lo, hi) == (-8, 8), want_sse=False)
        xh = nv.dequantize(codes, scales, g, torch.float32)
        rows[label] = _errors(x, xh)
        if bf is not None:
            valid = bf != -128
            out_of_window = float(((bf < -2) | (bf > 6)).logical_and(valid).sum()) / max(1, int(valid.sum()))
        del codes, scales, g, bf, xh
    torch.cuda.empty_cache()
    res = {"workload": name, "elements": n, "formats": {}}
    mx = rows["MXFP4 (32, E8M0)"][0]
    base = rows["NVFP4 max-scaling {0}"][0]
    for label, (se, ae, ax) in rows.items():
        res["formats"][label] = {
            "mse": se / n, "norm_abs_err": ae / ax,
            "mse_lower_than_mxfp4": 1.0 - se / mx, "mse_lower_than_max_scaling": 1.0 - se / base,
        }
    res["best_offset_outside_[-2,6]_with_[-8,8]"] = out_of_window
    return res


def markdown(results: list[dict]) -> str:
    out = ["| workload | format | MSE | norm. abs. error | MSE vs MXFP4 | MSE vs max-scaling |",
           "|---|---|---|---|---|---|"]
    for r in results:
        for label, v in r["formats"].items():
            out.append(f"| {r['workload']} | {label} | {v['mse']:.4e} | {100 * v['norm_abs_err']:.2f} % | "
                       f"{-100 * v['mse_lower_than_mxfp4']:+.1f} % | {-100 * v['mse_lower_than_max_scaling']:+.1f} % |")
    out.append("")
    out.append("| workload | blocks whose best offset in [-8,8] lies outside [-2,6] |")
    out.append("|---|---|")
    for r in results:
        out.append(f"| {r['workload']} | {100 * r['best_offset_outside_[-2,6]_with_[-8,8]']:.2f} % |")
    return "\n".join(out)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--scale", type=float, default=1.0)
    ap.add_argument("--json", default=None)
    ap.add_argument("--workloads", default=",".join(W.NAMES))
    a = ap.parse_args()
    results = [study(name, a.scale) for name in a.workloads.split(",")]
    print(markdown(results))
    if a.json:
        with open(a.json, "w") as fh:
            json.dump(results, fh, indent=1)


if __name__ == "__main__":
    main()
