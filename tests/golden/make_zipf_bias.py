"""Writes moe_inputs/zipf_bias.json: the per-expert router bias column b_e of the skewed
workload (T=32768, d=4096, n=8, K=2), calibrated so that expert selection frequencies follow
a Zipf(1.2) law (expert e gets K*T*(e+1)^-1.2 / H rows; the busiest about 3x the mean).

Only the oracle's router is used: x has feature 0 set to 1 and W_g[0, e] = b_e, so b_e
shifts expert e's logit; 30 fixed-point steps b_e += 0.5 * ln(target_e / count_e) from
b = 0 on the CPU-drawn sample of the workload.

    python -m tests.golden.make_zipf_bias
"""
import json
import math
import os

import numpy as np
import torch

import moe_inputs
import oracle

OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))),
                   "moe_inputs", "zipf_bias.json")


def calibrate(w: moe_inputs.Workload, steps: int = 30):
    x = moe_inputs.make_x(w)
    bias = [0.0] * w.n
    layer = moe_inputs.make_layer(w.replace(F=64), bias=bias)   # only W_g is used
    target = moe_inputs.zipf_target_loads(w.T, w.n, w.K, w.zipf)
    counts = None
    for _ in range(steps):
        layer["Wg"][0, :] = torch.tensor(bias, dtype=torch.float32)
        _, idx, _ = oracle.route(x, layer["Wg"], w.n, w.K)
        counts = np.bincount(idx.reshape(-1), minlength=w.n)
        bias = [b + 0.5 * math.log(t / max(c, 0.5)) for b, t, c in zip(bias, target, counts)]
        bias = [float(np.float32(b)) for b in bias]
    layer["Wg"][0, :] = torch.tensor(bias, dtype=torch.float32)
    _, idx, _ = oracle.route(x, layer["Wg"], w.n, w.K)
    counts = np.bincount(idx.reshape(-1), minlength=w.n)
    return bias, counts.tolist(), target


if __name__ == "__main__":
    w = moe_inputs.WORKLOADS["skewed_t32768"]
    bias, counts, target = calibrate(w)
    table = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            table = json.load(f)
    table[f"n{w.n}_s{w.zipf}"] = {
        "bias": bias, "achieved_counts_cpu_sample": counts,
        "target_counts": [round(t, 1) for t in target],
        "workload": f"T={w.T} d={w.d} n={w.n} K={w.K} seed={w.seed}",
        "made_by": "tests/golden/make_zipf_bias.py (oracle router only)"}
    with open(OUT, "w") as f:
        json.dump(table, f, indent=1)
    print(json.dumps(table, indent=1))
