"""bench.py's host-side legs on the CPU: the CPU-baseline leg's parity block (the oracle's
result for the tokens it timed, compared with a given GPU result) and the reference arm's
JSON line, whose workload label must be the GPU arm's."""
import argparse
import contextlib
import io
import json

import numpy as np
import torch

import bench
import moe_inputs
import oracle


def _stack_case():
    w = moe_inputs.small(T=40, d=128, F=256, layers=3)
    x = moe_inputs.make_x(w)
    layer = moe_inputs.make_layer(w)
    ref, _, _ = oracle.block_forward(x.double().numpy(), layer["Wg"], layer["W1"], layer["W3"],
                                     layer["W2"], w.n, w.K, 1e-5)
    return w, x, layer, torch.from_numpy(ref).float()


def test_cpu_baseline_parity_block_of_a_stack():
    w, x, layer, ref = _stack_case()
    base, par = bench.cpu_baseline(w, x, layer, 4, seconds=0.2, gpu_out=ref)
    assert base["kind"] == "oracle" and base["value"] > 0 and base["cores"] >= 1
    assert par["ok"] and par["max_abs"] == 0.0 and par["rel_l2"] == 0.0
    assert par["tokens"] >= 4 and par["exempt"] == 0
    bad = ref.clone()
    bad[:, 5] += 0.5                                    # a wrong column in every token
    _, par = bench.cpu_baseline(w, x, layer, 4, seconds=0.2, gpu_out=bad)
    assert not par["ok"] and abs(par["max_abs"] - 0.5) < 0.02


def test_cpu_baseline_parity_block_of_one_block():
    w = moe_inputs.small(T=24, d=128, F=128)
    x = moe_inputs.make_x(w)
    layer = moe_inputs.make_layer(w)
    y, _, _ = oracle.moe_forward(x, layer["Wg"], layer["W1"], layer["W3"], layer["W2"], w.n,
                                 w.K)
    ref = torch.from_numpy(oracle.round_array(y, oracle.BF16)).float()
    _, par = bench.cpu_baseline(w, x, layer, 4, seconds=0.2, gpu_out=ref)
    assert par["ok"] and par["max_abs"] == 0.0
    assert np.isclose(par["rel_l2"], 0.0)


def test_reference_arm_line_uses_the_gpu_arms_label():
    w, _, _, _ = _stack_case()
    args = argparse.Namespace(steps=2, warmup=3, cpu_tokens=4)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, w)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"]["workload"] == bench.workload_label(w)
    assert "bf16" in line["config"]["workload"] and "3 x (RMSNorm" in line["config"]["workload"]
    assert line["unit"] == "tokens/s" and line["metric"] == bench.METRIC
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
