"""Seeded synthetic inputs for the Mixtral sparse-MoE block, shared by the tests, the smoke
check and the benchmark.

This module only draws random numbers and shapes them into the distributions the workloads
call for; it holds none of the MoE block's arithmetic (no routing, no experts, no combine).
Both the CUDA library and the CPU oracle receive exactly the tensors made here.

Shapes follow "Mixtral of Experts" (arXiv 2401.04088), method section: hidden size 4096,
n = 8 SwiGLU experts of intermediate width 14336, top-2 routing, 32 layers.

Recipe (seed s, per-tensor sub-seeds x: s+0, W_g: s+1, W1: s+2, W3: s+3, W2: s+4; layer l of
the stack adds 1000*l):
  x   ~ N(0, 1); for the bf16 workloads each row is then RMS-normalised in fp32
        (x / sqrt(mean(x^2) + 1e-5)) and rounded to bf16;
  W_g ~ N(0, 1/d), always fp32, stored [d][n];
  W1, W3 ~ N(0, 1/d) stored [n][F][d];  W2 ~ N(0, 1/F) stored [n][d][F];
  the skewed workload sets x[:, 0] = 1 and W_g[0, e] = b_e, a per-expert bias column whose
  values (zipf_bias.json) were calibrated so that expert selection frequencies follow a
  Zipf(1.2) law (busiest expert about 3x the mean load).
Values are drawn in fp32 by torch's generator on the requested device (CPU: mt19937,
CUDA: Philox) and then cast; the same seed therefore gives different but equally
distributed tensors on the two device types.
"""
from __future__ import annotations

import dataclasses
import json
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    F: int
    n: int = 8
    K: int = 2
    dtype: str = "bf16"          # "bf16" or "f32": x, W1, W3, W2 and out
    rms_x: bool = True           # RMS-normalise x rows (bf16 workloads)
    zipf: float = 0.0            # > 0: per-expert bias column giving a Zipf(s) load skew
    layers: int = 1              # > 1: stack of RMSNorm -> MoE -> residual blocks
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw):
        return dataclasses.replace(self, **kw)


# The five workloads of the benchmark and parity suite, then variants of the expert count n
# and of K on the same hidden and expert widths (the paper's remark that n and K are free
# parameters of the layer): they move the rows per expert M_e = T*K/n down to ~128, where
# the expert GEMMs sit near the HBM/tensor ridge, and exercise grouping with many groups.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", T=64, d=128, F=256, dtype="f32", rms_x=False),
    "decode_t16": Workload("decode_t16", T=16, d=4096, F=14336),
    "prefill_t4096": Workload("prefill_t4096", T=4096, d=4096, F=14336),
    "skewed_t32768": Workload("skewed_t32768", T=32768, d=4096, F=14336, zipf=1.2),
    "stack32_t8192": Workload("stack32_t8192", T=8192, d=4096, F=14336, layers=32),
    "experts16_top1_t4096": Workload("experts16_top1_t4096", T=4096, d=4096, F=14336, n=16,
                                     K=1),
    "experts16_top4_t4096": Workload("experts16_top4_t4096", T=4096, d=4096, F=14336, n=16,
                                     K=4),
    "experts64_top2_t4096": Workload("experts64_top2_t4096", T=4096, d=4096, F=14336, n=64,
                                     K=2),
    "experts64_top4_t16": Workload("experts64_top4_t16", T=16, d=4096, F=14336, n=64, K=4),
    # the rows per expert of experts64_top2_t4096 (M_e = 128) on 8 experts: the mid-size
    # tiling at an eighth of the weights (a case small enough for full profiler captures)
    "experts8_top2_t512": Workload("experts8_top2_t512", T=512, d=4096, F=14336),
    # the rows per expert of experts16_top1_t4096 (M_e = 256) on 4 experts (profiler captures)
    "experts4_top1_t1024": Workload("experts4_top1_t1024", T=1024, d=4096, F=14336, n=4, K=1),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, seed, device, out_dtype, chunk_dim0=True):
    """N(0, std^2) in fp32, cast to out_dtype; drawn one leading slice at a time so that the
    fp32 temporary stays small for the large expert tensors."""
    g = _gen(device, seed)
    out = torch.empty(shape, dtype=out_dtype, device=device)
    if chunk_dim0 and len(shape) == 3:
        for e in range(shape[0]):
            out[e].copy_(torch.randn(shape[1:], generator=g, device=device,
                                     dtype=torch.float32).mul_(std))
    else:
        out.copy_(torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(std))
    return out


def zipf_bias(n: int = 8, s: float = 1.2):
    """Calibrated per-expert router bias b_e for the skewed workload (see zipf_bias.json)."""
    with open(os.path.join(_HERE, "zipf_bias.json")) as f:
        table = json.load(f)
    key = f"n{n}_s{s}"
    if key not in table:
        raise KeyError(f"no calibrated bias for {key}")
    return [float(v) for v in table[key]["bias"]]


def zipf_target_loads(T: int, n: int, K: int, s: float):
    """Rows each expert should receive under a Zipf(s) law: K*T*(e+1)^-s / H_{n,s}."""
    H = sum((e + 1) ** -s for e in range(n))
    return [K * T * (e + 1) ** -s / H for e in range(n)]


def make_x(w: Workload, device="cpu", T: int | None = None) -> torch.Tensor:
    """Token activations x [T][d] in the workload dtype."""
    T = w.T if T is None else T
    g = _gen(device, w.seed + 0)
    x = torch.randn((T, w.d), generator=g, device=device, dtype=torch.float32)
    if w.rms_x:
        x = x / torch.sqrt(x.pow(2).mean(dim=1, keepdim=True) + 1e-5)
    if w.zipf > 0:
        x[:, 0] = 1.0
    return x.to(w.torch_dtype).contiguous()


def make_layer(w: Workload, layer: int = 0, device="cpu", bias=None) -> dict:
    """Weights of one MoE block: W_g [d][n] fp32, W1/W3 [n][F][d], W2 [n][d][F]."""
    s = w.seed + 1000 * layer
    Wg = _normal((w.d, w.n), 1.0 / math.sqrt(w.d), s + 1, device, torch.float32)
    if w.zipf > 0:
        b = zipf_bias(w.n, w.zipf) if bias is None else bias
        Wg[0, :] = torch.tensor(b, dtype=torch.float32, device=device)
    W1 = _normal((w.n, w.F, w.d), 1.0 / math.sqrt(w.d), s + 2, device, w.torch_dtype)
    W3 = _normal((w.n, w.F, w.d), 1.0 / math.sqrt(w.d), s + 3, device, w.torch_dtype)
    W2 = _normal((w.n, w.d, w.F), 1.0 / math.sqrt(w.F), s + 4, device, w.torch_dtype)
    return {"Wg": Wg.contiguous(), "W1": W1, "W3": W3, "W2": W2}


def small(name="small", T=200, d=256, F=384, n=8, K=2, dtype="bf16", **kw) -> Workload:
    """A parity-sized workload (oracle finishes in seconds) with ragged tails."""
    return Workload(name, T=T, d=d, F=F, n=n, K=K, dtype=dtype,
                    rms_x=(dtype == "bf16") if "rms_x" not in kw else kw.pop("rms_x"), **kw)
