"""moe_forward_noalloc: the forward entry point for callers that cannot allocate device
memory (for instance a plugin whose host application owns every device allocation, or a loop
that must not call cudaMalloc because it can synchronise the device).  It runs the same
kernels as moe_forward on a workspace held in a fixed device array inside the library.

This file is collected last on purpose, so that a run stopping at its first failure has
already run every other test.  Each check makes two calls in a row, because the array keeps
the previous call's contents; the status call for the array must read zero afterwards."""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

import moe_inputs
from tests import parity

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - these tests need a B200
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_mixture_experts_18_b200 as moe  # noqa: E402

MOE_ERR_WORKSPACE = 3
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [moe_inputs.small(T=16, d=256, F=384), moe_inputs.small(T=200, d=256, F=384),
         moe_inputs.small(T=50, d=64, F=96, dtype="f32"), moe_inputs.WORKLOADS["decode_t16"]]
IDS = ["small_batch", "prefill_tiles", "fp32_simt", "mixtral_decode_t16"]


def _inputs(w):
    x = moe_inputs.make_x(w, device="cuda")
    L = moe_inputs.make_layer(w, device="cuda")
    ref = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K)
    torch.cuda.synchronize()
    return x, L, ref.double().cpu().numpy()


@pytest.mark.parametrize("w", CASES, ids=IDS)
@pytest.mark.parametrize("side_stream", [False, True], ids=["current_stream", "side_stream"])
def test_noalloc_matches_moe_forward_on_two_calls(w, side_stream):
    x, L, ref64 = _inputs(w)
    s = torch.cuda.Stream() if side_stream else None   # torch's streams are non-blocking
    if s is not None:
        s.wait_stream(torch.cuda.current_stream())
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        if s is not None:
            out.record_stream(s)
            s.wait_stream(torch.cuda.current_stream())
        moe.moe_forward_noalloc(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, out=out, stream=s)
        assert moe.moe_noalloc_status(s) == (0, 0)
        rep = parity.compare_outputs(out.float().cpu().numpy(), ref64, x.dtype)
        assert rep["ok"], rep


def test_noalloc_first_call_on_a_side_stream_in_a_fresh_process():
    """The array's header is zeroed by the first call on the caller's stream: in a fresh
    process whose first library call is a noalloc call on a non-blocking stream, the result
    must still equal moe_forward's."""
    code = textwrap.dedent("""
        import sys, torch
        sys.path.insert(0, %r)
        import moe_inputs
        import sparse_mixture_experts_18_b200 as moe
        w = moe_inputs.small(T=16, d=256, F=384)
        x = moe_inputs.make_x(w, device="cuda")
        L = moe_inputs.make_layer(w, device="cuda")
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        outs = []
        with torch.cuda.stream(s):
            for _ in range(2):
                outs.append(moe.moe_forward_noalloc(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K,
                                                    stream=s))
        assert moe.moe_noalloc_status(s) == (0, 0)
        ref = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K)
        torch.cuda.synchronize()
        assert all(torch.equal(o, ref) for o in outs)
        print("fresh-process noalloc ok")
    """ % ROOT)
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "fresh-process noalloc ok" in res.stdout


def test_noalloc_rejects_shapes_beyond_its_workspace():
    w = moe_inputs.small(T=32, d=4096, F=14336)          # needs ~36 MB > 32 MiB
    assert moe.moe_workspace_bytes(w.T, w.d, w.F, w.n, w.K, torch.bfloat16) > 32 << 20
    x = torch.zeros((w.T, w.d), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros((w.d, w.n), dtype=torch.float32, device="cuda")
    w13 = torch.zeros((w.n, 1, w.d), dtype=torch.bfloat16, device="cuda")  # never read
    out = torch.empty_like(x)
    code = moe.lib().moe_forward_noalloc(
        x.data_ptr(), wg.data_ptr(), w13.data_ptr(), w13.data_ptr(), w13.data_ptr(), w.T, w.d,
        w.F, w.n, w.K, moe.MOE_BF16, out.data_ptr(), None)
    assert code == MOE_ERR_WORKSPACE
