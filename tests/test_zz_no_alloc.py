"""moe_forward_noalloc: the forward entry point for callers that cannot allocate device
memory (for instance a plugin whose host application owns every device allocation, or a loop
that must not call cudaMalloc because it can synchronise the device).  It runs the same
kernels as moe_forward on a workspace held in a fixed device array inside the library.

This file is collected last on purpose, so that a run stopping at its first failure has
already run every other test.  Each check makes two calls in a row, because the array keeps
the previous call's contents."""
import pytest
import torch

import moe_inputs
from tests import parity

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - these tests need a B200
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_mixture_experts_18_b200 as moe  # noqa: E402

MOE_ERR_WORKSPACE = 3


@pytest.mark.parametrize("w", [moe_inputs.small(T=16, d=256, F=384),
                               moe_inputs.small(T=200, d=256, F=384),
                               moe_inputs.WORKLOADS["decode_t16"]],
                         ids=["small_batch", "prefill_tiles", "mixtral_decode_t16"])
def test_noalloc_matches_moe_forward_on_two_calls(w):
    x = moe_inputs.make_x(w, device="cuda")
    L = moe_inputs.make_layer(w, device="cuda")
    ref = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K)
    torch.cuda.synchronize()
    ref64 = ref.double().cpu().numpy()
    for _ in range(2):
        out = torch.full_like(x, float("nan"))
        moe.moe_forward_noalloc(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, out=out)
        torch.cuda.synchronize()
        rep = parity.compare_outputs(out.float().cpu().numpy(), ref64, x.dtype)
        assert rep["ok"], rep


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
