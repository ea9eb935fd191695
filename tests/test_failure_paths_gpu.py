"""Failure detection on the GPU, without faulting it: the device status word and the
bounded pipeline waits of the one-CTA tensor-core kernel.

  - Status word: bits planted in a workspace's status word by the test (as a kernel would
    set them) come back from moe_workspace_status as MOE_ERR_TIMEOUT / MOE_ERR_DEVICE with
    the raw mask, and the word reads zero afterwards.
  - Bounded wait: moe_debug_forward_withheld makes the gate/up kernel issue none of its
    loads, so its tensor-core thread waits on a barrier that nothing will complete.  The wait
    runs out after a short limit (about a millisecond), the kernel records the timeout,
    unwinds (nothing in flight, tensor memory freed) and returns; the status call reports
    MOE_ERR_TIMEOUT, and after moe_workspace_init the same workspace gives results bit for
    bit equal to a clean run, so the context and the library stay usable."""
import pytest
import torch

import moe_inputs

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - these tests need a B200
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_mixture_experts_18_b200 as moe  # noqa: E402

MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE, MOE_ERR_UNSUPPORTED = 0, 5, 6, 2
DEV_ERR_TIMEOUT, DEV_ERR_EXPERT, DEV_ERR_ROW = 1, 2, 4
SHORT_LIMIT = 2_000_000   # SM clock cycles: about 1 ms at 2 GHz


def _plant(ws: torch.Tensor, bits: int):
    ws[:4].copy_(torch.tensor([bits], dtype=torch.int32).view(torch.uint8).to(ws.device))


@pytest.mark.parametrize("bits,code", [(DEV_ERR_TIMEOUT, MOE_ERR_TIMEOUT),
                                       (DEV_ERR_EXPERT, MOE_ERR_DEVICE),
                                       (DEV_ERR_ROW, MOE_ERR_DEVICE),
                                       (DEV_ERR_TIMEOUT | DEV_ERR_ROW, MOE_ERR_TIMEOUT)])
def test_status_word_is_reported_and_cleared(bits, code):
    ws = moe.alloc_workspace(4096)
    _plant(ws, bits)
    assert moe.moe_workspace_status(ws) == (code, bits)
    assert moe.moe_workspace_status(ws) == (MOE_OK, 0)


@pytest.mark.parametrize("T", [16, 400, 2000], ids=["small_batch", "mid_size", "128_row_tiles"])
def test_withheld_loads_time_out_and_the_workspace_recovers(T):
    w = moe_inputs.small(T=T, d=256, F=384)
    plan = moe.moe_plan_info(w.T, w.d, w.F, w.n, w.K)
    assert not plan["pair"] and plan["small_batch"] == (T == 16) and plan["mid"] == (T == 400)
    x = moe_inputs.make_x(w).cuda()
    L = {k: v.cuda() for k, v in moe_inputs.make_layer(w).items()}
    nbytes = moe.moe_workspace_bytes(w.T, w.d, w.F, w.n, w.K, torch.bfloat16)
    clean = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K,
                            workspace=moe.alloc_workspace(nbytes))
    ws = moe.alloc_workspace(nbytes)
    moe.moe_debug_forward_withheld(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, SHORT_LIMIT,
                                   workspace=ws)
    code, raw = moe.moe_workspace_status(ws)
    assert code == MOE_ERR_TIMEOUT and raw & DEV_ERR_TIMEOUT, (code, raw)
    moe.lib().moe_workspace_init(ws.data_ptr(), ws.numel(), None)
    for _ in range(2):
        again = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, workspace=ws)
        assert moe.moe_workspace_status(ws) == (MOE_OK, 0)
        assert torch.equal(again, clean)


def test_withheld_loads_hook_refuses_other_kernels():
    w = moe_inputs.small(T=2600, d=256, F=384)           # CTA-pair tiling
    assert moe.moe_plan_info(w.T, w.d, w.F, w.n, w.K)["pair"]
    x = torch.zeros((w.T, w.d), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros((w.d, w.n), dtype=torch.float32, device="cuda")
    w13 = torch.zeros((w.n, 1, w.d), dtype=torch.bfloat16, device="cuda")  # never read
    out = torch.empty_like(x)
    code = moe.lib().moe_debug_forward_withheld(
        x.data_ptr(), wg.data_ptr(), w13.data_ptr(), w13.data_ptr(), w13.data_ptr(), w.T, w.d,
        w.F, w.n, w.K, moe.MOE_BF16, out.data_ptr(), out.data_ptr(), 1 << 30, None, SHORT_LIMIT)
    assert code == MOE_ERR_UNSUPPORTED
