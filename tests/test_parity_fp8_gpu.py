"""GPU parity of the FP8-weight variant (MXFP8: E4M3 expert weights with an E8M0 scale per
32 elements, on the small-batch decode path) against the oracle's FP8 block: quantisation
codes and block scales bit for bit, block outputs within the bf16 bars."""
import numpy as np
import pytest
import torch

import moe_inputs
from tests import parity

pytestmark = pytest.mark.gpu

cuda = pytest.importorskip("torch").cuda
if not cuda.is_available():  # pragma: no cover - these tests need a B200
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_mixture_experts_18_b200 as moe  # noqa: E402


def _quantize_layer(L, n, F, d):
    W1q, s1 = moe.moe_quantize_mx_e4m3(L["W1"])
    W3q, s3 = moe.moe_quantize_mx_e4m3(L["W3"])
    W2q, s2 = moe.moe_quantize_mx_e4m3(L["W2"])
    return W1q, W3q, W2q, s1, s3, s2


_plain_scales = parity.plain_scales


def _run_fp8(w, gen_device="cpu", budget=None):
    x = moe_inputs.make_x(w, device=gen_device)
    layer = moe_inputs.make_layer(w, device=gen_device)
    xd = x.cuda()
    L = {k: v.cuda() for k, v in layer.items()}
    W1q, W3q, W2q, s1, s3, s2 = _quantize_layer(L, w.n, w.F, w.d)
    out = moe.moe_forward_fp8(xd, L["Wg"], W1q, W3q, W2q, s1, s3, s2, w.K)
    torch.cuda.synchronize()
    xc = x.cpu()
    wg = layer["Wg"].cpu()
    n, F, d = w.n, w.F, w.d
    q = [t.cpu().numpy() for t in (W1q, W3q, W2q)]
    q += [_plain_scales(s1.cpu().numpy(), n * F, d).reshape(n, F, d // 32),
          _plain_scales(s3.cpu().numpy(), n * F, d).reshape(n, F, d // 32),
          _plain_scales(s2.cpu().numpy(), n * d, F).reshape(n, d, F // 32)]
    del L
    logits, _, _ = parity.oracle.route(xc, wg, w.n, w.K)
    exempt = {t for t in range(w.T) if parity.oracle.tie_band(logits[t], w.K,
                                                               parity.TIE_REL)[0]}
    tokens = [t for t in range(w.T) if t not in exempt]
    if budget is not None:
        tokens = tokens[:budget]
    y, _, _ = parity.oracle.moe_forward_fp8(xc, wg, *q, w.n, w.K, tokens=tokens)
    ref = parity.oracle.round_array(y, parity.oracle.BF16)
    got = out.float().cpu().numpy()[tokens]
    rep = parity.compare_outputs(got, ref, torch.bfloat16)
    rep.update(exempt=len(exempt), tokens=len(tokens))
    assert rep["ok"], rep
    return rep


def test_quantize_mx_bit_exact():
    # codes and block scales against the oracle's quantiser, bit for bit: rows of very
    # different magnitudes (tiny, subnormal-range, huge, all-zero), a block whose maximum is a
    # power of two, and a dominant element that saturates its block's other codes' range
    g = torch.Generator().manual_seed(5)
    scales = torch.tensor([1e-4, 0.01, 1.0, 7.0, 300.0, 0.0, 1e3, 2.5, 2.0 ** -125, 1e30])
    v = (torch.randn(256, 1024, generator=g) * scales.repeat(26)[:256, None]).to(torch.bfloat16)
    v[3, 17] = -v[3, 17].abs().max() * 4
    v[7, 64:96] = torch.linspace(-2, 2, 32).to(torch.bfloat16)
    q, sf = moe.moe_quantize_mx_e4m3(v.cuda())
    torch.cuda.synchronize()
    qo, so = parity.oracle.quantize_mx_e4m3(v)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(_plain_scales(sf.cpu().numpy(), 256, 1024), so)


@pytest.mark.parametrize("T", [1, 5, 16, 32, 33, 37, 64])   # 32 / 33: the 32-slot boundary
def test_fp8_small_batch(T):
    _run_fp8(moe_inputs.small(T=T, d=512, F=768))


@pytest.mark.parametrize("n,K", [(16, 4), (64, 2), (1, 1), (8, 1)])
def test_fp8_expert_counts(n, K):
    _run_fp8(moe_inputs.small(T=12, d=256, F=384, n=n, K=K))


def test_fp8_minimal_widths():
    # d = F = 128: one K block per row, one scale chunk per tile
    _run_fp8(moe_inputs.small(T=9, d=128, F=128, n=4, K=2))


def test_fp8_one_launch_routing_at_its_limit():
    _run_fp8(moe_inputs.small(T=64, d=256, F=384, n=64, K=16))


def test_fp8_decode_t16_full():
    # Mixtral shapes: 1.4 GB of E4M3 expert weights instead of 2.8 GB of bf16
    rep = _run_fp8(moe_inputs.WORKLOADS["decode_t16"], gen_device="cuda")
    assert rep["tokens"] + rep["exempt"] == 16


def test_fp8_repeat_calls_bitwise():
    w = moe_inputs.small(T=16, d=512, F=768)
    x = moe_inputs.make_x(w).cuda()
    L = {k: v.cuda() for k, v in moe_inputs.make_layer(w).items()}
    qs = _quantize_layer(L, w.n, w.F, w.d)
    ws = moe.alloc_workspace(moe.moe_workspace_bytes_fp8(w.T, w.d, w.F, w.n, w.K))
    a = moe.moe_forward_fp8(x, L["Wg"], *qs, w.K, workspace=ws).clone()
    b = moe.moe_forward_fp8(x, L["Wg"], *qs, w.K, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert moe.moe_workspace_status(ws)[0] == 0


def test_fp8_decode_error_against_the_bf16_block():
    """How far the FP8 variant's output is from the exact block on the unquantised bf16
    weights (the oracle's bf16 block), on the Mixtral decode shape.  Reported in the run's
    parity summary.  E4M3's nearest rounding errs by at most 2^-4 relative (3 mantissa bits),
    about 0.02-0.03 RMS for values spread over the binade; four quantisations lie on the path
    (x, W1/W3, h, W2), so the expected relative L2 error is a few 1e-2.  The bar, 0.1, only
    catches a lost scale or a wrong code (errors of order 1)."""
    w = moe_inputs.WORKLOADS["decode_t16"]
    x = moe_inputs.make_x(w, device="cuda")
    L = moe_inputs.make_layer(w, device="cuda")
    qs = _quantize_layer(L, w.n, w.F, w.d)
    out = moe.moe_forward_fp8(x, L["Wg"], *qs, w.K)
    torch.cuda.synchronize()
    xc = x.cpu()
    lc = {k: v.cpu() for k, v in L.items()}
    del L, qs
    logits, idx, _ = parity.oracle.route(xc, lc["Wg"], w.n, w.K)
    ref = parity.oracle_outputs(xc, lc["Wg"], lc["W1"], lc["W3"], lc["W2"], w.n, w.K,
                                np.arange(w.T), idx, [])
    err = out.float().cpu().numpy().astype(np.float64) - ref
    rep = {"tokens": w.T, "exempt": 0, "max_abs": float(np.max(np.abs(err))),
           "rel_l2": float(np.linalg.norm(err) / np.linalg.norm(ref)), "ok": True}
    rep["ok"] = rep["rel_l2"] <= 0.1
    parity.record("decode_t16 MXFP8 weights vs the bf16 block (error of the format)", rep)
    assert rep["ok"], rep
