"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle, element by
element on the same seeded inputs.  Small cases span several tiles and ragged tails on both
the prefill tiling and the small-batch (swap-AB, split-K) tiling; full-size workloads are
checked on all tokens' routing and on sampled tokens' outputs."""
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


def _run(w: moe_inputs.Workload, gen_device="cpu", budget=None, layer_kw=None, x=None,
         layer=None):
    """Run one block on the GPU and compare with the oracle.  Every token's routing and the
    grouping are checked exactly; outputs on all tokens, or (budget < T) on a sample that has
    a row in every 128-row tile of every expert's group.  The workspace status word must read
    zero afterwards.  Returns a report dict (also printed in the run's summary)."""
    if x is None:
        x = moe_inputs.make_x(w, device=gen_device)
    if layer is None:
        layer = moe_inputs.make_layer(w, device=gen_device, **(layer_kw or {}))
    xd = x.cuda()
    L = {k: v.cuda() for k, v in layer.items()}
    ws = moe.alloc_workspace(moe.moe_workspace_bytes(w.T, w.d, w.F, w.n, w.K, x.dtype))
    out, idx, gate, counts, offsets, rows = moe.moe_forward_debug(
        xd, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, workspace=ws)
    ws_status = moe.moe_workspace_status(ws)
    assert ws_status == (0, 0), ws_status
    xc = x.cpu()
    lc = {k: v.cpu() for k, v in layer.items()}
    del L, xd, ws
    idx_h, gate_h = idx.cpu().numpy(), gate.cpu().numpy()
    counts_h, offsets_h, rows_h = counts.cpu().numpy(), offsets.cpu().numpy(), rows.cpu().numpy()
    logits, _, _ = parity.oracle.route(xc, lc["Wg"], w.n, w.K)
    exempt, errors = parity.check_routing(logits, idx_h, gate_h, w.K)
    assert not errors, errors[:5]
    parity.check_permutation(idx_h, counts_h, offsets_h, rows_h, w.n, w.K)
    tokens = parity.sample_tokens(w.T, idx_h, exempt, w.n, budget or w.T, rows=rows_h,
                                  offsets=offsets_h, counts=counts_h)
    ref = parity.oracle_outputs(xc, lc["Wg"], lc["W1"], lc["W3"], lc["W2"], w.n, w.K, tokens,
                                idx_h, exempt)
    got = out.float().cpu().numpy()[tokens]
    rep = parity.compare_outputs(got, ref, x.dtype)
    rep.update(exempt=len(exempt), tokens=len(tokens), counts=counts_h.tolist(),
               status=ws_status)
    parity.record(f"{w.name} T={w.T} d={w.d} F={w.F} n={w.n} K={w.K} {w.dtype}", rep)
    assert rep["ok"], rep
    return rep


# ------------------------------------------------------------------ small, ragged cases

def test_tiny_f32_full():
    rep = _run(moe_inputs.WORKLOADS["tiny_f32"])
    assert rep["tokens"] == 64


@pytest.mark.parametrize("T,d,F", [(1400, 320, 448), (2000, 256, 384), (1000, 512, 1024)])
def test_prefill_tiling_small(T, d, F):
    # 160 n < T*K < 640 n: the 128-row tile path; d % 256 and F % 128 ragged in the first case
    plan = moe.moe_plan_info(T, d, F, 8, 2)
    assert not (plan["small_batch"] or plan["pair"] or plan["mid"]), plan
    _run(moe_inputs.small(T=T, d=d, F=F), budget=400)


@pytest.mark.parametrize("T,d,F,n,K", [(300, 320, 448, 8, 2), (640, 256, 384, 8, 2),
                                       (600, 512, 1024, 8, 2), (600, 256, 384, 16, 1),
                                       (1024, 256, 384, 16, 2), (1000, 256, 256, 64, 2),
                                       (260, 192, 320, 5, 3), (150, 256, 384, 1, 1),
                                       (150, 256, 384, 4, 4), (300, 256, 384, 64, 1),
                                       (257, 192, 256, 2, 1)])
def test_mid_tiling(T, d, F, n, K):
    # 64 n <= T*K <= 160 n: weight-stationary tiles, each expert's rows (64 to 192 per pass,
    # from the mean group size) as the MMA's N, SwiGLU fused into the up-projection; ragged
    # d, F and pass tails; one expert (n = 1), every expert chosen (K = n), 64 experts with
    # about five rows each (many empty), T just above the small-batch bound
    plan = moe.moe_plan_info(T, d, F, n, K)
    assert plan["mid"] and not plan["small_batch"], plan
    _run(moe_inputs.small(T=T, d=d, F=F, n=n, K=K), budget=400)


@pytest.mark.parametrize("T", [500, 640])
def test_mid_tiling_skewed(T):
    # Zipf(1.2) routing over 8 experts: the largest group (~43% of the rows) takes three
    # passes over each weight block, the smallest (~4%) part of one
    w = moe_inputs.small(T=T, d=256, F=384, zipf=1.2)
    assert moe.moe_plan_info(w.T, w.d, w.F, w.n, w.K)["mid"]
    _run(w, budget=T)


@pytest.mark.parametrize("T,d,F,n,K", [(3000, 256, 384, 8, 2), (2700, 320, 448, 8, 2),
                                       (2600, 256, 256, 4, 1), (5200, 128, 256, 16, 2)])
def test_pair_tiling_small(T, d, F, n, K):
    # T*K >= 640*n: 256-row tiles on CTA pairs (cta_group::2); ragged d and F tails
    assert moe.moe_plan_info(T, d, F, n, K)["small_batch"] is False
    _run(moe_inputs.small(T=T, d=d, F=F, n=n, K=K))


@pytest.mark.parametrize("T,d,F,n,K", [(3000, 256, 384, 8, 2), (2700, 320, 448, 8, 2)])
def test_pair_tiling_gather_x(monkeypatch, T, d, F, n, K):
    # the alternative CTA-pair data path: A rows gathered from x by token (TMA gather4), gates
    # applied in the down-projection epilogue
    monkeypatch.setenv("MOE_GATHER_X", "1")
    _run(moe_inputs.small(T=T, d=d, F=F, n=n, K=K))


@pytest.mark.parametrize("T", [2600])
def test_all_tokens_to_two_experts_gather_x(monkeypatch, T):
    monkeypatch.setenv("MOE_GATHER_X", "1")
    test_all_tokens_to_two_experts(T)


@pytest.mark.parametrize("T,d,n,K", [(1024, 4096, 8, 2), (1100, 4096, 8, 2), (2501, 4096, 8, 2),
                                     (1500, 256, 5, 2), (1300, 320, 12, 3), (1030, 512, 16, 8),
                                     (1100, 256, 32, 3), (1500, 512, 48, 2), (1024, 256, 64, 4),
                                     (1030, 64, 8, 2), (1100, 192, 8, 2), (4100, 8192, 8, 2)])
def test_router_tc_tiles(T, d, n, K):
    # the tensor-core router (T >= 1024, n <= 64, K <= 8): an exact multiple of its 128-token
    # tile, ragged last tiles, clusters splitting d (4 where d / 64 allows, 1 at d = 320), a
    # single and three K blocks (d = 64, 192), a wide d (8192), and accumulators of 16
    # (n = 5) to 192 (n = 64) columns; a narrow expert width keeps the oracle quick
    _run(moe_inputs.small(T=T, d=d, F=128, n=n, K=K), budget=300)


@pytest.mark.parametrize("T", [1, 5, 16, 37, 100, 255])
def test_small_batch_tiling(T):
    # T <= 256 and T*K < 64*n: weights as the 128-row MMA operand, split-K
    _run(moe_inputs.small(T=T, d=512, F=768))


@pytest.mark.parametrize("T,small,pair", [(64, True, False), (65, True, False),
                                           (255, True, False), (256, False, False),
                                           (1023, False, False), (1024, False, False),
                                           (2559, False, False), (2560, False, True)])
def test_path_selection_boundaries(T, small, pair):
    """Both sides of every tiling switch (n = 8, K = 2): the one-launch routing (T <= 64), the
    small-batch tiling (T*K < 64 n), the tensor-core router (T >= 1024) and the CTA pairs
    (T*K >= 640 n)."""
    w = moe_inputs.small(T=T, d=256, F=384)
    plan = moe.moe_plan_info(w.T, w.d, w.F, w.n, w.K)
    assert plan["small_batch"] == small and plan["pair"] == pair, plan
    _run(w, budget=200)


@pytest.mark.parametrize("n,K", [(8, 1), (4, 4), (16, 2), (64, 2), (1, 1), (32, 3)])
def test_expert_counts(n, K):
    _run(moe_inputs.small(T=333, d=256, F=256, n=n, K=K))
    _run(moe_inputs.small(T=24, d=256, F=256, n=n, K=K))


def test_one_launch_routing_at_its_limit():
    # T = 64 tokens x K = 16 of n = 64: 1024 (token, slot) entries, the most the one-launch
    # router takes; up to 64 tokens per expert in the gathered small-batch tiles
    w = moe_inputs.small(T=64, d=256, F=384, n=64, K=16)
    assert moe.moe_plan_info(w.T, w.d, w.F, w.n, w.K)["small_batch"] is True
    _run(w)


@pytest.mark.parametrize("T", [7, 200, 1100])
def test_f32_path_ragged(T):
    _run(moe_inputs.small(T=T, d=136, F=200, dtype="f32", rms_x=False))


def _biased_layer(w, bias):
    layer = moe_inputs.make_layer(w)
    layer["Wg"][0, :] = torch.tensor(bias, dtype=torch.float32)
    return layer


@pytest.mark.parametrize("T", [16, 900, 2600])
def test_all_tokens_to_two_experts(T):
    # T = 2600 takes the CTA-pair tiling: 2600 rows per expert are ten 256-row tiles and one
    # 128-row tile (M = 128), and six experts have no rows; T = 900 the 128-row tiling
    w = moe_inputs.small(T=T, d=256, F=384, zipf=0.0)
    x = moe_inputs.make_x(w)
    x[:, 0] = 1.0
    layer = _biased_layer(w, [0, 0, 0, 40.0, 0, 30.0, 0, 0])
    rep = _run(w, x=x, layer=layer)
    assert rep["counts"] == [0, 0, 0, T, 0, T, 0, 0]


def test_expert_with_no_tokens():
    w = moe_inputs.small(T=640, d=256, F=256)
    x = moe_inputs.make_x(w)
    x[:, 0] = 1.0
    layer = _biased_layer(w, [0, -50.0, 0, 0, 0, 0, -50.0, 0])
    rep = _run(w, x=x, layer=layer)
    assert rep["counts"][1] == 0 and rep["counts"][6] == 0


def test_exact_ties_pick_lowest_index():
    w = moe_inputs.small(T=40, d=128, F=128)
    x = moe_inputs.make_x(w)
    layer = moe_inputs.make_layer(w)
    layer["Wg"][:] = layer["Wg"][:, :1]          # identical columns: every logit ties
    xd = x.cuda()
    L = {k: v.cuda() for k, v in layer.items()}
    out, idx, gate, counts, _, _ = moe.moe_forward_debug(xd, L["Wg"], L["W1"], L["W3"], L["W2"],
                                                         w.K)
    assert torch.all(idx.cpu() == torch.tensor([0, 1], dtype=torch.int32))
    assert torch.all(gate.cpu() == 0.5)
    ref = parity.oracle_outputs(x, layer["Wg"], layer["W1"], layer["W3"], layer["W2"], w.n,
                                w.K, np.arange(w.T), idx.cpu().numpy(), [])
    assert parity.compare_outputs(out.float().cpu().numpy(), ref, x.dtype)["ok"]


def test_zero_tokens_is_noop():
    w = moe_inputs.small(T=8, d=128, F=128)
    layer = {k: v.cuda() for k, v in moe_inputs.make_layer(w).items()}
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    out = moe.moe_forward(x, layer["Wg"], layer["W1"], layer["W3"], layer["W2"], 2)
    assert out.shape == (0, 128)


def test_repeat_calls_same_workspace_bitwise():
    w = moe_inputs.small(T=300, d=256, F=384)
    x = moe_inputs.make_x(w).cuda()
    L = {k: v.cuda() for k, v in moe_inputs.make_layer(w).items()}
    ws = moe.alloc_workspace(moe.moe_workspace_bytes(w.T, w.d, w.F, w.n, w.K, torch.bfloat16))
    a = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, workspace=ws)
    b = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, workspace=ws)
    assert torch.equal(a, b)
    assert moe.moe_workspace_status(ws) == (0, 0)


def test_host_io_matches_device_path():
    w = moe_inputs.small(T=64, d=256, F=384)
    x = moe_inputs.make_x(w)
    L = {k: v.cuda() for k, v in moe_inputs.make_layer(w).items()}
    ws = moe.alloc_workspace(moe.moe_workspace_bytes(w.T, w.d, w.F, w.n, w.K, torch.bfloat16))
    ref = moe.moe_forward(x.cuda(), L["Wg"], L["W1"], L["W3"], L["W2"], w.K, workspace=ws)
    xh = x.pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    xd, od = torch.empty_like(ref), torch.empty_like(ref)
    moe.moe_forward_host_io(xh, xd, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, od, oh, ws)
    torch.cuda.synchronize()
    assert torch.equal(oh, ref.cpu())


def _stack_block_check(x_in, x_out_gpu, layer, n, K, eps=1e-5):
    """Teacher-forced check of one stacked block: the oracle's block x + MoE(RMSNorm(x)) on
    the GPU's own input rows x_in (bf16 values, float64 array) against the GPU's output rows.
    Near-tie tokens of this block's own logits (1e-4 relative) are compared with the oracle's
    output for the admissible expert set closest to the GPU's result.  Bars: the bf16 bars,
    with the per-element allowance of 2^-7 |ref| of the residual stream."""
    lc = {k: v.cpu() for k, v in layer.items()}
    ref, _, _ = parity.oracle.block_forward(x_in, lc["Wg"], lc["W1"], lc["W3"], lc["W2"], n, K,
                                            eps)
    xn = parity.oracle.rmsnorm(x_in, eps, parity.oracle.BF16)
    xn_t = torch.from_numpy(xn).to(torch.bfloat16)
    logits, _, _ = parity.oracle.route(xn_t, lc["Wg"], n, K)
    exempt = 0
    for r in range(x_in.shape[0]):
        is_ex, sets = parity.oracle.tie_band(logits[r], K, parity.TIE_REL)
        if not is_ex:
            continue
        exempt += 1
        best = None
        for S in sets:
            y = parity.oracle.moe_token_with_experts(xn_t[r:r + 1], lc["Wg"], lc["W1"], lc["W3"],
                                                     lc["W2"], n, 0, list(S))
            cand = parity.oracle.round_array(x_in[r] + y, parity.oracle.BF16)
            err = float(np.max(np.abs(cand - x_out_gpu[r])))
            if best is None or err < best[0]:
                best = (err, cand)
        ref[r] = best[1]
    rep = parity.compare_outputs(x_out_gpu, ref, torch.bfloat16, stacked=True)
    rep.update(exempt=exempt, tokens=x_in.shape[0])
    return rep


def _stack_teacher_forced(w, x, layers, tokens):
    """One call over all L blocks, and L one-block calls keeping each block's input and output
    rows of `tokens`: the two must agree bit for bit, and every block must pass the
    teacher-forced check.  Returns the per-block reports."""
    x_all = x.clone()
    moe.moe_stack_forward(x_all, layers, w.K)
    xs = x.clone()
    ws = moe.alloc_workspace(moe.moe_stack_workspace_bytes(w.T, w.d, w.F, w.n, w.K))
    tok = torch.as_tensor(tokens, device="cuda")
    ins, outs = [], []
    for l in range(len(layers)):
        ins.append(xs[tok].float().cpu().numpy().astype(np.float64))
        moe.moe_stack_forward(xs, layers[l:l + 1], w.K, workspace=ws)
        outs.append(xs[tok].float().cpu().numpy().astype(np.float64))
    assert moe.moe_workspace_status(ws) == (0, 0)
    torch.cuda.synchronize()
    assert torch.equal(x_all, xs), "one call over L blocks differs from L one-block calls"
    assert torch.isfinite(xs.float()).all()
    del x_all, xs, ws
    reports = []
    for l in range(len(layers)):
        rep = _stack_block_check(ins[l], outs[l], layers[l], w.n, w.K)
        parity.record(f"{w.name} block {l + 1}/{len(layers)} (teacher-forced)", rep)
        reports.append(rep)
    bad = [(l + 1, r) for l, r in enumerate(reports) if not r["ok"]]
    assert not bad, bad
    return reports


def test_stack_host_io_and_profiled_match_the_device_path():
    """moe_stack_forward_host_io (host x in, host out) and moe_stack_forward_profiled (stage
    events of every block) give the stack's result bit for bit."""
    w = moe_inputs.small(T=300, d=256, F=512, layers=3)
    x = moe_inputs.make_x(w)
    layers = [{k: v.cuda() for k, v in moe_inputs.make_layer(w, layer=l).items()}
              for l in range(w.layers)]
    ref = x.cuda()
    moe.moe_stack_forward(ref, layers, w.K)
    xh = x.pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(ref)
    moe.moe_stack_forward_host_io(xh, xd, layers, w.K, oh)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6 * w.layers)]
    for e in evs:
        e.record()
    xp = x.cuda()
    moe.moe_stack_forward_profiled(xp, layers, w.K, evs)
    torch.cuda.synchronize()
    assert torch.equal(oh, ref.cpu())
    assert torch.equal(xp, ref)
    for b in range(w.layers):
        g13 = evs[6 * b + 1].elapsed_time(evs[6 * b + 2])
        assert g13 > 0.0


@pytest.mark.parametrize("T", [300, 1100])
def test_stack_small(T):
    """Four stacked blocks (RMSNorm -> MoE -> residual), every token of every block checked
    against the oracle block on the GPU's own input.  At T = 1100 the combine also writes the
    next block's RMSNorm (the fused path), which must equal the separate RMSNorm bit for bit
    (one 4-block call against four 1-block calls)."""
    w = moe_inputs.small(T=T, d=256, F=512, layers=4)
    x = moe_inputs.make_x(w).cuda()
    layers = [{k: v.cuda() for k, v in moe_inputs.make_layer(w, layer=l).items()}
              for l in range(w.layers)]
    _stack_teacher_forced(w, x, layers, np.arange(w.T))


# ------------------------------------------------------------------ full-size workloads

def test_decode_t16_full():
    rep = _run(moe_inputs.WORKLOADS["decode_t16"])
    assert rep["tokens"] == 16


def test_prefill_t4096_sampled():
    rep = _run(moe_inputs.WORKLOADS["prefill_t4096"], gen_device="cuda", budget=24)
    assert rep["tokens"] >= 64          # a row in each of the 64+ 128-row tiles


def test_skewed_t32768_sampled():
    w = moe_inputs.WORKLOADS["skewed_t32768"]
    rep = _run(w, gen_device="cuda", budget=16)
    c = np.array(rep["counts"])
    assert c[0] > 2.5 * c.mean(), c   # busiest expert about 3x the mean load
    assert rep["tokens"] >= 512         # a row in each of the 512+ 128-row tiles


@pytest.mark.parametrize("name", ["experts16_top1_t4096", "experts16_top4_t4096",
                                  "experts64_top2_t4096", "experts64_top4_t16",
                                  "experts8_top2_t512", "experts4_top1_t1024"])
def test_expert_count_variants_full_size(name):
    """n = 16 / 64 experts with K = 1 / 2 / 4 at Mixtral's hidden and expert widths: every
    token's routing, the grouping, and sampled tokens' outputs."""
    w = moe_inputs.WORKLOADS[name]
    rep = _run(w, gen_device="cuda", budget=16)
    assert sum(rep["counts"]) == w.T * w.K


def test_stack32_t8192_teacher_forced():
    """32 blocks of Mixtral shape on T=8192 tokens (~90 GB of bf16 expert weights on the
    device).  The residual stream amplifies sub-ulp differences from block to block, so each
    block is checked on its own: 64 sampled tokens' GPU input rows of block l go through the
    oracle's block l and must match the GPU's output rows at the bf16 bars (plus the
    residual stream's per-element allowance), with near-ties of that block's logits taken
    from its own input.  One 32-block call must equal 32 one-block calls bit for bit."""
    w = moe_inputs.WORKLOADS["stack32_t8192"]
    x = moe_inputs.make_x(w, device="cuda")
    layers = [moe_inputs.make_layer(w, layer=l, device="cuda") for l in range(w.layers)]
    rng = np.random.default_rng(5)
    tokens = np.unique(np.concatenate([np.linspace(0, w.T - 1, 32).astype(np.int64),
                                       rng.integers(0, w.T, 40)]))[:64]
    assert len(tokens) == 64
    reports = _stack_teacher_forced(w, x, layers, tokens)
    assert len(reports) == 32
