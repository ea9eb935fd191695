"""Expert parallelism's GPU stages on one GPU, through the C ABI, against the oracle:

  - moe_route: routing equal to the block's, the unpadded grouping exact (rows of an expert
    contiguous and stable, each grouped row a bit copy of its token's row);
  - moe_experts_forward + moe_combine: R = 2 and 4 ranks emulated on one GPU.  Each virtual
    rank routes its own batch; the exchange is done by slicing, with the splits of
    ExpertPartition (the NCCL all-to-alls themselves are covered on CPU ranks by
    tests/test_ep_exchange.py); each rank's local experts run on the rows received from every
    source; the outputs go back and are combined.  Every rank's output must meet the block's
    parity bars against the oracle;
  - moe_forward_ep without a process group (one rank) against the oracle."""
import numpy as np
import pytest
import torch

import moe_inputs
from tests import parity

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - these tests need a B200
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_mixture_experts_18_b200 as moe  # noqa: E402
from sparse_mixture_experts_18_b200 import ep  # noqa: E402


def _check_against_oracle(name, w, x, layer, out, idx, budget=None):
    xc = x.cpu()
    lc = {k: v.cpu() for k, v in layer.items()}
    idx_h = idx.cpu().numpy()
    logits, _, _ = parity.oracle.route(xc, lc["Wg"], w.n, w.K)
    exempt = [t for t in range(w.T) if parity.oracle.tie_band(logits[t], w.K, parity.TIE_REL)[0]]
    tokens = parity.sample_tokens(w.T, idx_h, exempt, w.n, budget or w.T)
    ref = parity.oracle_outputs(xc, lc["Wg"], lc["W1"], lc["W3"], lc["W2"], w.n, w.K, tokens,
                                idx_h, exempt)
    rep = parity.compare_outputs(out.float().cpu().numpy()[tokens], ref, x.dtype)
    rep.update(exempt=len(exempt), tokens=len(tokens))
    parity.record(name, rep)
    assert rep["ok"], rep


@pytest.mark.parametrize("w", [moe_inputs.small(T=12, d=256, F=384),
                               moe_inputs.small(T=700, d=320, F=448, n=16, K=3),
                               moe_inputs.small(T=90, d=64, F=96, dtype="f32")],
                         ids=["one_launch_routing", "router_scan_permute", "fp32"])
def test_route_groups_rows_exactly(w):
    x = moe_inputs.make_x(w).cuda()
    L = {k: v.cuda() for k, v in moe_inputs.make_layer(w).items()}
    xg, idx, gate, counts, rows = moe.moe_route(x, L["Wg"], w.K)
    _, idx_ref, gate_ref, _, _, _ = moe.moe_forward_debug(x, L["Wg"], L["W1"], L["W3"], L["W2"],
                                                          w.K)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref) and torch.equal(gate, gate_ref)
    idx_h, counts_h, rows_h = idx.cpu().numpy(), counts.cpu().numpy(), rows.cpu().numpy()
    offsets = np.concatenate([[0], np.cumsum(counts_h)])
    parity.check_permutation(idx_h, counts_h, offsets, rows_h, w.n, w.K)
    assert offsets[-1] == w.T * w.K                      # unpadded
    tok = torch.arange(w.T, device="cuda").repeat_interleave(w.K)
    assert torch.equal(xg[rows.reshape(-1).long()], x[tok])


def _emulated_ep(ws, xs, layer, R):
    """The expert-parallel forward of R virtual ranks (batch xs[r] each) on one GPU, the
    exchanges done by slicing.  Returns (outputs, topk indices) per rank."""
    n, K = ws[0].n, ws[0].K
    parts = [ep.ExpertPartition(n, R, r) for r in range(R)]
    nl = parts[0].n_local
    routed = [moe.moe_route(x, layer["Wg"], K) for x in xs]      # (xg, idx, gate, counts, rows)
    counts = [r[3].cpu() for r in routed]
    send = [parts[s].send_splits(counts[s]) for s in range(R)]
    y_back_parts = [[None] * R for _ in range(R)]
    for q in range(R):                                           # virtual rank q's experts
        seg = torch.stack([counts[s][q * nl:(q + 1) * nl] for s in range(R)]).to(torch.int32)
        x_recv = torch.cat([routed[s][0][sum(send[s][:q]):sum(send[s][:q + 1])]
                            for s in range(R)])
        e = slice(q * nl, (q + 1) * nl)
        y_recv = moe.moe_experts_forward(x_recv, seg.cuda(), layer["W1"][e].contiguous(),
                                         layer["W3"][e].contiguous(),
                                         layer["W2"][e].contiguous())
        recv = ep.ExpertPartition.recv_splits(seg)
        for s in range(R):
            y_back_parts[s][q] = y_recv[sum(recv[:s]):sum(recv[:s + 1])]
    outs = []
    for s in range(R):
        y_back = torch.cat(y_back_parts[s])
        out = torch.empty_like(xs[s])
        moe.moe_combine(y_back, routed[s][4], routed[s][2], out)
        outs.append(out)
    torch.cuda.synchronize()
    return outs, [r[1] for r in routed]


@pytest.mark.parametrize("R,T,d,F,n,K,dtype", [
    (2, 40, 256, 384, 8, 2, "bf16"),       # small batches on every rank's local stage
    (2, 700, 256, 384, 8, 2, "bf16"),      # mid-size tiles locally
    (4, 1500, 256, 384, 8, 2, "bf16"),     # CTA-pair tiles locally (2 experts per rank)
    (2, 64, 64, 96, 8, 2, "f32"),          # fp32 SIMT path
    (4, 333, 320, 448, 16, 3, "bf16"),     # n = 16 over 4 ranks, K = 3, ragged d and F
])
def test_emulated_expert_parallel_forward(R, T, d, F, n, K, dtype):
    ws = [moe_inputs.small(name=f"ep{R}_rank{r}", T=T + 17 * r, d=d, F=F, n=n, K=K,
                           dtype=dtype, seed=10 + r) for r in range(R)]
    layer = {k: v.cuda() for k, v in moe_inputs.make_layer(ws[0].replace(seed=3)).items()}
    xs = [moe_inputs.make_x(w).cuda() for w in ws]
    outs, idxs = _emulated_ep(ws, xs, layer, R)
    for r in range(R):
        _check_against_oracle(f"EP x{R} rank {r}: T={ws[r].T} d={d} F={F} n={n} K={K} {dtype}",
                              ws[r], xs[r], layer, outs[r], idxs[r])


def test_emulated_expert_parallel_mixtral_shapes():
    """Two virtual ranks of 2048 tokens each at Mixtral's widths (4 experts per rank)."""
    base = moe_inputs.WORKLOADS["prefill_t4096"]
    ws = [base.replace(name=f"ep2_rank{r}", T=2048, seed=20 + r) for r in range(2)]
    layer = moe_inputs.make_layer(ws[0].replace(seed=0), device="cuda")
    xs = [moe_inputs.make_x(w, device="cuda") for w in ws]
    outs, idxs = _emulated_ep(ws, xs, layer, 2)
    for r in range(2):
        _check_against_oracle(f"EP x2 rank {r}: Mixtral shapes T=2048", ws[r], xs[r], layer,
                              outs[r], idxs[r], budget=48)


def _emulated_ep_placed(ws, xs, layer, R, slots):
    """As _emulated_ep with hot experts replicated (ExpertPlacement.balanced over the global
    loads): each source's grouped rows go into destination order with moe_gather_rows, each
    rank runs its experts (replicas included) on the parts it receives, and the returned rows
    go back into grouped order with moe_gather_rows before the combine."""
    n, K = ws[0].n, ws[0].K
    routed = [moe.moe_route(x, layer["Wg"], K) for x in xs]     # (xg, idx, gate, counts, rows)
    all_counts = torch.stack([r[3] for r in routed]).cpu()
    pl = ep.ExpertPlacement.balanced(all_counts.sum(dim=0), R, slots)
    plans = [pl.send_order(all_counts[s]) for s in range(R)]
    perms = [torch.tensor(o, dtype=torch.int32, device="cuda") for o, _ in plans]
    x_send = [moe.moe_gather_rows(routed[s][0], perms[s]) for s in range(R)]
    starts = [[sum(plans[s][1][:q]) for q in range(R + 1)] for s in range(R)]
    y_parts = [[None] * R for _ in range(R)]
    for q in range(R):
        local = pl.local_experts(q)
        seg = torch.tensor(pl.recv_counts(all_counts, q), dtype=torch.int32)
        x_recv = torch.cat([x_send[s][starts[s][q]:starts[s][q + 1]] for s in range(R)])
        idx = torch.tensor(local, device="cuda")
        y_recv = moe.moe_experts_forward(x_recv, seg.cuda(), layer["W1"][idx].contiguous(),
                                         layer["W3"][idx].contiguous(),
                                         layer["W2"][idx].contiguous())
        off = 0
        for s in range(R):
            c = int(seg[s].sum())
            y_parts[s][q] = y_recv[off:off + c]
            off += c
    outs = []
    for s in range(R):
        y_send_back = torch.cat(y_parts[s])
        inv = torch.empty_like(perms[s])
        inv[perms[s].long()] = torch.arange(len(perms[s]), dtype=torch.int32, device="cuda")
        y_back = moe.moe_gather_rows(y_send_back, inv)
        out = torch.empty_like(xs[s])
        moe.moe_combine(y_back, routed[s][4], routed[s][2], out)
        outs.append(out)
    torch.cuda.synchronize()
    return outs, [r[1] for r in routed], pl


@pytest.mark.parametrize("R,T,n,slots", [(2, 700, 8, 6), (4, 333, 8, 3), (4, 1500, 8, 4)])
def test_emulated_expert_parallel_with_replicas(R, T, n, slots):
    ws = [moe_inputs.small(name=f"epr{R}_rank{r}", T=T + 13 * r, d=256, F=384, n=n, K=2,
                           seed=40 + r) for r in range(R)]
    layer = {k: v.cuda() for k, v in moe_inputs.make_layer(ws[0].replace(seed=5)).items()}
    xs = [moe_inputs.make_x(w).cuda() for w in ws]
    outs, idxs, pl = _emulated_ep_placed(ws, xs, layer, R, slots)
    assert any(len(r) > 1 for r in pl.replicas)
    for r in range(R):
        _check_against_oracle(f"EP x{R} replicated ({slots} slots) rank {r}: T={ws[r].T}",
                              ws[r], xs[r], layer, outs[r], idxs[r])


def test_gather_rows():
    g = torch.Generator().manual_seed(2)
    src = torch.randn(300, 64, generator=g).cuda()
    index = torch.randint(0, 300, (500,), generator=g, dtype=torch.int32).cuda()
    index[7] = -1                                   # out of range: row left unwritten
    index[9] = 300
    out = torch.full((500, 64), 7.0, device="cuda")
    moe.moe_gather_rows(src, index, out=out)
    torch.cuda.synchronize()
    ok = index.long().clamp(0, 299)
    ref = src[ok]
    ref[7] = 7.0
    ref[9] = 7.0
    assert torch.equal(out, ref)
    xb = torch.randn(10, 4096, generator=g).to(torch.bfloat16).cuda()
    assert torch.equal(moe.moe_gather_rows(xb, torch.tensor([9, 0, 3], dtype=torch.int32,
                                                            device="cuda")), xb[[9, 0, 3]])


@pytest.mark.parametrize("w", [moe_inputs.small(T=200, d=256, F=384),
                               moe_inputs.WORKLOADS["decode_t16"]], ids=["small", "decode_t16"])
def test_forward_ep_single_rank(w):
    x = moe_inputs.make_x(w, device="cuda")
    L = moe_inputs.make_layer(w, device="cuda")
    out = ep.moe_forward_ep(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K)
    ref = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K)
    torch.cuda.synchronize()
    rep = parity.compare_outputs(out.float().cpu().numpy(), ref.double().cpu().numpy(), x.dtype)
    assert rep["ok"], rep
    _, idx, _, _, _ = moe.moe_route(x, L["Wg"], w.K)
    _check_against_oracle(f"EP x1: {w.name} T={w.T}", w, x, L, out, idx)


def test_forward_ep_placed_single_rank():
    """The placement path of moe_forward_ep on one rank (counts all-gather, row gathers, the
    local experts, combine) against moe_forward and the oracle."""
    w = moe_inputs.small(T=300, d=256, F=384)
    x = moe_inputs.make_x(w, device="cuda")
    L = moe_inputs.make_layer(w, device="cuda")
    pl = ep.ExpertPlacement.contiguous(w.n, 1)
    out = ep.moe_forward_ep(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K, placement=pl)
    ref = moe.moe_forward(x, L["Wg"], L["W1"], L["W3"], L["W2"], w.K)
    torch.cuda.synchronize()
    rep = parity.compare_outputs(out.float().cpu().numpy(), ref.double().cpu().numpy(), x.dtype)
    assert rep["ok"], rep
    _, idx, _, _, _ = moe.moe_route(x, L["Wg"], w.K)
    _check_against_oracle(f"EP x1 placed: T={w.T}", w, x, L, out, idx)

