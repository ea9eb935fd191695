"""Pins for the CPU oracle: each check ties it to something other than itself -- closed
forms, brute force on tiny inputs, special cases that reduce to textbook formulas evaluated
with torch float64 library matmuls, and a hand-worked example.  Definitions pinned:
G(x) = Softmax(TopK(x . W_g)) and y = sum_i G(x)_i SwiGLU_i(x) ("Mixtral of Experts",
arXiv 2401.04088, method section), and the statement that experts with zero gate need not
be computed (Indonesian news summary, section on how the MoE layer is computed)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def _silu(z):
    return z * _sig(z)


def _rand(shape, std, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(dtype)


def _layer(T, d, F, n, seed=0, dtype=torch.float32):
    x = _rand((T, d), 1.0, seed, dtype)
    Wg = _rand((d, n), d ** -0.5, seed + 1)
    W1 = _rand((n, F, d), d ** -0.5, seed + 2, dtype)
    W3 = _rand((n, F, d), d ** -0.5, seed + 3, dtype)
    W2 = _rand((n, d, F), F ** -0.5, seed + 4, dtype)
    return x, Wg, W1, W3, W2


def _swiglu64(xt, W1e, W3e, W2e):
    """SwiGLU expert with torch float64 library matmuls (independent of the oracle's loops)."""
    a = W1e.double() @ xt.double()
    b = W3e.double() @ xt.double()
    return W2e.double() @ (torch.nn.functional.silu(a) * b)


# ------------------------------------------------------------------ rounding helpers

def test_round_bf16_matches_torch_rne(oracle_lib):
    # Every fp32 value is exact in double, so torch's fp32 -> bf16 (round to nearest even)
    # is the reference; include ties, subnormals and large values.
    vals = torch.cat([
        _rand((4000,), 1.0, 7), _rand((1000,), 1e-39, 8), _rand((1000,), 1e30, 9),
        torch.tensor([1.00390625, 1.01171875, -1.00390625, 2.0 ** -130, 3.0e38, 0.0]),
    ]).float()
    ref = vals.to(torch.bfloat16).double()
    got = torch.tensor([oracle_lib.round_bf16(float(v)) for v in vals], dtype=torch.float64)
    assert torch.equal(got, ref)


def test_round_bf16_ties_to_even(oracle_lib):
    assert oracle_lib.round_bf16(1.0 + 2.0 ** -8) == 1.0          # tie -> even (1.0)
    assert oracle_lib.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert oracle_lib.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7


def test_silu_closed_forms(oracle_lib):
    assert oracle_lib.silu(0.0) == 0.0
    assert oracle_lib.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    for z in (-5.0, -0.3, 0.7, 4.0):
        # silu(z) - silu(-z) = z  (since sig(z) + sig(-z) = 1)
        assert oracle_lib.silu(z) - oracle_lib.silu(-z) == pytest.approx(z, rel=1e-14)
    assert oracle_lib.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    z = torch.linspace(-8, 8, 101, dtype=torch.float64)
    ref = torch.nn.functional.silu(z)
    got = torch.tensor([oracle_lib.silu(float(v)) for v in z], dtype=torch.float64)
    assert torch.allclose(got, ref, rtol=1e-14, atol=1e-300)


# ------------------------------------------------------------------ router: logits, TopK, G

@pytest.mark.parametrize("n,K", [(8, 2), (8, 1), (6, 3), (5, 5), (16, 2)])
def test_router_brute_force(oracle_lib, n, K):
    T, d = 64, 24
    x = _rand((T, d), 1.0, 11 + n)
    Wg = _rand((d, n), d ** -0.5, 12 + K)
    logits, idx, gate = oracle_lib.route(x, Wg, n, K)
    ref_logits = (x.double() @ Wg.double()).numpy()
    assert np.allclose(logits, ref_logits, rtol=1e-13, atol=1e-13)
    for t in range(T):
        l = logits[t]
        # brute force: the chosen subset maximises the sum of kept logits (equivalently every
        # kept logit >= every dropped one); ties resolved towards lower indices.
        best = max(itertools.combinations(range(n), K),
                   key=lambda s: (sorted((l[i] for i in s), reverse=True),
                                  [-i for i in sorted(s)]))
        assert sorted(idx[t].tolist()) == sorted(best)
        assert len(set(idx[t].tolist())) == K
        # slot order: descending logit
        assert all(l[idx[t, k]] >= l[idx[t, k + 1]] for k in range(K - 1))
        # G = softmax of the kept logits
        kept = np.array([l[i] for i in idx[t]])
        ref = np.exp(kept - kept.max()) / np.exp(kept - kept.max()).sum()
        assert np.allclose(gate[t], ref, rtol=1e-14, atol=0)
        assert gate[t].sum() == pytest.approx(1.0, abs=1e-15)
        assert np.all(np.diff(gate[t]) <= 0) and gate[t][0] >= 1.0 / K - 1e-15


def test_gate_closed_form_k2(oracle_lib):
    T, d, n = 128, 32, 8
    x = _rand((T, d), 1.0, 21)
    Wg = _rand((d, n), d ** -0.5, 22)
    logits, idx, gate = oracle_lib.route(x, Wg, n, 2)
    for t in range(T):
        l1, l2 = logits[t, idx[t, 0]], logits[t, idx[t, 1]]
        assert gate[t, 0] == pytest.approx(_sig(l1 - l2), rel=1e-14)
        assert gate[t, 1] == pytest.approx(_sig(l2 - l1), rel=1e-13)
        assert gate[t, 0] >= 0.5


def test_router_exact_ties_lowest_index(oracle_lib):
    d, n = 4, 8
    x = torch.tensor([[1.0, 2.0, -1.0, 0.5]])
    Wg = torch.ones((d, n)) * 0.25                     # all logits equal
    _, idx, gate = oracle_lib.route(x, Wg, n, 2)
    assert idx[0].tolist() == [0, 1] and gate[0].tolist() == [0.5, 0.5]
    Wg2 = Wg.clone()
    Wg2[:, 5] = 0.5                                     # expert 5 strictly largest
    Wg2[:, 3] = 0.4                                     # 3 and 6 tie for second
    Wg2[:, 6] = 0.4
    _, idx, _ = oracle_lib.route(x, Wg2, n, 2)
    assert idx[0].tolist() == [5, 3]
    _, idx, _ = oracle_lib.route(x, Wg2, n, 3)
    assert idx[0].tolist() == [5, 3, 6]


def test_tie_band_helper(oracle_lib):
    ex, sets = oracle_lib.tie_band(np.array([3.0, 1.0, 2.0, 2.0 + 1e-6]), 2)
    assert ex and sorted(sets) == [(0, 2), (0, 3)]
    ex, sets = oracle_lib.tie_band(np.array([3.0, 1.0, 2.0, 2.5]), 2)
    assert not ex and sets == [(0, 3)]


# ------------------------------------------------------------------ experts and the block

def test_hand_worked_token(oracle_lib):
    with open(os.path.join(HERE, "golden", "hand_worked_token.json")) as f:
        g = json.load(f)
    x = torch.tensor(g["x"], dtype=torch.float32)
    Wg = torch.tensor(g["W_g_rows_d_by_n"], dtype=torch.float32)
    W1 = torch.tensor(g["W1_n_F_d"], dtype=torch.float32)
    W3 = torch.tensor(g["W3_n_F_d"], dtype=torch.float32)
    W2 = torch.tensor(g["W2_n_d_F"], dtype=torch.float32)
    n, K = g["dims"]["n"], g["dims"]["K"]
    env = {"sig": _sig, "silu": _silu}
    logits, idx, gate = oracle_lib.route(x, Wg, n, K)
    assert logits.tolist() == g["expected_logits"]
    assert idx.tolist() == g["expected_idx"]
    assert gate[0] == pytest.approx([eval(e, env) for e in g["expected_gate_expr"]], rel=1e-15)
    y, idx2, _ = oracle_lib.moe_forward(x, Wg, W1, W3, W2, n, K, round_h=False)
    assert idx2.tolist() == g["expected_idx"]
    assert y[0] == pytest.approx([eval(e, env) for e in g["expected_y_expr"]], rel=1e-14)
    yd = oracle_lib.moe_dense(x, Wg, W1, W3, W2, n, K, round_h=False)
    assert yd[0] == pytest.approx(y[0], rel=1e-15)


def test_identity_experts_reduce_to_silu_times_x(oracle_lib):
    # F = d and W1 = W3 = W2 = I: every expert gives silu(x) * x, and the gates sum to 1.
    T, d, n = 16, 32, 8
    x = _rand((T, d), 2.0, 31)
    Wg = _rand((d, n), d ** -0.5, 32)
    eye = torch.eye(d).expand(n, d, d).contiguous()
    y, _, _ = oracle_lib.moe_forward(x, Wg, eye, eye, eye, n, 2, round_h=False)
    ref = (torch.nn.functional.silu(x.double()) * x.double()).numpy()
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-15)


def test_single_expert_is_plain_ffn(oracle_lib):
    # n = 1, K = 1: the block is one SwiGLU FFN (gate 1).  d != F catches transposed W.
    T, d, F = 8, 24, 40
    x, Wg, W1, W3, W2 = _layer(T, d, F, 1, seed=41)
    y, idx, gate = oracle_lib.moe_forward(x, Wg, W1, W3, W2, 1, 1, round_h=False)
    assert np.all(idx == 0) and np.all(gate == 1.0)
    for t in range(T):
        ref = _swiglu64(x[t], W1[0], W3[0], W2[0]).numpy()
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-14)


def test_k_equals_n_is_dense_softmax_moe(oracle_lib):
    # K = n: G is the full softmax of the logits -- the textbook dense mixture.
    T, d, F, n = 6, 16, 20, 4
    x, Wg, W1, W3, W2 = _layer(T, d, F, n, seed=51)
    y, _, _ = oracle_lib.moe_forward(x, Wg, W1, W3, W2, n, n, round_h=False)
    G = torch.softmax(x.double() @ Wg.double(), dim=1)
    for t in range(T):
        ref = sum(G[t, e] * _swiglu64(x[t], W1[e], W3[e], W2[e]) for e in range(n)).numpy()
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-14)


def test_top2_matches_library_reference(oracle_lib):
    # K = 2 of 8 against torch float64: topk (lowest index on ties is irrelevant for random
    # data), softmax over the two kept logits, explicit weighted sum of two experts.
    T, d, F, n = 12, 32, 48, 8
    x, Wg, W1, W3, W2 = _layer(T, d, F, n, seed=61)
    y, idx, gate = oracle_lib.moe_forward(x, Wg, W1, W3, W2, n, 2, round_h=False)
    l = x.double() @ Wg.double()
    top = torch.topk(l, 2, dim=1)
    assert torch.equal(torch.from_numpy(idx).long(), top.indices)
    G = torch.softmax(top.values, dim=1)
    for t in range(T):
        ref = sum(G[t, k] * _swiglu64(x[t], W1[top.indices[t, k]], W3[top.indices[t, k]],
                                      W2[top.indices[t, k]]) for k in range(2)).numpy()
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sparse_equals_dense_masked(oracle_lib, dtype):
    T, d, F, n = 10, 32, 64, 8
    x, Wg, W1, W3, W2 = _layer(T, d, F, n, seed=71, dtype=dtype)
    for round_h in (False, True):
        ys, _, _ = oracle_lib.moe_forward(x, Wg, W1, W3, W2, n, 2, round_h=round_h)
        yd = oracle_lib.moe_dense(x, Wg, W1, W3, W2, n, 2, round_h=round_h)
        assert np.allclose(ys, yd, rtol=1e-12, atol=1e-15)


def test_bf16_inputs_decoded_exactly(oracle_lib):
    # bf16 tensors and fp32 tensors holding the same values must give identical results.
    T, d, F, n = 8, 32, 40, 8
    x, Wg, W1, W3, W2 = _layer(T, d, F, n, seed=81, dtype=torch.bfloat16)
    yb, ib, gb = oracle_lib.moe_forward(x, Wg, W1, W3, W2, n, 2, round_h=False)
    yf, i_f, gf = oracle_lib.moe_forward(x.float(), Wg, W1.float(), W3.float(), W2.float(),
                                         n, 2, round_h=False)
    assert np.array_equal(ib, i_f) and np.array_equal(gb, gf) and np.array_equal(yb, yf)


def test_h_rounding_is_bf16(oracle_lib):
    # With n = 1, K = 1 and W2 = I, y = h exactly, so round_h must give bf16-representable
    # values equal to the library's fp64 -> fp32 -> bf16 rounding of silu(a)*b where that
    # double rounding cannot differ (checked on fp32-exact intermediate values).
    T, d = 6, 16
    x = _rand((T, d), 1.0, 91, torch.bfloat16)
    Wg = _rand((d, 1), 0.25, 92)
    W1 = _rand((1, d, d), d ** -0.5, 93, torch.bfloat16)
    W3 = _rand((1, d, d), d ** -0.5, 94, torch.bfloat16)
    W2 = torch.eye(d, dtype=torch.bfloat16).unsqueeze(0).contiguous()
    y, _, _ = oracle_lib.moe_forward(x, Wg, W1, W3, W2, 1, 1, round_h=True)
    yu, _, _ = oracle_lib.moe_forward(x, Wg, W1, W3, W2, 1, 1, round_h=False)
    yb = torch.from_numpy(y)
    assert torch.equal(yb.float().to(torch.bfloat16).double(), yb)          # representable
    assert np.all(np.abs(y - yu) <= np.abs(yu) * 2.0 ** -8 + 1e-30)          # half-ulp


def test_token_with_experts_matches_forward(oracle_lib):
    T, d, F, n = 5, 16, 24, 8
    x, Wg, W1, W3, W2 = _layer(T, d, F, n, seed=101)
    y, idx, _ = oracle_lib.moe_forward(x, Wg, W1, W3, W2, n, 2)
    for t in range(T):
        yt = oracle_lib.moe_token_with_experts(x, Wg, W1, W3, W2, n, t, idx[t])
        assert np.allclose(yt, y[t], rtol=1e-15, atol=0)
        yr = oracle_lib.moe_token_with_experts(x, Wg, W1, W3, W2, n, t, idx[t][::-1].copy())
        assert np.allclose(yr, y[t], rtol=1e-14, atol=1e-16)


# ------------------------------------------------------------------ stacked blocks

def test_rmsnorm_closed_form(oracle_lib):
    x = _rand((4, 64), 3.0, 111).double().numpy()
    got = oracle_lib.rmsnorm(x, 1e-5, oracle_lib.F32)
    ref = x / np.sqrt((x ** 2).mean(axis=1, keepdims=True) + 1e-5)
    assert np.allclose(got, ref.astype(np.float32).astype(np.float64), rtol=0, atol=0)
    c = np.full((1, 16), 3.0)
    assert np.allclose(oracle_lib.rmsnorm(c, 0.0, oracle_lib.F32), 1.0)


def test_block_forward_is_residual_plus_moe_of_norm(oracle_lib):
    T, d, F, n, eps = 6, 32, 48, 8, 1e-5
    x, Wg, W1, W3, W2 = _layer(T, d, F, n, seed=121)
    x64 = x.double().numpy()
    xn = oracle_lib.rmsnorm(x64, eps, oracle_lib.F32)
    y, idx_ref, _ = oracle_lib.moe_forward(torch.from_numpy(xn).float(), Wg, W1, W3, W2, n, 2)
    ref = (x64 + y).astype(np.float32).astype(np.float64)
    got, idx, _ = oracle_lib.block_forward(x64, Wg, W1, W3, W2, n, 2, eps)
    assert np.array_equal(idx, idx_ref)
    assert np.allclose(got, ref, rtol=0, atol=0)


# ------------------------------------------------------------------ FP8 (E4M3) expert weights

E4M3 = torch.float8_e4m3fn


def _e4m3_codes_torch(v):
    """E4M3 codes of binary32 values by torch's own float8 conversion (a library routine)."""
    return v.to(torch.float32).to(E4M3).view(torch.uint8)


def test_e4m3_table_closed_forms(oracle_lib):
    # the format's defining points: 448 largest finite, 2^-9 smallest subnormal, 2^-6
    # smallest normal, 1.0 = exponent 7, NaN at S.1111.111, sign bit 0x80
    assert oracle_lib.e4m3_value(0x7E) == 448.0
    assert oracle_lib.e4m3_value(0x01) == 2.0 ** -9
    assert oracle_lib.e4m3_value(0x08) == 2.0 ** -6
    assert oracle_lib.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert oracle_lib.e4m3_value(0x38) == 1.0
    assert oracle_lib.e4m3_value(0xB8) == -1.0
    assert math.isnan(oracle_lib.e4m3_value(0x7F)) and math.isnan(oracle_lib.e4m3_value(0xFF))
    # every finite code is its own nearest code; codes increase with value
    vals = [oracle_lib.e4m3_value(c) for c in range(127)]
    assert all(b > a for a, b in zip(vals, vals[1:]))
    for c in list(range(127)) + list(range(128, 255)):
        assert oracle_lib.e4m3_code(oracle_lib.e4m3_value(c)) == c
    # saturation
    assert oracle_lib.e4m3_code(1e30) == 0x7E and oracle_lib.e4m3_code(-500.0) == 0xFE


def test_e4m3_rounding_matches_torch(oracle_lib):
    # nearest code, ties to even: every midpoint between neighbouring codes, points just
    # beside them, and a dense random set, against torch's float8_e4m3fn conversion
    vals = [oracle_lib.e4m3_value(c) for c in range(127)]
    pts = []
    for a, b in zip(vals, vals[1:]):
        m = (a + b) / 2
        pts += [m, np.nextafter(np.float32(m), np.float32(0)), np.nextafter(np.float32(m),
                                                                            np.float32(1e9))]
    g = torch.Generator().manual_seed(7)
    rnd = torch.randn(4000, generator=g) * torch.exp(torch.randn(4000, generator=g) * 3)
    pts = torch.tensor(np.array(pts, np.float32))
    pts = torch.cat([pts, -pts, rnd.clamp(-448, 448)])
    ours = np.array([oracle_lib.e4m3_code(float(v)) for v in pts], np.uint8)
    assert np.array_equal(ours, _e4m3_codes_torch(pts).numpy())


def _mx_exponent_by_search(amax: float) -> int:
    """The block exponent from its definition, the smallest E with amax <= 448 2^E (no element
    overflows E4M3 once divided by 2^E), found by stepping E; clamped to [-127, 127]; 0 for an
    all-zero block."""
    if amax == 0.0:
        return 0
    E = int(math.floor(math.log2(amax))) - 8
    while 448.0 * 2.0 ** E < amax:
        E += 1
    while 448.0 * 2.0 ** (E - 1) >= amax:
        E -= 1
    return max(-127, min(127, E))


def _mx_quantize_ref(v: torch.Tensor):
    """MXFP8 block quantisation by library steps: the exponent by search, the element codes by
    torch's float8_e4m3fn conversion of v / 2^E clamped to +-448.  v float32 [rows, cols]."""
    rows, cols = v.shape
    blocks = v.reshape(rows, cols // 32, 32)
    amax = blocks.abs().amax(dim=2).double().numpy()
    E = np.vectorize(_mx_exponent_by_search, otypes=[np.int64])(amax)
    X = torch.from_numpy(np.ldexp(1.0, E))
    scaled = (blocks.double() / X[..., None]).clamp(-448.0, 448.0).float()
    q = _e4m3_codes_torch(scaled).reshape(rows, cols)
    return q.numpy(), (E + 127).astype(np.uint8)


def test_e8m0_and_block_scale_closed_forms(oracle_lib):
    assert oracle_lib.e8m0_value(127) == 1.0 and oracle_lib.e8m0_value(0) == 2.0 ** -127
    assert oracle_lib.e8m0_value(254) == 2.0 ** 127 and math.isnan(oracle_lib.e8m0_value(255))
    code = lambda v: oracle_lib.mx_scale_code(np.array(v, np.float32))
    assert code([1.0] + [0.0] * 31) == 127 - 8          # max 1 -> X = 2^-8, 1 / X = 256
    assert code([0.5, -1.75]) == 127 - 8                # 1.75 / 2^-8 = 448 still fits
    assert code([0.5, -1.7500001]) == 127 - 7           # just above: one binade up
    assert code([-2.0, 1.0]) == 127 - 7                 # 2 / 2^-7 = 256
    assert code([448.0, 3.0]) == 127                    # 448 = 1.75 * 2^8 -> X = 1
    assert code([449.0]) == 128                         # 449 > 448: X = 2
    assert code([0.0] * 32) == 127                      # all-zero block: X = 1
    assert code([2.0 ** -140, 0.0]) == 0                # clamped at 2^-127 (subnormal max)
    assert code([3.0e38]) == 127 + 127 - 8 + 1          # 3e38 = 1.76 * 2^127 > 1.75 * 2^127


def test_quantize_mx_e4m3(oracle_lib):
    # every block: the largest element divided by X lies in (224, 448], so no code saturates;
    # codes match torch's conversion of v / X; the exponents match the search on the defining
    # inequality; all-zero blocks read X = 1
    g = torch.Generator().manual_seed(11)
    scale = torch.tensor([1e-3, 1, 3, 50, 1e3, 0, 2.0 ** -130, 1e30])[:, None]
    v = (torch.randn(8, 256, generator=g) * scale).to(torch.bfloat16).float()
    v[1, :32] = torch.linspace(-1, 1, 32)             # exact power-of-two maximum
    v[2, 32:64] = 0.0                                 # one zero block inside a row
    q, sf = oracle_lib.quantize_mx_e4m3(v)
    qr, sfr = _mx_quantize_ref(v)
    np.testing.assert_array_equal(sf, sfr)
    np.testing.assert_array_equal(q, qr)
    X = np.ldexp(1.0, sf.astype(np.int64) - 127)
    blocks = v.double().numpy().reshape(8, 8, 32)
    amax = np.abs(blocks).max(axis=2)
    nz = amax > 0
    free = nz & (sf > 0)                 # exponent not clamped at -127 (row 6: below 2^-119)
    assert np.all((amax / X)[free] > 224) and np.all((amax / X)[free] <= 448)
    assert np.all(sf[nz & ~free] == 0) and np.all((amax / X)[nz & ~free] <= 224)
    assert np.all(sf[~nz] == 127)
    deq = np.array([[oracle_lib.e4m3_value(int(c)) for c in row] for row in q]).reshape(8, 8, 32)
    deq = deq * X[..., None]
    # dequantised error: half a unit in the last place of E4M3 (relative 2^-4 in the normal
    # range, 2^-10 X below it); nothing saturates
    tol = np.maximum(np.abs(blocks) * 2.0 ** -4, X[..., None] * 2.0 ** -10)
    assert not np.any(np.abs(blocks) / X[..., None] > 448)
    assert np.all(np.abs(deq - blocks) <= tol)


def _fp8_layer(T, d, F, n, seed):
    x, Wg, W1, W3, W2 = _layer(T, d, F, n, seed=seed, dtype=torch.bfloat16)
    W1q, s1 = oracle_lib_module().quantize_mx_e4m3(W1.reshape(n * F, d))
    W3q, s3 = oracle_lib_module().quantize_mx_e4m3(W3.reshape(n * F, d))
    W2q, s2 = oracle_lib_module().quantize_mx_e4m3(W2.reshape(n * d, F))
    return (x, Wg, W1q.reshape(n, F, d), W3q.reshape(n, F, d), W2q.reshape(n, d, F),
            s1.reshape(n, F, d // 32), s3.reshape(n, F, d // 32), s2.reshape(n, d, F // 32))


def oracle_lib_module():
    import oracle
    return oracle


def _dequant(q, sf):
    """float64 values of E4M3 codes q [..., cols] with E8M0 block scales sf [..., cols / 32]."""
    v = torch.from_numpy(np.ascontiguousarray(q)).view(E4M3).to(torch.float64)
    X = torch.from_numpy(np.ldexp(1.0, sf.astype(np.int64) - 127))
    return (v.reshape(*sf.shape, 32) * X[..., None]).reshape(v.shape)


def _fp8_reference_torch(x, Wg, W1q, W3q, W2q, s1, s3, s2, K):
    """The MXFP8 block from torch library steps: float64 matmuls on dequantised codes, x and h
    block-quantised by the search-based reference quantiser."""
    T, d = x.shape
    xq, xs = _mx_quantize_ref(x.float())
    xd = _dequant(xq, xs)
    l = x.double() @ Wg.double()
    top = torch.topk(l, K, dim=1)
    G = torch.softmax(top.values, dim=1)
    W1d, W3d, W2d = _dequant(W1q, s1), _dequant(W3q, s3), _dequant(W2q, s2)
    y = torch.zeros(T, d, dtype=torch.float64)
    for t in range(T):
        for k in range(K):
            e = int(top.indices[t, k])
            a = W1d[e] @ xd[t]
            b = W3d[e] @ xd[t]
            h = (torch.nn.functional.silu(a) * b).float()
            hq, hs = _mx_quantize_ref(h[None, :])
            y[t] += G[t, k] * (W2d[e] @ _dequant(hq, hs)[0])
    return y.numpy(), top.indices.numpy()


def test_fp8_block_matches_library_reference(oracle_lib):
    T, d, F, n, K = 6, 64, 96, 4, 2
    L = _fp8_layer(T, d, F, n, seed=71)
    y, idx, gate = oracle_lib.moe_forward_fp8(*L, n, K)
    ref, ridx = _fp8_reference_torch(*L, K)
    assert np.array_equal(idx, ridx)
    assert np.allclose(y, ref, rtol=1e-9, atol=1e-12)


def test_fp8_block_routing_and_scale_linearity(oracle_lib):
    # routing is the bf16 block's, and y is linear in the W2 block scales: one more in every
    # W2 scale code (X doubled) doubles y bit for bit
    T, d, F, n, K = 5, 64, 64, 8, 2
    x, Wg, W1q, W3q, W2q, s1, s3, s2 = _fp8_layer(T, d, F, n, seed=81)
    y, idx, gate = oracle_lib.moe_forward_fp8(x, Wg, W1q, W3q, W2q, s1, s3, s2, n, K)
    _, ridx, rgate = oracle_lib.route(x, Wg, n, K)
    assert np.array_equal(idx, ridx) and np.array_equal(gate, rgate)
    y2, _, _ = oracle_lib.moe_forward_fp8(x, Wg, W1q, W3q, W2q, s1, s3, s2 + 1, n, K)
    assert np.array_equal(y2, 2 * y)
