"""The large-batch router runs x . W_g on the tensor cores with W_g split into three bf16 parts,
hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid), and relies on hi + mid + lo == w
exactly for every fp32 w (each part takes the next 8 significant bits; the subtractions are
exact in fp32), and on bf16 x bf16 products being exact in fp32.  Both claims are checked here
on the CPU with torch's own round-to-nearest-even bf16 conversion, on random weights of the
router's scale and on values at the edges (powers of two, halfway cases, tiny and huge)."""
import numpy as np
import torch


def _split(w: torch.Tensor):
    hi = w.to(torch.bfloat16).float()
    r1 = w - hi
    mid = r1.to(torch.bfloat16).float()
    r2 = r1 - mid
    lo = r2.to(torch.bfloat16).float()
    return hi, mid, lo, r1, r2


def _edge_values():
    g = torch.Generator().manual_seed(3)
    base = torch.randn(200000, generator=g) / 64.0           # the router's N(0, 1/d) scale
    bits = torch.randint(0, 2 ** 31 - 1, (200000,), generator=g, dtype=torch.int64)
    anyf = torch.from_numpy(bits.numpy().astype(np.uint32).view(np.float32).copy())
    anyf = anyf[torch.isfinite(anyf) & (anyf.abs() > 1e-30) & (anyf.abs() < 1e30)]
    powers = torch.tensor([2.0 ** k for k in range(-100, 100)])
    # values whose lower 16 bits sit exactly halfway, just below and just above
    halves = torch.from_numpy(np.array([0x3F808000, 0x3F807FFF, 0x3F808001, 0x3F7FFFFF,
                                        0xBF808000, 0x3C008080, 0x3C00807F, 0x3C008081],
                                       dtype=np.uint32).view(np.float32).copy())
    return torch.cat([base, -base, anyf, powers, -powers, halves])


def test_three_bf16_parts_sum_to_the_fp32_weight_exactly():
    w = _edge_values()
    hi, mid, lo, r1, r2 = _split(w)
    # the two subtractions are exact: checked in float64
    assert torch.equal(r1.double(), w.double() - hi.double())
    assert torch.equal(r2.double(), r1.double() - mid.double())
    # the third part needs no rounding, and the three parts add up to w exactly
    assert torch.equal(lo, r2)
    assert torch.equal(hi.double() + mid.double() + lo.double(), w.double())


def test_bf16_products_are_exact_in_fp32():
    g = torch.Generator().manual_seed(4)
    a = torch.randn(100000, generator=g).to(torch.bfloat16).float()
    b = (torch.randn(100000, generator=g) / 64.0).to(torch.bfloat16).float()
    assert torch.equal((a * b).double(), a.double() * b.double())


def test_split_logits_match_fp64_within_fp32_accumulation():
    # what the tensor cores then sum: three partial dot products in fp32, (hi + mid) + lo;
    # against the exact logit the error is that of fp32 accumulation, far inside the 1e-4
    # relative band of the routing checks
    g = torch.Generator().manual_seed(5)
    d, n = 4096, 8
    x = torch.randn(64, d, generator=g).to(torch.bfloat16).float()
    Wg = torch.randn(d, n, generator=g) / 64.0
    hi, mid, lo, _, _ = _split(Wg)
    l = ((x @ hi) + (x @ mid)) + (x @ lo)
    ref = x.double() @ Wg.double()            # logits of order 1 (x ~ N(0,1), w ~ N(0,1/d))
    err = (l.double() - ref).abs().max().item()
    assert err < 1e-5 * ref.abs().median().item(), err
