"""C-ABI checks that need no GPU: the library loads, exports every entry point the header
declares, sizes workspaces, and rejects bad arguments synchronously, before any launch."""
import ctypes
import os
import re

import pytest

import sparse_mixture_experts_18_b200 as moe
from sparse_mixture_experts_18_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
BF16, F32 = 1, 0


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def _declared():
    with open(HEADER) as f:
        src = f.read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)


def test_header_declares_entry_points():
    names = _declared()
    for want in ("moe_forward", "moe_forward_debug", "moe_workspace_bytes", "moe_stack_forward",
                 "moe_status_string", "moe_forward_host_io", "moe_workspace_init",
                 "moe_workspace_status", "moe_forward_profiled", "moe_plan_info",
                 "moe_stack_forward_profiled", "moe_stack_forward_host_io",
                 "moe_debug_forward_withheld", "moe_forward_noalloc", "moe_noalloc_status",
                 "moe_route", "moe_route_workspace_bytes", "moe_experts_forward",
                 "moe_experts_workspace_bytes", "moe_combine"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name   # dlsym through ctypes


def test_abi_version_and_status_strings(L):
    assert L.moe_abi_version() >= 1
    for code in range(7):
        assert L.moe_status_string(code)
    assert L.moe_status_string(99) == b"unknown status"


def test_workspace_bytes(L):
    ws = moe.moe_workspace_bytes
    assert ws(16, 4096, 14336, 8, 2, BF16) > 0
    assert ws(4096, 4096, 14336, 8, 2, BF16) > ws(16, 4096, 14336, 8, 2, BF16)
    assert ws(0, 4096, 14336, 8, 2, BF16) > 0                   # T = 0 is valid
    assert ws(16, 4000, 14336, 8, 2, BF16) == 0                 # d % 64 on the bf16 path
    assert ws(16, 4096, 14300, 8, 2, BF16) == 0                 # F % 64
    assert ws(16, 136, 200, 8, 2, F32) > 0                      # fp32 path: multiples of 8
    assert ws(16, 4096, 14336, 65, 2, BF16) == 0                # n > 64
    assert ws(16, 4096, 14336, 8, 9, BF16) == 0                 # K > n
    assert ws(16, 4096, 14336, 8, 0, BF16) == 0                 # K < 1
    # the prefill layouts hold at least the routed rows of X, h and Y (mid-size tiles at
    # T = 600, 128-row tiles at T = 2000, CTA pairs at T = 4096)
    for T, d, F in ((600, 4096, 14336), (2000, 4096, 14336), (4096, 4096, 14336)):
        assert ws(T, d, F, 8, 2, BF16) >= T * 2 * (d * 2 + F * 2 + d * 4)
    assert moe.moe_stack_workspace_bytes(8192, 4096, 14336, 8, 2) > ws(8192, 4096, 14336, 8, 2,
                                                                       BF16)
    assert moe.moe_stack_workspace_bytes(64, 128, 256, 8, 2, F32) == 0


def _plan(L, T, d, F, n, K, dt=BF16):
    v = [ctypes.c_int(-1) for _ in range(5)]
    rc = L.moe_plan_info(T, d, F, n, K, dt, *[ctypes.byref(i) for i in v])
    return rc, [i.value for i in v]


def test_plan_selection(L):
    rc, (small, s13, s2, launches, pair) = _plan(L, 16, 4096, 14336, 8, 2)
    assert rc == OK and small == 1 and s13 >= 1 and s2 >= 1 and launches == 5  # fused route
    assert pair == 0 and 4096 // 64 % s13 == 0 and 14336 // 64 % s2 == 0
    rc, (small, s13, s2, launches, pair) = _plan(L, 4096, 4096, 14336, 8, 2)
    # W_g split, tensor-core router, scan, permute, G13, G2, combine
    assert rc == OK and small == 0 and s13 == 1 and s2 == 1 and launches == 7 and pair == 1
    rc, (_, _, _, launches, _) = _plan(L, 512, 4096, 14336, 8, 2)   # CUDA-core router
    assert rc == OK and launches == 6
    rc, (small, _, _, _, tiling) = _plan(L, 600, 4096, 14336, 8, 2)   # mid-size tiles
    assert rc == OK and small == 0 and tiling == 2
    rc, (small, _, _, _, tiling) = _plan(L, 4096, 4096, 14336, 64, 2)
    assert rc == OK and small == 0 and tiling == 2
    rc, (small, _, _, _, tiling) = _plan(L, 4096, 4096, 14336, 16, 1)   # 256 rows per expert
    assert rc == OK and small == 0 and tiling == 0
    rc, (small, _, _, _, tiling) = _plan(L, 600, 4096, 14336, 8, 2, F32)  # bf16 only
    assert rc == OK and small == 0 and tiling == 0
    rc, (small, _, _, launches, pair) = _plan(L, 2000, 4096, 14336, 8, 2)  # 128-row tiles
    assert rc == OK and small == 0 and pair == 0 and launches == 7
    rc, (small, _, _, _, pair) = _plan(L, 64, 128, 256, 8, 2, F32)
    assert rc == OK and small == 0 and pair == 0
    assert L.moe_plan_info(16, 4096, 14336, 8, 2, BF16, None, None, None, None, None) == OK
    assert _plan(L, 16, 100, 256, 8, 2)[0] == UNSUPPORTED
    assert _plan(L, 16, 128, 256, 8, 9)[0] == INVALID


P = ctypes.c_void_p


def _fwd(L, x=0x1000, wg=0x2000, w1=0x3000, w3=0x4000, w2=0x5000, T=16, d=256, F=256, n=8,
         K=2, dt=BF16, out=0x6000, ws=0x10000, ws_bytes=1 << 40):
    return L.moe_forward(P(x), P(wg), P(w1), P(w3), P(w2), T, d, F, n, K, dt, P(out), P(ws),
                         ws_bytes, None)


def test_forward_rejects_bad_arguments_before_launch(L):
    assert _fwd(L, x=0) == INVALID
    assert _fwd(L, wg=0) == INVALID
    assert _fwd(L, w1=0) == INVALID and _fwd(L, w3=0) == INVALID and _fwd(L, w2=0) == INVALID
    assert _fwd(L, out=0) == INVALID
    assert _fwd(L, ws=0) == INVALID
    assert _fwd(L, x=0x1008) == INVALID            # x not 16-byte aligned
    assert _fwd(L, ws=0x10080) == INVALID          # workspace not 256-byte aligned
    assert _fwd(L, out=0x1000) == INVALID          # out aliases x
    assert _fwd(L, K=0) == INVALID and _fwd(L, K=9) == INVALID and _fwd(L, n=0) == INVALID
    assert _fwd(L, T=-1) == INVALID
    assert _fwd(L, d=200) == UNSUPPORTED
    assert _fwd(L, n=65, K=2) == UNSUPPORTED
    assert _fwd(L, dt=7) == INVALID
    assert _fwd(L, ws_bytes=1024) == WORKSPACE


def test_zero_tokens_is_a_noop_without_touching_pointers(L):
    assert _fwd(L, T=0, x=0, w1=0, out=0, ws=0) == OK


def test_profiled_needs_six_events(L):
    evs = (P * 6)(*([P(0x1)] * 6))
    rc = L.moe_forward_profiled(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), 16, 256,
                                256, 8, 2, BF16, P(0x6000), P(0x10000), 1 << 40, None, evs, 5)
    assert rc == INVALID


def test_stack_validation(L):
    arr = (P * 2)(P(0x3000), P(0x3000))
    assert L.moe_stack_forward(P(0x1000), arr, arr, arr, arr, 2, 16, 256, 256, 8, 2, F32,
                               ctypes.c_float(1e-5), P(0x10000), 1 << 40, None) == UNSUPPORTED
    assert L.moe_stack_forward(P(0x1000), None, arr, arr, arr, 2, 16, 256, 256, 8, 2, BF16,
                               ctypes.c_float(1e-5), P(0x10000), 1 << 40, None) == INVALID
    assert L.moe_stack_forward(P(0x1000), arr, arr, arr, arr, 2, 16, 256, 256, 8, 2, BF16,
                               ctypes.c_float(1e-5), P(0x10000), 1024, None) == WORKSPACE


def test_stack_profiled_and_host_io_validation(L):
    arr = (P * 2)(P(0x3000), P(0x3000))
    evs = (P * 12)(*([P(0x1)] * 12))
    prof = L.moe_stack_forward_profiled
    args = (P(0x1000), arr, arr, arr, arr, 2, 16, 256, 256, 8, 2, BF16, ctypes.c_float(1e-5),
            P(0x10000), 1 << 40, None)
    assert prof(*args, evs, 11) == INVALID                   # six events per block
    assert prof(*args, None, 12) == INVALID
    assert prof(*args[:11], F32, *args[12:], evs, 12) == UNSUPPORTED
    assert prof(P(0x1000), arr, arr, arr, arr, 2, 16, 256, 256, 8, 2, BF16,
                ctypes.c_float(1e-5), P(0x10000), 1024, None, evs, 12) == WORKSPACE
    hio = L.moe_stack_forward_host_io
    assert hio(None, P(0x1000), arr, arr, arr, arr, 2, 16, 256, 256, 8, 2, BF16,
               ctypes.c_float(1e-5), P(0x7000), P(0x10000), 1 << 40, None) == INVALID
    assert hio(P(0x8000), P(0x1000), arr, arr, arr, arr, 2, 16, 256, 256, 8, 2, BF16,
               ctypes.c_float(1e-5), None, P(0x10000), 1 << 40, None) == INVALID
    assert hio(P(0x8000), P(0x1000), arr, arr, arr, arr, 2, 16, 256, 256, 8, 2, F32,
               ctypes.c_float(1e-5), P(0x7000), P(0x10000), 1 << 40, None) == UNSUPPORTED


def test_withheld_hook_validation(L):
    def call(T=16, d=256, F=256, dt=BF16, limit=1000):
        return L.moe_debug_forward_withheld(P(0x1000), P(0x2000), P(0x3000), P(0x4000),
                                            P(0x5000), T, d, F, 8, 2, dt, P(0x6000),
                                            P(0x10000), 1 << 40, None, limit)
    assert call(limit=0) == INVALID and call(limit=-5) == INVALID
    assert call(limit=5_000_000_000) == INVALID              # above the kernels' own limit
    assert call(dt=F32) == UNSUPPORTED                       # the fp32 kernel has no pipeline
    assert call(T=4096) == UNSUPPORTED                       # CTA-pair tiling
    assert call(T=0) == OK


def test_expert_parallel_stage_validation(L):
    rb = L.moe_route_workspace_bytes
    assert rb(16, 4096, 8, 2, BF16) > 0 and rb(16, 4000, 8, 2, BF16) == 0
    # the route-only workspace holds no expert stages: far smaller than the block's
    assert rb(4096, 4096, 8, 2, BF16) < moe.moe_workspace_bytes(4096, 4096, 14336, 8, 2, BF16) / 50
    route = L.moe_route
    args = [P(0x1000), P(0x2000), 16, 256, 8, 2, BF16, P(0x3000), P(0x4000), P(0x5000),
            P(0x6000), P(0x7000), P(0x10000), 1 << 40, None]
    assert route(*args[:7], P(0x1000), *args[8:]) == INVALID     # x_grouped aliases x
    assert route(*args[:7], None, *args[8:]) == INVALID
    assert route(*args[:13], 64, None) == WORKSPACE
    assert route(*args[:5], 9, *args[6:]) == INVALID               # K > n
    assert route(P(0), P(0), 0, 256, 8, 2, BF16, *([P(0)] * 6), 0, None) == OK   # T = 0
    eb = L.moe_experts_workspace_bytes
    assert eb(100, 4096, 14336, 4, BF16) > 0 and eb(100, 4096, 14300, 4, BF16) == 0
    exf = L.moe_experts_forward
    eargs = [P(0x1000), 100, P(0x2000), 2, P(0x3000), P(0x4000), P(0x5000), 256, 256, 4, BF16,
             P(0x6000), P(0x10000), 1 << 40, None]
    assert exf(*eargs[:3], 0, *eargs[4:]) == INVALID                # no source
    assert exf(*eargs[:3], 1024, *eargs[4:]) == INVALID             # S * n_local > 2048
    assert exf(*eargs[:2], None, *eargs[3:]) == INVALID
    assert exf(*eargs[:13], 512, None) == WORKSPACE
    assert exf(*eargs[:7], 200, *eargs[8:]) == UNSUPPORTED          # d % 64
    assert exf(P(0), 0, P(0), 2, P(0), P(0), P(0), 256, 256, 4, BF16, P(0), P(0), 0, None) == OK
    comb = L.moe_combine
    assert comb(P(0x1000), P(0x2000), P(0x3000), 16, 256, 0, BF16, P(0x4000), None) == INVALID
    assert comb(P(0x1000), P(0x2000), P(0x3000), 16, 250, 2, BF16, P(0x4000), None) == UNSUPPORTED
    assert comb(P(0x1008), P(0x2000), P(0x3000), 16, 256, 2, BF16, P(0x4000), None) == INVALID
    assert comb(None, None, None, 0, 256, 2, BF16, None, None) == OK


def test_host_io_validation(L):
    rc = L.moe_forward_host_io(None, P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(0x5000), 16,
                               256, 256, 8, 2, BF16, P(0x6000), P(0x7000), P(0x10000), 1 << 40,
                               None)
    assert rc == INVALID


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "sparse_mixture_experts_18_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, fn)) as f:
                    src = f.read()
                assert not re.search(r"\boracle\b", src), fn
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        assert "oracle" not in f.read()


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    from sparse_mixture_experts_18_b200 import moe as binding
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(ImportError):
        binding.lib()
    importlib.reload(binding)


def _fwd8(L, x=0x1000, wg=0x2000, w1=0x3000, w3=0x4000, w2=0x5000, s1=0x7000, s3=0x8000,
          s2=0x9000, T=16, d=256, F=384, n=8, K=2, out=0x6000, ws=0x10000, ws_bytes=1 << 40,
          events=None, n_events=0):
    return L.moe_forward_fp8(P(x), P(wg), P(w1), P(w3), P(w2), P(s1), P(s3), P(s2), T, d, F, n,
                             K, P(out), P(ws), ws_bytes, None, events, n_events)


def test_fp8_workspace_and_supported_shapes(L):
    ws8 = L.moe_workspace_bytes_fp8
    assert ws8(16, 4096, 14336, 8, 2) > 0                        # Mixtral decode
    assert ws8(64, 4096, 14336, 8, 2) > 0
    assert ws8(65, 4096, 14336, 8, 2) == 0                       # past the one-launch routing
    assert ws8(16, 4032, 14336, 8, 2) == 0                       # d % 128
    assert ws8(16, 4096, 14272, 8, 2) == 0                       # F % 128
    assert ws8(64, 256, 384, 1, 1) == 0                          # T*K >= 64 n: not small batch
    assert ws8(0, 4096, 14336, 8, 2) > 0


def test_fp8_forward_rejects_bad_arguments_before_launch(L):
    assert _fwd8(L, x=0) == INVALID and _fwd8(L, w2=0) == INVALID
    assert _fwd8(L, s1=0) == INVALID and _fwd8(L, s2=0x9004) == INVALID   # null / misaligned
    assert _fwd8(L, out=0x1000) == INVALID                                # aliases x
    assert _fwd8(L, d=192) == UNSUPPORTED and _fwd8(L, T=100) == UNSUPPORTED
    assert _fwd8(L, K=9) == INVALID
    assert _fwd8(L, ws_bytes=4096) == WORKSPACE
    assert _fwd8(L, n_events=5, events=(P * 6)(*([P(0x1)] * 6))) == INVALID
    assert _fwd8(L, T=0, x=0, out=0) == OK


def test_quantize_mx_validation(L):
    q = L.moe_quantize_mx_e4m3
    assert q(P(0x1000), 128, 192, P(0x2000), P(0x3000), None) == INVALID    # cols % 128
    assert q(P(0x1000), 96, 128, P(0x2000), P(0x3000), None) == INVALID     # rows % 128
    assert q(None, 128, 128, P(0x2000), P(0x3000), None) == INVALID
    assert q(P(0x1004), 128, 128, P(0x2000), P(0x3000), None) == INVALID    # v not 8-byte aligned
    assert q(P(0x1000), 128, 128, P(0x2000), P(0x3008), None) == INVALID    # sf not 16-byte
    assert q(P(0x1000), 0, 128, None, None, None) == OK                     # no rows: no-op


def test_gather_rows_validation(L):
    g = L.moe_gather_rows
    assert g(P(0x1000), 10, P(0x2000), 5, 24, P(0x3000), None) == INVALID    # row bytes % 16
    assert g(None, 10, P(0x2000), 5, 32, P(0x3000), None) == INVALID
    assert g(P(0x1008), 10, P(0x2000), 5, 32, P(0x3000), None) == INVALID    # in not 16-byte
    assert g(P(0x1000), 10, P(0x2002), 5, 32, P(0x3000), None) == INVALID    # index not 4-byte
    assert g(P(0x1000), 10, P(0x2000), 5, 32, P(0x1000), None) == INVALID    # in == out
    assert g(P(0x1000), -1, P(0x2000), 5, 32, P(0x3000), None) == INVALID
    assert g(None, 0, None, 0, 32, None, None) == OK                          # no rows: no-op
