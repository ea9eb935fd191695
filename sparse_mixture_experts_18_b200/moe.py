"""Thin ctypes binding of libmoe.so (declared in include/moe.h).

Argument marshalling only: every step of the MoE block runs in the library's CUDA kernels.
torch supplies device memory and streams.  There is no fallback: if the library is missing
or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
          3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_DEVICE"}


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {STATUS.get(code, code)} ({msg})")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by sparse_mixture_experts_18_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_mixture_experts_18_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.moe_workspace_bytes.restype = SZ
        L.moe_workspace_bytes.argtypes = [I64, I64, I64, I32, I32, I32]
        L.moe_stack_workspace_bytes.restype = SZ
        L.moe_stack_workspace_bytes.argtypes = [I64, I64, I64, I32, I32, I32]
        L.moe_workspace_init.restype = I32
        L.moe_workspace_init.argtypes = [P, SZ, P]
        L.moe_workspace_status.restype = I32
        L.moe_workspace_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
        L.moe_forward.restype = I32
        L.moe_forward.argtypes = [P, P, P, P, P, I64, I64, I64, I32, I32, I32, P, P, SZ, P]
        L.moe_forward_debug.restype = I32
        L.moe_forward_debug.argtypes = [P, P, P, P, P, I64, I64, I64, I32, I32, I32, P, P, SZ, P,
                                        P, P, P, P, P]
        L.moe_forward_host_io.restype = I32
        L.moe_forward_host_io.argtypes = [P, P, P, P, P, P, I64, I64, I64, I32, I32, I32, P, P, P,
                                          SZ, P]
        L.moe_stack_forward.restype = I32
        L.moe_stack_forward.argtypes = [P, P, P, P, P, I32, I64, I64, I64, I32, I32, I32,
                                        ctypes.c_float, P, SZ, P]
        L.moe_forward_profiled.restype = I32
        L.moe_forward_profiled.argtypes = [P, P, P, P, P, I64, I64, I64, I32, I32, I32, P, P, SZ,
                                           P, ctypes.POINTER(P), I32]
        IP = ctypes.POINTER(ctypes.c_int)
        L.moe_plan_info.restype = I32
        L.moe_plan_info.argtypes = [I64, I64, I64, I32, I32, I32, IP, IP, IP, IP, IP]
        L.moe_forward_noalloc.restype = I32
        L.moe_forward_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, I32, I32, I32, P, P]
        L.moe_noalloc_status.restype = I32
        L.moe_noalloc_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
        L.moe_stack_forward_profiled.restype = I32
        L.moe_stack_forward_profiled.argtypes = [P, P, P, P, P, I32, I64, I64, I64, I32, I32,
                                                 I32, ctypes.c_float, P, SZ, P,
                                                 ctypes.POINTER(P), I32]
        L.moe_stack_forward_host_io.restype = I32
        L.moe_stack_forward_host_io.argtypes = [P, P, P, P, P, P, I32, I64, I64, I64, I32, I32,
                                                I32, ctypes.c_float, P, P, SZ, P]
        L.moe_debug_forward_withheld.restype = I32
        L.moe_debug_forward_withheld.argtypes = [P, P, P, P, P, I64, I64, I64, I32, I32, I32, P,
                                                 P, SZ, P, I64]
        L.moe_route_workspace_bytes.restype = SZ
        L.moe_route_workspace_bytes.argtypes = [I64, I64, I32, I32, I32]
        L.moe_route.restype = I32
        L.moe_route.argtypes = [P, P, I64, I64, I32, I32, I32, P, P, P, P, P, P, SZ, P]
        L.moe_experts_workspace_bytes.restype = SZ
        L.moe_experts_workspace_bytes.argtypes = [I64, I64, I64, I32, I32]
        L.moe_experts_forward.restype = I32
        L.moe_experts_forward.argtypes = [P, I64, P, I32, P, P, P, I64, I64, I32, I32, P, P, SZ,
                                          P]
        L.moe_combine.restype = I32
        L.moe_combine.argtypes = [P, P, P, I64, I64, I32, I32, P, P]
        L.moe_gather_rows.restype = I32
        L.moe_gather_rows.argtypes = [P, I64, P, I64, I64, P, P]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [I32]
        L.moe_abi_version.restype = I32
        L.moe_abi_version.argtypes = []
        L.moe_quantize_mx_e4m3.restype = I32
        L.moe_quantize_mx_e4m3.argtypes = [P, I64, I64, P, P, P]
        L.moe_workspace_bytes_fp8.restype = SZ
        L.moe_workspace_bytes_fp8.argtypes = [I64, I64, I64, I32, I32]
        L.moe_forward_fp8.restype = I32
        L.moe_forward_fp8.argtypes = [P, P, P, P, P, P, P, P, I64, I64, I64, I32, I32, P, P, SZ,
                                      P, ctypes.POINTER(P), I32]
        _lib = L
    return _lib


def _check(fn: str, code: int):
    if code != 0:
        raise MoeError(fn, code, lib().moe_status_string(code).decode())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def moe_workspace_bytes(T, d, F, n, K, dtype) -> int:
    dt = MOE_BF16 if dtype in (torch.bfloat16, MOE_BF16) else MOE_F32
    return int(lib().moe_workspace_bytes(T, d, F, n, K, dt))


def moe_stack_workspace_bytes(T, d, F, n, K, dtype=torch.bfloat16) -> int:
    dt = MOE_BF16 if dtype in (torch.bfloat16, MOE_BF16) else MOE_F32
    return int(lib().moe_stack_workspace_bytes(T, d, F, n, K, dt))


def alloc_workspace(nbytes: int, device=None, stream=None) -> torch.Tensor:
    """Device buffer of nbytes (256-byte aligned by torch's allocator), initialised."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")
    _check("moe_workspace_init", lib().moe_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))
    return ws


def moe_workspace_status(ws: torch.Tensor, stream=None) -> tuple[int, int]:
    raw = ctypes.c_uint32(0)
    code = lib().moe_workspace_status(_ptr(ws), _stream(stream), ctypes.byref(raw))
    return code, raw.value


def _dims(x, W1, W_g):
    T, d = x.shape
    n, F, d1 = W1.shape
    if d1 != d or tuple(W_g.shape) != (d, n):
        raise ValueError("shape mismatch between x, W_g and W1")
    return T, d, F, n


def moe_forward(x, W_g, W1, W3, W2, K: int, out=None, workspace=None, stream=None):
    """out[t] = sum_k G(x_t)_k SwiGLU_{e_k}(x_t) on the GPU; returns out."""
    T, d, F, n = _dims(x, W1, W_g)
    dt = _dt(x)
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = alloc_workspace(moe_workspace_bytes(T, d, F, n, K, dt), x.device, stream)
    _check("moe_forward", lib().moe_forward(
        _ptr(x), _ptr(W_g), _ptr(W1), _ptr(W3), _ptr(W2), T, d, F, n, K, dt, _ptr(out),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def moe_forward_noalloc(x, W_g, W1, W3, W2, K: int, out=None, stream=None):
    """moe_forward for callers that cannot allocate device memory: the library's own
    fixed-size device workspace is used (see include/moe.h for its size, its first-call
    set-up and why overlapping calls race).  `out` may be preallocated by the caller."""
    T, d, F, n = _dims(x, W1, W_g)
    dt = _dt(x)
    if out is None:
        out = torch.empty_like(x)
    _check("moe_forward_noalloc", lib().moe_forward_noalloc(
        _ptr(x), _ptr(W_g), _ptr(W1), _ptr(W3), _ptr(W2), T, d, F, n, K, dt, _ptr(out),
        _stream(stream)))
    return out


def moe_forward_profiled(x, W_g, W1, W3, W2, K: int, events, out=None, workspace=None,
                         stream=None):
    """moe_forward that records six torch.cuda.Event objects at the stage boundaries (see
    include/moe.h).  The events must have been recorded once (so they exist)."""
    T, d, F, n = _dims(x, W1, W_g)
    dt = _dt(x)
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = alloc_workspace(moe_workspace_bytes(T, d, F, n, K, dt), x.device, stream)
    handles = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check("moe_forward_profiled", lib().moe_forward_profiled(
        _ptr(x), _ptr(W_g), _ptr(W1), _ptr(W3), _ptr(W2), T, d, F, n, K, dt, _ptr(out),
        _ptr(workspace), workspace.numel(), _stream(stream), handles, len(events)))
    return out


def moe_plan_info(T, d, F, n, K, dtype=torch.bfloat16) -> dict:
    """The work plan the library picks for a shape."""
    dt = MOE_BF16 if dtype in (torch.bfloat16, MOE_BF16) else MOE_F32
    v = [ctypes.c_int(0) for _ in range(5)]
    _check("moe_plan_info", lib().moe_plan_info(T, d, F, n, K, dt, *[ctypes.byref(i) for i in v]))
    return {"small_batch": bool(v[0].value), "split13": v[1].value, "split2": v[2].value,
            "launches": v[3].value, "pair": v[4].value == 1, "mid": v[4].value == 2}


def moe_forward_debug(x, W_g, W1, W3, W2, K: int, out=None, workspace=None, stream=None):
    """moe_forward plus the routing state: (out, topk_idx, topk_gate, expert_counts,
    expert_offsets, token_rows)."""
    T, d, F, n = _dims(x, W1, W_g)
    dt = _dt(x)
    dev = x.device
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = alloc_workspace(moe_workspace_bytes(T, d, F, n, K, dt), dev, stream)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    gate = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty((n,), dtype=torch.int32, device=dev)
    offsets = torch.empty((n + 1,), dtype=torch.int32, device=dev)
    rows = torch.empty((T, K), dtype=torch.int32, device=dev)
    _check("moe_forward_debug", lib().moe_forward_debug(
        _ptr(x), _ptr(W_g), _ptr(W1), _ptr(W3), _ptr(W2), T, d, F, n, K, dt, _ptr(out),
        _ptr(workspace), workspace.numel(), _stream(stream), _ptr(idx), _ptr(gate),
        _ptr(counts), _ptr(offsets), _ptr(rows)))
    return out, idx, gate, counts, offsets, rows


def moe_forward_host_io(x_host, x_dev, W_g, W1, W3, W2, K: int, out_dev, out_host, workspace,
                        stream=None):
    """Host x in, host out: H2D copy, forward, D2H copy, all enqueued on the stream."""
    T, d, F, n = _dims(x_host, W1, W_g)
    dt = _dt(x_host)
    _check("moe_forward_host_io", lib().moe_forward_host_io(
        _ptr(x_host), _ptr(x_dev), _ptr(W_g), _ptr(W1), _ptr(W3), _ptr(W2), T, d, F, n, K, dt,
        _ptr(out_dev), _ptr(out_host), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out_host


def _layer_ptrs(layers):
    arr = ctypes.c_void_p * max(len(layers), 1)
    return tuple(arr(*[l[k].data_ptr() for l in layers]) for k in ("Wg", "W1", "W3", "W2"))


def _stack_ws(x, layers, K, workspace, stream):
    T, d = x.shape
    n, F, _ = layers[0]["W1"].shape
    if workspace is None:
        workspace = alloc_workspace(moe_stack_workspace_bytes(T, d, F, n, K, _dt(x)), x.device,
                                    stream)
    return T, d, F, n, workspace


def moe_stack_forward(x, layers, K: int, eps: float = 1e-5, workspace=None, stream=None):
    """In place on x: for each layer dict (W_g, W1, W3, W2), x <- x + MoE(RMSNorm(x))."""
    T, d, F, n, workspace = _stack_ws(x, layers, K, workspace, stream)
    pg, p1, p3, p2 = _layer_ptrs(layers)
    _check("moe_stack_forward", lib().moe_stack_forward(
        _ptr(x), pg, p1, p3, p2, len(layers), T, d, F, n, K, _dt(x), float(eps),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return x


def moe_stack_forward_profiled(x, layers, K: int, events, eps: float = 1e-5, workspace=None,
                               stream=None):
    """moe_stack_forward recording six torch.cuda.Event per block (a list of 6*L events, each
    recorded once beforehand so that it exists) at the stage boundaries."""
    T, d, F, n, workspace = _stack_ws(x, layers, K, workspace, stream)
    pg, p1, p3, p2 = _layer_ptrs(layers)
    handles = (ctypes.c_void_p * max(len(events), 1))(
        *[ctypes.c_void_p(e.cuda_event) for e in events])
    _check("moe_stack_forward_profiled", lib().moe_stack_forward_profiled(
        _ptr(x), pg, p1, p3, p2, len(layers), T, d, F, n, K, _dt(x), float(eps),
        _ptr(workspace), workspace.numel(), _stream(stream), handles, len(events)))
    return x


def moe_stack_forward_host_io(x_host, x_dev, layers, K: int, out_host, eps: float = 1e-5,
                              workspace=None, stream=None):
    """Host x in, host out: H2D copy into x_dev, the L blocks in place on x_dev, D2H copy to
    out_host, all enqueued on the stream (synchronise before reading out_host)."""
    T, d, F, n, workspace = _stack_ws(x_dev, layers, K, workspace, stream)
    pg, p1, p3, p2 = _layer_ptrs(layers)
    _check("moe_stack_forward_host_io", lib().moe_stack_forward_host_io(
        _ptr(x_host), _ptr(x_dev), pg, p1, p3, p2, len(layers), T, d, F, n, K, _dt(x_dev),
        float(eps), _ptr(out_host), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out_host


def moe_noalloc_status(stream=None) -> tuple[int, int]:
    """Status code and raw bits of the array moe_forward_noalloc uses (read and cleared)."""
    raw = ctypes.c_uint32(0)
    code = lib().moe_noalloc_status(_stream(stream), ctypes.byref(raw))
    return code, raw.value


def moe_debug_forward_withheld(x, W_g, W1, W3, W2, K: int, wait_limit_cycles: int, out=None,
                               workspace=None, stream=None):
    """Failure-path test hook: the block with the gate/up kernel's loads withheld so that its
    pipeline wait runs out after wait_limit_cycles (see include/moe.h).  Returns out (its
    values are undefined)."""
    T, d, F, n = _dims(x, W1, W_g)
    dt = _dt(x)
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = alloc_workspace(moe_workspace_bytes(T, d, F, n, K, dt), x.device, stream)
    _check("moe_debug_forward_withheld", lib().moe_debug_forward_withheld(
        _ptr(x), _ptr(W_g), _ptr(W1), _ptr(W3), _ptr(W2), T, d, F, n, K, dt, _ptr(out),
        _ptr(workspace), workspace.numel(), _stream(stream), int(wait_limit_cycles)))
    return out


# ------------------------------------------------------------------ expert parallelism stages

def moe_route(x, W_g, K: int, workspace=None, stream=None):
    """Router, TopK, softmax and the grouping of the (token, slot) rows by expert, unpadded:
    returns (x_grouped [T*K, d], topk_idx [T, K], topk_gate [T, K], expert_counts [n],
    token_rows [T, K]); expert e's rows are x_grouped[sum(counts[:e]) : sum(counts[:e+1])]."""
    T, d = x.shape
    n = W_g.shape[1]
    dt = _dt(x)
    dev = x.device
    if workspace is None:
        workspace = alloc_workspace(int(lib().moe_route_workspace_bytes(T, d, n, K, dt)), dev,
                                    stream)
    xg = torch.empty((T * K, d), dtype=x.dtype, device=dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    gate = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty((n,), dtype=torch.int32, device=dev)
    rows = torch.empty((T, K), dtype=torch.int32, device=dev)
    _check("moe_route", lib().moe_route(
        _ptr(x), _ptr(W_g), T, d, n, K, dt, _ptr(xg), _ptr(idx), _ptr(gate), _ptr(counts),
        _ptr(rows), _ptr(workspace), workspace.numel(), _stream(stream)))
    return xg, idx, gate, counts, rows


def moe_experts_forward(x_rows, seg_counts, W1, W3, W2, workspace=None, stream=None):
    """y_rows[r] = SwiGLU_e(x_rows[r]) in fp32 for rows that arrive in S segments, each grouped
    by the n_local experts of W1/W3/W2 (seg_counts: int32 [S, n_local] on the device)."""
    rows, d = x_rows.shape
    nl, F, _ = W1.shape
    S = seg_counts.shape[0]
    dt = _dt(x_rows)
    if workspace is None:
        workspace = alloc_workspace(
            int(lib().moe_experts_workspace_bytes(rows, d, F, nl, dt)), x_rows.device, stream)
    y = torch.empty((rows, d), dtype=torch.float32, device=x_rows.device)
    _check("moe_experts_forward", lib().moe_experts_forward(
        _ptr(x_rows), rows, _ptr(seg_counts.contiguous()), S, _ptr(W1), _ptr(W3), _ptr(W2), d,
        F, nl, dt, _ptr(y), _ptr(workspace), workspace.numel(), _stream(stream)))
    return y


def moe_gather_rows(rows_in, index, out=None, stream=None):
    """out[i] = rows_in[index[i]] (index: int32 on the device); rows of any dtype whose byte
    width is a multiple of 16."""
    n_out = index.shape[0]
    if out is None:
        out = torch.empty((n_out,) + tuple(rows_in.shape[1:]), dtype=rows_in.dtype,
                          device=rows_in.device)
    row_bytes = rows_in[0].numel() * rows_in.element_size() if rows_in.shape[0] else \
        out[0].numel() * out.element_size() if n_out else 16
    _check("moe_gather_rows", lib().moe_gather_rows(
        _ptr(rows_in), rows_in.shape[0], _ptr(index.contiguous()), n_out, row_bytes, _ptr(out),
        _stream(stream)))
    return out


def moe_combine(y_rows, token_rows, topk_gate, out, stream=None):
    """out[t] = sum_k topk_gate[t, k] * y_rows[token_rows[t, k]] (fp32 sum, one rounding)."""
    T, K = token_rows.shape
    d = y_rows.shape[1]
    _check("moe_combine", lib().moe_combine(
        _ptr(y_rows), _ptr(token_rows), _ptr(topk_gate), T, d, K, _dt(out), _ptr(out),
        _stream(stream)))
    return out


# ------------------------------------------------------------------ FP8 (MXFP8) expert weights

def moe_quantize_mx_e4m3(v: torch.Tensor, stream=None):
    """MXFP8 codes (uint8, same shape) and E8M0 block scales (uint8, numel / 32, in the tile
    order documented in moe.h) of a bf16 CUDA tensor whose last dimension is the row; rows
    and columns multiples of 128."""
    if v.dtype != torch.bfloat16 or not v.is_cuda:
        raise TypeError("moe_quantize_mx_e4m3 takes a bf16 CUDA tensor")
    v = v.contiguous()
    cols = v.shape[-1]
    rows = v.numel() // cols
    q = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    sf = torch.empty(v.numel() // 32, dtype=torch.uint8, device=v.device)
    _check("moe_quantize_mx_e4m3", lib().moe_quantize_mx_e4m3(
        _ptr(v), rows, cols, _ptr(q), _ptr(sf), _stream(stream)))
    return q, sf


def moe_workspace_bytes_fp8(T, d, F, n, K) -> int:
    return int(lib().moe_workspace_bytes_fp8(T, d, F, n, K))


def moe_forward_fp8(x, W_g, W1q, W3q, W2q, sf1, sf3, sf2, K: int, out=None, workspace=None,
                    stream=None, events=None):
    """The block with MXFP8 expert weights (E4M3 codes W1q/W3q [n,F,d], W2q [n,d,F]; their
    block scales sf1/sf3/sf2 as moe_quantize_mx_e4m3 returns them); x and out bf16.  events:
    None or six torch.cuda.Event recorded at the stage boundaries by the library.  Returns
    out."""
    T, d = x.shape
    n, F, _ = W1q.shape
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = alloc_workspace(moe_workspace_bytes_fp8(T, d, F, n, K), x.device, stream)
    ev, nev = None, 0
    if events is not None:
        ev = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in events])
        nev = 6
    _check("moe_forward_fp8", lib().moe_forward_fp8(
        _ptr(x), _ptr(W_g), _ptr(W1q), _ptr(W3q), _ptr(W2q), _ptr(sf1), _ptr(sf3), _ptr(sf2),
        T, d, F, n, K, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream), ev, nev))
    return out
