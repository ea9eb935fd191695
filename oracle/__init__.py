"""CPU oracle for the Mixtral sparse-MoE block forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import this
package.  It wraps ``moe_oracle.c`` (plain C, IEEE double, OpenMP over tokens) with ctypes
and shares no code with the CUDA library.  What each function computes, and the passage of
"Mixtral of Experts" (arXiv 2401.04088) it follows, is stated in ``moe_oracle.c``.

Inputs are torch CPU tensors (or numpy arrays) in their stored dtype: bf16 tensors are
passed as their raw 16-bit patterns, fp32 as fp32, the router weight W_g always fp32.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

F32, BF16 = 0, 1
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP).  Returns the library path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.oracle_round_bf16.restype = D
        L.oracle_round_bf16.argtypes = [D]
        L.oracle_round_array.restype = None
        L.oracle_round_array.argtypes = [P, I64, I32]
        L.oracle_silu.restype = D
        L.oracle_silu.argtypes = [D]
        L.oracle_route.restype = I32
        L.oracle_route.argtypes = [I64, I64, I32, I32, I32, P, P, P, P, P]
        L.oracle_moe_forward.restype = I32
        L.oracle_moe_forward.argtypes = [I64, I64, I64, I32, I32, I32, P, P, P, P, P, I32,
                                         I64, P, P, P, P]
        L.oracle_moe_token_with_experts.restype = I32
        L.oracle_moe_token_with_experts.argtypes = [I64, I64, I64, I32, I32, I32, P, P, P, P,
                                                    P, I32, I64, P, P]
        L.oracle_moe_dense.restype = I32
        L.oracle_moe_dense.argtypes = [I64, I64, I64, I32, I32, I32, P, P, P, P, P, I32, I64,
                                       P, P]
        L.oracle_rmsnorm.restype = None
        L.oracle_rmsnorm.argtypes = [I64, I64, I32, D, P, P]
        L.oracle_block_forward.restype = I32
        L.oracle_block_forward.argtypes = [I64, I64, I64, I32, I32, I32, D, P, P, P, P, P, P,
                                           P]
        L.oracle_e4m3_value.restype = D
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_code.restype = ctypes.c_uint8
        L.oracle_e4m3_code.argtypes = [ctypes.c_float]
        L.oracle_e8m0_value.restype = D
        L.oracle_e8m0_value.argtypes = [ctypes.c_uint8]
        L.oracle_mx_scale_code.restype = ctypes.c_uint8
        L.oracle_mx_scale_code.argtypes = [P, I32]
        L.oracle_quantize_mx_e4m3.restype = None
        L.oracle_quantize_mx_e4m3.argtypes = [I64, I64, I32, P, P, P]
        L.oracle_moe_forward_fp8.restype = I32
        L.oracle_moe_forward_fp8.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, P, P, P,
                                             I64, P, P, P, P]
        _lib = L
    return _lib


# ------------------------------------------------------------------ marshalling helpers

def _raw(t):
    """Contiguous numpy view of a CPU tensor/array in its stored dtype, plus its dtype code."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().contiguous().cpu()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy(), BF16
            if t.dtype == torch.float32:
                return t.numpy(), F32
            raise TypeError(f"unsupported dtype {t.dtype}")
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(t)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype in (np.uint16, np.int16):
        return a, BF16
    raise TypeError(f"unsupported dtype {a.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _wg(Wg):
    a, dt = _raw(Wg)
    if dt != F32:
        raise TypeError("W_g must be fp32")
    return a


def round_bf16(v: float) -> float:
    return lib().oracle_round_bf16(float(v))


def round_array(v: np.ndarray, dtype: int) -> np.ndarray:
    """Copy of v (float64) rounded element-wise to bf16 (dtype=BF16) or fp32 (dtype=F32)."""
    out = np.ascontiguousarray(v, np.float64).copy()
    lib().oracle_round_array(_ptr(out), out.size, int(dtype))
    return out


def silu(z: float) -> float:
    return lib().oracle_silu(float(z))


def route(x, Wg, n: int, K: int):
    """Router, TopK and Softmax for every token.  Returns (logits [T,n] f64, idx [T,K] i32,
    gate [T,K] f64)."""
    xa, dt = _raw(x)
    T, d = xa.shape
    wg = _wg(Wg)
    logits = np.zeros((T, n), np.float64)
    idx = np.zeros((T, K), np.int32)
    gate = np.zeros((T, K), np.float64)
    rc = lib().oracle_route(T, d, n, K, dt, _ptr(xa), _ptr(wg), _ptr(logits), _ptr(idx),
                            _ptr(gate))
    if rc:
        raise ValueError(f"oracle_route failed ({rc})")
    return logits, idx, gate


def _weights(W1, W3, W2, dt):
    w1, d1 = _raw(W1)
    w3, d3 = _raw(W3)
    w2, d2 = _raw(W2)
    if not (d1 == d3 == d2 == dt):
        raise TypeError("x, W1, W3, W2 must share a dtype")
    return w1, w3, w2


def moe_forward(x, Wg, W1, W3, W2, n: int, K: int, tokens=None, round_h: bool = True):
    """Sparse MoE block output (unrounded, f64) for the given token rows (default: all).
    Returns (y [len(tokens), d] f64, idx [len, K] i32, gate [len, K] f64)."""
    xa, dt = _raw(x)
    T, d = xa.shape
    w1, w3, w2 = _weights(W1, W3, W2, dt)
    F = w1.shape[1]
    tok = np.arange(T, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    y = np.zeros((len(tok), d), np.float64)
    idx = np.zeros((len(tok), K), np.int32)
    gate = np.zeros((len(tok), K), np.float64)
    rc = lib().oracle_moe_forward(T, d, F, n, K, dt, _ptr(xa), _ptr(_wg(Wg)), _ptr(w1),
                                  _ptr(w3), _ptr(w2), int(round_h), len(tok), _ptr(tok),
                                  _ptr(y), _ptr(idx), _ptr(gate))
    if rc:
        raise ValueError(f"oracle_moe_forward failed ({rc})")
    return y, idx, gate


def moe_token_with_experts(x, Wg, W1, W3, W2, n: int, t: int, experts, round_h=True):
    """Block output of token t with an explicitly given expert set (gates from its logits)."""
    xa, dt = _raw(x)
    T, d = xa.shape
    w1, w3, w2 = _weights(W1, W3, W2, dt)
    F = w1.shape[1]
    ex = np.asarray(experts, np.int32)
    y = np.zeros(d, np.float64)
    rc = lib().oracle_moe_token_with_experts(T, d, F, n, len(ex), dt, _ptr(xa),
                                             _ptr(_wg(Wg)), _ptr(w1), _ptr(w3), _ptr(w2),
                                             int(round_h), int(t), _ptr(ex), _ptr(y))
    if rc:
        raise ValueError(f"oracle_moe_token_with_experts failed ({rc})")
    return y


def moe_dense(x, Wg, W1, W3, W2, n: int, K: int, tokens=None, round_h: bool = True):
    """Dense-masked block output: all n experts evaluated, weighted by G (0 off the top-K)."""
    xa, dt = _raw(x)
    T, d = xa.shape
    w1, w3, w2 = _weights(W1, W3, W2, dt)
    F = w1.shape[1]
    tok = np.arange(T, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    y = np.zeros((len(tok), d), np.float64)
    rc = lib().oracle_moe_dense(T, d, F, n, K, dt, _ptr(xa), _ptr(_wg(Wg)), _ptr(w1),
                                _ptr(w3), _ptr(w2), int(round_h), len(tok), _ptr(tok), _ptr(y))
    if rc:
        raise ValueError(f"oracle_moe_dense failed ({rc})")
    return y


def rmsnorm(x: np.ndarray, eps: float, dtype: int):
    x = np.ascontiguousarray(x, np.float64)
    out = np.zeros_like(x)
    lib().oracle_rmsnorm(x.shape[0], x.shape[1], dtype, float(eps), _ptr(x), _ptr(out))
    return out


def block_forward(x: np.ndarray, Wg, W1, W3, W2, n: int, K: int, eps: float):
    """One stacked block x <- round(x + MoE(RMSNorm(x))) on independent rows, in place on a
    float64 copy.  x holds values of the weights' dtype.  Returns (x_new, idx, gate)."""
    w1, d1 = _raw(W1)
    w3, _ = _raw(W3)
    w2, _ = _raw(W2)
    xs = np.ascontiguousarray(x, np.float64).copy()
    rows, d = xs.shape
    F = w1.shape[1]
    K = int(K)
    idx = np.zeros((rows, K), np.int32)
    gate = np.zeros((rows, K), np.float64)
    rc = lib().oracle_block_forward(rows, d, F, n, K, d1, float(eps), _ptr(xs), _ptr(_wg(Wg)),
                                    _ptr(w1), _ptr(w3), _ptr(w2), _ptr(idx), _ptr(gate))
    if rc:
        raise ValueError(f"oracle_block_forward failed ({rc})")
    return xs, idx, gate


def tie_band(logits_row: np.ndarray, K: int, rel: float = 1e-4):
    """Admissible TopK sets of one token when logits near the K-th place tie within a
    relative band: the experts strictly above the band are kept, and any choice among those
    inside it is correct.  Returns (is_exempt, list of sorted expert tuples)."""
    import itertools
    n = len(logits_row)
    order = sorted(range(n), key=lambda i: (-logits_row[i], i))
    if K >= n:
        return False, [tuple(sorted(order))]
    lk, lk1 = logits_row[order[K - 1]], logits_row[order[K]]
    band = rel * max(abs(lk), abs(lk1))
    if abs(lk - lk1) > band:
        return False, [tuple(sorted(order[:K]))]
    near = [i for i in range(n) if abs(logits_row[i] - lk) <= band]
    sure = [i for i in order[:K] if i not in near]
    sets = [tuple(sorted(sure + list(c))) for c in itertools.combinations(near, K - len(sure))]
    return True, sets


# ------------------------------------------------------------------ FP8 expert weights

def e4m3_value(code: int) -> float:
    """Value of an OCP FP8 E4M3 code (NaN for S.1111.111)."""
    return lib().oracle_e4m3_value(int(code) & 0xFF)


def e4m3_code(v: float) -> int:
    """Nearest E4M3 code to the binary32 value v (ties to even, saturating at 448)."""
    return int(lib().oracle_e4m3_code(float(v)))


def e8m0_value(code: int) -> float:
    """Value of an E8M0 scale code, 2^(code - 127) (NaN for 255)."""
    return lib().oracle_e8m0_value(int(code) & 0xFF)


def mx_scale_code(block) -> int:
    """E8M0 code of the shared scale of one block of binary32 values:
    floor(log2(max |v|)) - 8 + 127, clamped to [0, 254]; 127 for an all-zero block."""
    v = np.ascontiguousarray(block, np.float32)
    return int(lib().oracle_mx_scale_code(_ptr(v), len(v)))


def quantize_mx_e4m3(v):
    """MXFP8 quantisation of a [rows][cols] bf16/fp32 tensor (cols % 32 == 0): blocks of 32
    along each row share an E8M0 scale X; codes = E4M3(v / X).  Returns (q uint8
    [rows, cols], sf uint8 [rows, cols // 32]) with the scale codes in plain row order."""
    a, dt = _raw(v)
    a = a.reshape(-1, a.shape[-1])
    rows, cols = a.shape
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    q = np.zeros((rows, cols), np.uint8)
    sf = np.zeros((rows, cols // 32), np.uint8)
    lib().oracle_quantize_mx_e4m3(rows, cols, dt, _ptr(a), _ptr(q), _ptr(sf))
    return q, sf


def moe_forward_fp8(x, Wg, W1q, W3q, W2q, sf1, sf3, sf2, n: int, K: int, tokens=None):
    """Block output (unrounded, f64) with MXFP8 expert weights for the given token rows:
    W1q/W3q [n,F,d] and W2q [n,d,F] uint8 E4M3 codes, sf1/sf3 [n,F,d//32] and sf2
    [n,d,F//32] uint8 E8M0 block-scale codes.  Returns (y [len, d] f64, idx [len, K] i32,
    gate [len, K] f64)."""
    xa, dt = _raw(x)
    if dt != BF16:
        raise TypeError("the FP8-weight block takes bf16 activations")
    T, d = xa.shape
    w1 = np.ascontiguousarray(W1q, np.uint8)
    w3 = np.ascontiguousarray(W3q, np.uint8)
    w2 = np.ascontiguousarray(W2q, np.uint8)
    F = w1.shape[1]
    a1 = np.ascontiguousarray(sf1, np.uint8)
    a3 = np.ascontiguousarray(sf3, np.uint8)
    a2 = np.ascontiguousarray(sf2, np.uint8)
    if a1.size != n * F * d // 32 or a3.size != a1.size or a2.size != n * d * F // 32:
        raise ValueError("block-scale arrays do not match the weights")
    tok = np.arange(T, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    y = np.zeros((len(tok), d), np.float64)
    idx = np.zeros((len(tok), K), np.int32)
    gate = np.zeros((len(tok), K), np.float64)
    rc = lib().oracle_moe_forward_fp8(T, d, F, n, K, _ptr(xa), _ptr(_wg(Wg)), _ptr(w1),
                                      _ptr(w3), _ptr(w2), _ptr(a1), _ptr(a3), _ptr(a2),
                                      len(tok), _ptr(tok), _ptr(y), _ptr(idx), _ptr(gate))
    if rc:
        raise ValueError(f"oracle_moe_forward_fp8 failed ({rc})")
    return y, idx, gate
