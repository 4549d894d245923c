"""ctypes binding to the float64 C oracle (``oracle/mglu_oracle.c``).

Test infrastructure: see the package docstring.  Arrays are numpy; every
floating-point argument is converted to C-contiguous float64 first, so the
values the oracle sees are exactly the rounded inputs the GPU also consumes.

Conventions (reading of "Masked Gated Linear Unit", "Approach"):
  x   [T][d]            activations
  Ws  [h][d]            W stored transposed, Ws[j, k] = W[k, j]
  masks [n_m][h][d]     uint8 in {0, 1}, masks[i, j, k] = M_i[k, j]
  packed                n_m bits per weight, weight (j, k) at bit offset
                        (j*d + k)*n_m, bit i = mask i, LSB-first bytes
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

ACT_SWISH = 0
ACT_GELU = 1
ACT_RELU = 2
# OR-ed into act: the dense-gate ablation, out = sum_i act(x W) * v_i
GATE_DENSE = 16

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mglu_oracle.c")
_LIB = os.path.join(_HERE, "libmglu_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libmglu_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            P = ctypes.c_void_p
            lib.oracle_activation.argtypes = [i32, dbl]
            lib.oracle_activation.restype = dbl
            lib.oracle_packed_bytes.argtypes = [i32, i64, i64]
            lib.oracle_packed_bytes.restype = i64
            lib.oracle_pack_masks.argtypes = [P, i32, i64, i64, P]
            lib.oracle_pack_masks.restype = None
            lib.oracle_unpack_masks.argtypes = [P, i32, i64, i64, P]
            lib.oracle_unpack_masks.restype = None
            lib.oracle_gate_value.argtypes = [P, i64, P, P, i32, i64, i64, P, P, P, P, P]
            lib.oracle_gate_value.restype = None
            lib.oracle_forward.argtypes = [P, i64, i64, P, i64, P, i32, i32, P]
            lib.oracle_forward.restype = dbl
            lib.oracle_forward_elems.argtypes = [P, i64, P, P, i32, i32, i64, P, P, P]
            lib.oracle_forward_elems.restype = dbl
            lib.oracle_down.argtypes = [P, i64, i64, P, i64, P]
            lib.oracle_down.restype = None
            lib.oracle_down_elems.argtypes = [P, i64, P, i64, P, P, P]
            lib.oracle_down_elems.restype = None
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = i32
            lib.oracle_set_threads.argtypes = [i32]
            lib.oracle_set_threads.restype = None
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _u8(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.uint8)


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int64)


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def activation(act: int, z: float) -> float:
    """act(z): Swish (beta=1), exact-erf GELU or ReLU."""
    return _load().oracle_activation(int(act), float(z))


def packed_bytes(n_m: int, d: int, h: int) -> int:
    return int(_load().oracle_packed_bytes(n_m, d, h))


def pack_masks(masks: np.ndarray) -> np.ndarray:
    """masks [n_m][h][d] in {0,1} -> packed uint8 stream (bit by bit)."""
    m = _u8(masks)
    n_m, h, d = m.shape
    out = np.zeros(packed_bytes(n_m, d, h), dtype=np.uint8)
    _load().oracle_pack_masks(_p(m), n_m, d, h, _p(out))
    return out


def unpack_masks(packed: np.ndarray, n_m: int, d: int, h: int) -> np.ndarray:
    """packed stream -> masks [n_m][h][d] in {0,1}."""
    pk = _u8(packed)
    if pk.size < packed_bytes(n_m, d, h):
        raise ValueError("packed buffer too small")
    out = np.zeros((n_m, h, d), dtype=np.uint8)
    _load().oracle_unpack_masks(_p(pk), n_m, d, h, _p(out))
    return out


def gate_value(x, Ws, packed, n_m: int, b: int, j: int):
    """(D, g[n_m], v[n_m], sum|xW|, worst |g_i+v_i-D|) for one output element."""
    x, Ws, pk = _f64(x), _f64(Ws), _u8(packed)
    d = x.shape[1]
    D = np.zeros(1)
    g = np.zeros(8)
    v = np.zeros(8)
    absw = np.zeros(1)
    res = np.zeros(1)
    _load().oracle_gate_value(_p(x), d, _p(Ws), _p(pk), n_m, b, j,
                              _p(D), _p(g), _p(v), _p(absw), _p(res))
    return float(D[0]), g[:n_m].copy(), v[:n_m].copy(), float(absw[0]), float(res[0])


def forward(x, Ws, packed, n_m: int, act: int):
    """out [T][h] for every element; returns (out, worst relative residual of
    the invariant g_i + v_i = D)."""
    x, Ws, pk = _f64(x), _f64(Ws), _u8(packed)
    T, d = x.shape
    h = Ws.shape[0]
    if Ws.shape[1] != d:
        raise ValueError("W must be [h][d]")
    if pk.size < packed_bytes(n_m, d, h):
        raise ValueError("packed buffer too small")
    out = np.zeros((T, h))
    r = _load().oracle_forward(_p(x), T, d, _p(Ws), h, _p(pk), n_m, act, _p(out))
    if r < 0:
        raise ValueError("unsupported n_m or act")
    return out, r


def forward_elems(x, Ws, packed, n_m: int, act: int, b_idx, j_idx):
    """out[b_idx[e], j_idx[e]] for a list of elements (exact subset)."""
    x, Ws, pk = _f64(x), _f64(Ws), _u8(packed)
    b_idx, j_idx = _i64(b_idx), _i64(j_idx)
    d = x.shape[1]
    out = np.zeros(b_idx.size)
    r = _load().oracle_forward_elems(_p(x), d, _p(Ws), _p(pk), n_m, act, b_idx.size,
                                     _p(b_idx), _p(j_idx), _p(out))
    if r < 0:
        raise ValueError("unsupported n_m or act")
    return out, r


def down(hid, Wd):
    """y [T][d] = hid [T][h] @ Wd[d][h]^T in float64."""
    hid, Wd = _f64(hid), _f64(Wd)
    T, h = hid.shape
    d = Wd.shape[0]
    y = np.zeros((T, d))
    _load().oracle_down(_p(hid), T, h, _p(Wd), d, _p(y))
    return y


def down_elems(hid_rows, Wd, row_idx, c_idx):
    """y for elements (row_idx[e] of hid_rows, column c_idx[e])."""
    hid_rows, Wd = _f64(hid_rows), _f64(Wd)
    row_idx, c_idx = _i64(row_idx), _i64(c_idx)
    h = hid_rows.shape[1]
    y = np.zeros(row_idx.size)
    _load().oracle_down_elems(_p(hid_rows), h, _p(Wd), row_idx.size, _p(row_idx), _p(c_idx), _p(y))
    return y


def max_threads() -> int:
    """OpenMP threads the oracle's loops use."""
    return int(_load().oracle_max_threads())


def set_threads(n: int) -> None:
    """Set the oracle's OpenMP thread count (timing only; results do not depend on it)."""
    _load().oracle_set_threads(int(n))
