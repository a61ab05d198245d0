"""fp64 CPU oracle for packed LoRA forward/backward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The library
(``packed_lora_fine_b200``) never imports it and shares no code with it; both
read their inputs from ``plora_workloads``.

The arithmetic lives in ``oracle.c`` (plain double loops; see its header for
the equations and the passages they follow).  This module compiles it with gcc
on first use and marshals numpy arrays into it.

Pinned by ``tests/test_oracle.py`` against properties the mathematics fixes:
weight merging (X (W + s A B) as one library matmul), B = 0, rank-1 closed
forms, packed == each adapter alone, linearity in s, exact central finite
differences of <dY, Y>, a hand-derived integer example and the segment
signature.  ``adamw`` (the optimizer step of the LoRA training loop) is pinned by
torch.optim.AdamW in float64 and by its first-step and zero-gradient closed forms.
No function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, List, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_I64P = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2 -fopenmp). Returns the path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC,
                        "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _lib_setup(lib):
    i64, i32, ci = ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    pp = ctypes.POINTER(_P)
    lib.oracle_forward.argtypes = [ci, i64, i64, i32, _P, _P, _P, _P, _P, pp, pp, i64, _P, _P, _P, i64, ci]
    lib.oracle_input_grad.argtypes = [ci, i64, i64, i32, _P, _P, _P, _P, pp, pp, _P, i64, _P, _P, _P, i64, ci]
    lib.oracle_weight_grads.argtypes = [ci, i64, i64, i32, _P, _P, _P, _P, pp, pp, _P, pp, pp, i64, _P, i64, _P,
                                        ci]
    for fn in ("oracle_forward", "oracle_input_grad", "oracle_weight_grads"):
        getattr(lib, fn).restype = ctypes.c_int
    d = ctypes.c_double
    lib.oracle_adamw.argtypes = [i64, _P, _P, _P, _P, d, d, d, d, d, ci]
    lib.oracle_adamw.restype = None
    lib.oracle_num_procs.restype = ctypes.c_int


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        _lib_setup(lib)
        _lib = lib
    return _lib


class use_library:
    """Test hook: run the oracle functions on another build of oracle.c (for example a copy with a
    planted mistake), inside a `with` block."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        _load()
        self.saved = _lib
        _lib = None
        lib = ctypes.CDLL(self.path)
        _lib_setup(lib)
        _lib = lib
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def num_procs() -> int:
    return int(_load().oracle_num_procs())


def _dt(p) -> int:
    return 0 if p.dtype == "bf16" else 1


def _common(p):
    off = np.ascontiguousarray(p.off, dtype=np.int64)
    rank = np.ascontiguousarray(p.ranks, dtype=np.int32)
    scale = np.ascontiguousarray(p.scales, dtype=np.float32)
    A = [np.ascontiguousarray(a) for a in p.A]
    B = [np.ascontiguousarray(b) for b in p.B]
    Ap = (_P * max(1, len(A)))(*[a.ctypes.data for a in A])
    Bp = (_P * max(1, len(B)))(*[b.ctypes.data for b in B])
    keep = (off, rank, scale, A, B, Ap, Bp)
    return keep


def _rows(p, rows):
    if rows is None:
        return None, p.T
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    return rows, len(rows)


def forward(p, rows: Optional[np.ndarray] = None, nthreads: int = 1, want_H: bool = False) -> Dict:
    """Y (and optionally H) in float64 for all rows, or for the listed rows."""
    lib = _load()
    off, rank, scale, A, B, Ap, Bp = _common(p)
    rows, R = _rows(p, rows)
    X = np.ascontiguousarray(p.X)
    W = np.ascontiguousarray(p.W)
    Y = np.zeros((R, p.d_out), dtype=np.float64)
    hld = int(max(1, rank.max() if len(rank) else 1))
    H = np.zeros((R, hld), dtype=np.float64) if want_H else None
    rc = lib.oracle_forward(_dt(p), ctypes.c_int64(p.d_in), ctypes.c_int64(p.d_out),
                            ctypes.c_int32(p.n_adapters), off.ctypes.data, rank.ctypes.data,
                            scale.ctypes.data, X.ctypes.data, W.ctypes.data, Ap, Bp,
                            ctypes.c_int64(R), None if rows is None else rows.ctypes.data,
                            Y.ctypes.data, None if H is None else H.ctypes.data,
                            ctypes.c_int64(hld), ctypes.c_int(nthreads))
    if rc != 0:
        raise ValueError("oracle_forward: a requested row lies outside every segment")
    out = {"Y": Y}
    if want_H:
        out["H"] = H
    return out


def input_grad(p, rows: Optional[np.ndarray] = None, nthreads: int = 1, want_G: bool = False) -> Dict:
    """dX (and optionally G) in float64 for all rows, or for the listed rows."""
    lib = _load()
    off, rank, scale, A, B, Ap, Bp = _common(p)
    rows, R = _rows(p, rows)
    W = np.ascontiguousarray(p.W)
    dY = np.ascontiguousarray(p.dY)
    dX = np.zeros((R, p.d_in), dtype=np.float64)
    gld = int(max(1, rank.max() if len(rank) else 1))
    G = np.zeros((R, gld), dtype=np.float64) if want_G else None
    rc = lib.oracle_input_grad(_dt(p), ctypes.c_int64(p.d_in), ctypes.c_int64(p.d_out),
                               ctypes.c_int32(p.n_adapters), off.ctypes.data, rank.ctypes.data,
                               scale.ctypes.data, W.ctypes.data, Ap, Bp, dY.ctypes.data,
                               ctypes.c_int64(R), None if rows is None else rows.ctypes.data,
                               dX.ctypes.data, None if G is None else G.ctypes.data,
                               ctypes.c_int64(gld), ctypes.c_int(nthreads))
    if rc != 0:
        raise ValueError("oracle_input_grad: a requested row lies outside every segment")
    out = {"dX": dX}
    if want_G:
        out["G"] = G
    return out


def weight_grads(p, nthreads: int = 1, cols_a: Optional[np.ndarray] = None,
                 cols_b: Optional[np.ndarray] = None) -> Dict[str, List[np.ndarray]]:
    """dA_i ([r_i][d_in]) and dB_i ([d_out][r_i]) in float64 for every adapter.
    With cols_a / cols_b, only those hidden columns of dA / rows of dB are computed
    (the rest stay zero)."""
    lib = _load()
    off, rank, scale, A, B, Ap, Bp = _common(p)
    X = np.ascontiguousarray(p.X)
    dY = np.ascontiguousarray(p.dY)
    dA = [np.zeros((int(r), p.d_in), dtype=np.float64) for r in rank]
    dB = [np.zeros((p.d_out, int(r)), dtype=np.float64) for r in rank]
    ca = None if cols_a is None else np.ascontiguousarray(cols_a, dtype=np.int64)
    cb = None if cols_b is None else np.ascontiguousarray(cols_b, dtype=np.int64)
    dAp = (_P * max(1, len(dA)))(*[a.ctypes.data for a in dA])
    dBp = (_P * max(1, len(dB)))(*[b.ctypes.data for b in dB])
    lib.oracle_weight_grads(_dt(p), ctypes.c_int64(p.d_in), ctypes.c_int64(p.d_out),
                            ctypes.c_int32(p.n_adapters), off.ctypes.data, rank.ctypes.data,
                            scale.ctypes.data, X.ctypes.data, Ap, Bp, dY.ctypes.data,
                            dAp, dBp,
                            ctypes.c_int64(0 if cols_a is None else len(ca)), None if cols_a is None else ca.ctypes.data,
                            ctypes.c_int64(0 if cols_b is None else len(cb)), None if cols_b is None else cb.ctypes.data,
                            ctypes.c_int(nthreads))
    return {"dA": dA, "dB": dB}


def adamw(p, m, v, g, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, step=1):
    """One AdamW step in float64 on copies of p, m, v (any shape); returns (p, m, v)."""
    lib = _load()
    p = np.array(p, dtype=np.float64, copy=True, order="C")
    m = np.array(m, dtype=np.float64, copy=True, order="C")
    v = np.array(v, dtype=np.float64, copy=True, order="C")
    g = np.ascontiguousarray(g, dtype=np.float64)
    assert p.shape == m.shape == v.shape == g.shape
    lib.oracle_adamw(ctypes.c_int64(p.size), p.ctypes.data, m.ctypes.data, v.ctypes.data, g.ctypes.data,
                     float(lr), float(beta1), float(beta2), float(eps), float(weight_decay), int(step))
    return p, m, v


def full(p, nthreads: int = 1) -> Dict:
    """Every output of one packed forward + backward: Y, dX, dA, dB (float64)."""
    out = forward(p, nthreads=nthreads)
    out.update(input_grad(p, nthreads=nthreads))
    out.update(weight_grads(p, nthreads=nthreads))
    return out
