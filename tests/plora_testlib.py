"""Helpers shared by the GPU tests, bench and smoke check: move a seeded problem
to the device, run the library through its C ABI, compare with the oracle."""
from __future__ import annotations

import numpy as np

import plora_workloads as wl

BF16_TOL = 2e-2
FP32_TOL = 1e-5


def torch_dtype(p):
    import torch
    return torch.bfloat16 if p.dtype == "bf16" else torch.float32


def to_dev(a, p, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if p.dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.to(device)


def from_dev(t, p=None) -> np.ndarray:
    import torch
    return t.detach().float().cpu().numpy().astype(np.float64)


class DeviceProblem:
    def __init__(self, p, device="cuda"):
        self.p = p
        self.X = to_dev(p.X, p, device)
        self.W = to_dev(p.W, p, device)
        self.dY = to_dev(p.dY, p, device)
        self.A = [to_dev(a, p, device) for a in p.A]
        self.B = [to_dev(b, p, device) for b in p.B]


def run(p, simt=False, dev=None, want_dX=True, engine=None, max_tokens=None, unfused=False, base_pair=False):
    """One packed forward + backward through the C ABI. Returns numpy float64 outputs."""
    import torch
    import packed_lora_fine_b200 as pl
    d = dev or DeviceProblem(p)
    own = engine is None
    if own:
        engine = pl.PackedLoRA(p.d_in, p.d_out, p.dtype, max_adapters=max(1, p.n_adapters),
                               max_rank=int(max(p.ranks)) if p.n_adapters else 1,
                               max_tokens=max_tokens or max(1, p.T), simt=simt, unfused=unfused,
                               base_pair=base_pair)
    off = p.off
    Y, saved = engine.forward(d.X, d.W, off, p.scales, d.A, d.B)
    dX, dA, dB = engine.backward(d.X, d.W, d.dY, off, p.scales, d.A, d.B, saved, want_dX=want_dX)
    torch.cuda.synchronize()
    st = pl.plora_check(engine.h, 0)
    assert st == pl.PLORA_OK, pl.status_string(st)
    out = {"Y": from_dev(Y), "dA": [from_dev(x) for x in dA], "dB": [from_dev(x) for x in dB],
           "saved": saved, "engine": engine}
    if want_dX:
        out["dX"] = from_dev(dX)
    if own:
        out.pop("engine")
        engine.close()
    return out


def rel_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


def compare(p, g, o, tol, rows=None, cols_a=None, cols_b=None):
    """Per-tensor max|err|/max|ref| for Y, dX (optionally on sampled rows) and every dA_i, dB_i."""
    errs = {}
    Yg = g["Y"] if rows is None else g["Y"][rows]
    errs["Y"] = rel_err(Yg, o["Y"])
    if "dX" in g and "dX" in o:
        dXg = g["dX"] if rows is None else g["dX"][rows]
        errs["dX"] = rel_err(dXg, o["dX"])
    for i in range(p.n_adapters):
        ga, oa = g["dA"][i], o["dA"][i]
        gb, ob = g["dB"][i], o["dB"][i]
        if cols_a is not None:
            ga, oa = ga[:, cols_a], oa[:, cols_a]
        if cols_b is not None:
            gb, ob = gb[cols_b], ob[cols_b]
        errs[f"dA{i}"] = rel_err(ga, oa)
        errs[f"dB{i}"] = rel_err(gb, ob)
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    return errs, bad


def row_subproblem(p, rows):
    """The problem restricted to the given rows (sorted): each adapter keeps only its sampled rows
    of X and dY, as one contiguous segment.  A row of Y or dX depends only on that row of X or dY
    and on its adapter, so the oracle run on this small problem gives exactly those rows of the
    full problem's Y and dX (checked on the CPU by tests/test_oracle.py); full-size tests use it
    so that the oracle never copies a multi-GB input."""
    import dataclasses
    rows = np.asarray(rows, dtype=np.int64)
    assert np.all(np.diff(rows) > 0)
    seg = np.searchsorted(p.off, rows, side="right") - 1
    counts = np.bincount(seg, minlength=p.n_adapters).astype(np.int64)
    off = np.zeros(p.n_adapters + 1, np.int64)
    off[1:] = np.cumsum(counts)
    return dataclasses.replace(p, off=off, X=np.ascontiguousarray(p.X[rows]), dY=np.ascontiguousarray(p.dY[rows]))


def adapter_subproblem(p, i, out_cols=None, A_rows=None):
    """Adapter i alone over its own rows (the packed result equals each adapter run alone; pinned on
    the CPU).  out_cols / A_rows select one output block's columns of W, dY, B and its rows of A."""
    import dataclasses
    a, b = int(p.off[i]), int(p.off[i + 1])
    cols = slice(None) if out_cols is None else out_cols
    A = p.A[i] if A_rows is None else p.A[i][A_rows]
    W = p.W[cols]
    dY = np.ascontiguousarray(p.dY[a:b, cols])
    return dataclasses.replace(p, d_out=int(W.shape[0]), off=np.array([0, b - a], np.int64),
                               ranks=p.ranks[i:i + 1], alphas=p.alphas[i:i + 1], scales=p.scales[i:i + 1],
                               X=np.ascontiguousarray(p.X[a:b]), W=np.ascontiguousarray(W), dY=dY,
                               A=[np.ascontiguousarray(A)], B=[np.ascontiguousarray(p.B[i][cols])])


def run_sampled(p, rows, engine=None, unfused=False, base_pair=False, out_blocks=None):
    """One packed forward + backward through the C ABI; returns the sampled rows of Y and dX
    (gathered on the device) and every dA_i, dB_i, as numpy float64."""
    import torch
    import packed_lora_fine_b200 as pl
    d = DeviceProblem(p)
    own = engine is None
    if own:
        engine = pl.PackedLoRA(p.d_in, p.d_out, p.dtype, max_adapters=max(1, p.n_adapters),
                               max_rank=int(max(p.ranks)), max_tokens=max(1, p.T), unfused=unfused,
                               base_pair=base_pair, out_blocks=out_blocks)
    Y, saved = engine.forward(d.X, d.W, p.off, p.scales, d.A, d.B)
    dX, dA, dB = engine.backward(d.X, d.W, d.dY, p.off, p.scales, d.A, d.B, saved)
    torch.cuda.synchronize()
    st = pl.plora_check(engine.h, 0)
    assert st == pl.PLORA_OK, pl.status_string(st)
    idx = torch.from_numpy(np.asarray(rows, np.int64)).to(Y.device)
    out = {"Y": from_dev(Y.index_select(0, idx)), "dX": from_dev(dX.index_select(0, idx)),
           "dA": [from_dev(x) for x in dA], "dB": [from_dev(x) for x in dB]}
    del Y, dX, saved, d
    if own:
        engine.close()
    return out


_PROBLEMS = {}


def cached_problem(key, factory):
    """One draw per test session of a large seeded problem (drawing config 3 takes half a minute on one
    host core); callers must not modify the arrays in place."""
    if key not in _PROBLEMS:
        _PROBLEMS[key] = factory()
    return _PROBLEMS[key]
