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
