"""The autograd wrapper (packed_lora, a torch.autograd.Function over plora_forward / plora_backward)
against the fp64 oracle: Y, and the gradients autograd hands back for X and every A_i, B_i (in the
parameters' dtype, bf16) after backward of <dY, Y>, within max|err|/max|ref| <= 2e-2 per tensor."""
import dataclasses

import numpy as np
import pytest

import oracle
import plora_workloads as wl
from plora_testlib import BF16_TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def test_autograd_matches_the_oracle():
    r = np.array([4, 16, 1])
    p = wl.make_problem("ag", "bf16", 264, 392, r, [130, 7, 60], 2.0 * r, wl.init_llm(264), 77)
    eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=3, max_rank=16, max_tokens=p.T)
    X = to_dev(p.X, p).requires_grad_(True)
    W = to_dev(p.W, p)
    A = [to_dev(a, p).requires_grad_(True) for a in p.A]
    B = [to_dev(b, p).requires_grad_(True) for b in p.B]
    dY = to_dev(p.dY, p)
    Y = pl.packed_lora(eng, X, W, p.off, p.scales, A, B)
    (Y.float() * dY.float()).sum().backward()   # so that every gradient autograd returns is for <dY, Y>
    o = oracle.full(p)
    assert A[0].grad.dtype == torch.bfloat16 and B[0].grad.dtype == torch.bfloat16
    assert rel_err(np64(Y), o["Y"]) <= BF16_TOL
    assert rel_err(np64(X.grad), o["dX"]) <= BF16_TOL
    for i in range(3):
        assert rel_err(np64(A[i].grad), o["dA"][i]) <= BF16_TOL, i
        assert rel_err(np64(B[i].grad), o["dB"][i]) <= BF16_TOL, i
    eng.close()


def test_autograd_refuses_trainable_base():
    eng = pl.PackedLoRA(64, 64, "bf16", max_adapters=1, max_rank=8, max_tokens=8)
    W = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda", requires_grad=True)
    with pytest.raises(ValueError):
        pl.packed_lora(eng, torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda"), W, [0, 8], [1.0],
                       [torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")],
                       [torch.zeros((64, 8), dtype=torch.bfloat16, device="cuda")])
    eng.close()


def test_autograd_with_output_blocks_matches_the_oracle():
    # q | k | v stacked: W [512+256+256][d_in], A_i [3 r_i][d_in], B_i [1024][r_i]; block b of Y is
    # X W_b^T + s X A_{i,b}^T B_{i,b}^T, so each block is checked against the oracle run on that
    # projection alone, and dX against the sum of the three projections' input gradients.
    widths, r = [512, 256, 256], np.array([8, 24])
    d_in, d_out = 200, sum(widths)
    p = wl.make_problem("agb", "bf16", d_in, d_out, r, [150, 70], 2.0 * r, wl.init_llm(d_in), 78)
    q = wl.make_problem("agb2", "bf16", d_in, d_out, 3 * r, [150, 70], 2.0 * r, wl.init_llm(d_in), 79)
    eng = pl.PackedLoRA(d_in, d_out, "bf16", max_adapters=2, max_rank=24, max_tokens=p.T, out_blocks=widths)
    X = to_dev(p.X, p).requires_grad_(True)
    W = to_dev(p.W, p)
    A = [to_dev(a, p).requires_grad_(True) for a in q.A]           # [3 r_i][d_in]
    B = [to_dev(b, p).requires_grad_(True) for b in p.B]           # [d_out][r_i]
    dY = to_dev(p.dY, p)
    Y = pl.packed_lora(eng, X, W, p.off, p.scales, A, B)
    (Y.float() * dY.float()).sum().backward()

    dX_ref, c0 = 0.0, 0
    for b, w in enumerate(widths):
        cols = slice(c0, c0 + w)
        pb = dataclasses.replace(p, d_out=w, W=np.ascontiguousarray(p.W[cols]),
                                 dY=np.ascontiguousarray(p.dY[:, cols]),
                                 A=[np.ascontiguousarray(a[b * int(ri):(b + 1) * int(ri)]) for a, ri in zip(q.A, r)],
                                 B=[np.ascontiguousarray(x[cols]) for x in p.B])
        o = oracle.full(pb)
        assert rel_err(np64(Y)[:, cols], o["Y"]) <= BF16_TOL, b
        dX_ref = dX_ref + o["dX"]
        for i, ri in enumerate(r):
            ri = int(ri)
            assert rel_err(np64(A[i].grad)[b * ri:(b + 1) * ri], o["dA"][i]) <= BF16_TOL, (b, i)
            assert rel_err(np64(B[i].grad)[cols], o["dB"][i]) <= BF16_TOL, (b, i)
        c0 += w
    assert rel_err(np64(X.grad), dX_ref) <= BF16_TOL
    eng.close()
