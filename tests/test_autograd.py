"""The autograd wrapper against a plain PyTorch fp32 reference of the same packed layer."""
import numpy as np
import pytest

import plora_workloads as wl
from plora_testlib import BF16_TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402


def test_autograd_matches_torch_fp32_reference():
    r = np.array([4, 16, 1])
    p = wl.make_problem("ag", "bf16", 264, 392, r, [130, 7, 60], 2.0 * r, wl.init_llm(264), 77)
    eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=3, max_rank=16, max_tokens=p.T)
    X = to_dev(p.X, p).requires_grad_(True)
    W = to_dev(p.W, p)
    A = [to_dev(a, p).requires_grad_(True) for a in p.A]
    B = [to_dev(b, p).requires_grad_(True) for b in p.B]
    dY = to_dev(p.dY, p)
    Y = pl.packed_lora(eng, X, W, p.off, p.scales, A, B)
    (Y.float() * dY.float()).sum().backward()

    # reference: the same layer in fp32 PyTorch ops on the same (bf16-valued) tensors
    Xr = X.detach().float().requires_grad_(True)
    Ar = [a.detach().float().requires_grad_(True) for a in A]
    Br = [b.detach().float().requires_grad_(True) for b in B]
    Wr = W.float()
    parts = []
    for i in range(3):
        a, b = int(p.off[i]), int(p.off[i + 1])
        xi = Xr[a:b]
        parts.append(xi @ Wr.t() + float(p.scales[i]) * (xi @ Ar[i].t()) @ Br[i].t())
    Yr = torch.cat(parts)
    (Yr * dY.float()).sum().backward()

    assert rel_err(Y.float().detach().cpu().numpy(), Yr.detach().cpu().numpy()) <= BF16_TOL
    assert rel_err(X.grad.float().cpu().numpy(), Xr.grad.cpu().numpy()) <= BF16_TOL
    for i in range(3):
        assert rel_err(A[i].grad.float().cpu().numpy(), Ar[i].grad.cpu().numpy()) <= BF16_TOL
        assert rel_err(B[i].grad.float().cpu().numpy(), Br[i].grad.cpu().numpy()) <= BF16_TOL
    eng.close()


def test_autograd_refuses_trainable_base():
    eng = pl.PackedLoRA(64, 64, "bf16", max_adapters=1, max_rank=8, max_tokens=8)
    W = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda", requires_grad=True)
    with pytest.raises(ValueError):
        pl.packed_lora(eng, torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda"), W, [0, 8], [1.0],
                       [torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")],
                       [torch.zeros((64, 8), dtype=torch.bfloat16, device="cuda")])
    eng.close()


def test_autograd_with_output_blocks_matches_torch_fp32_reference():
    # q | k | v stacked: W [512+256+256][d_in], A_i [3 r_i][d_in], B_i [1024][r_i]; block b of Y is
    # X W_b^T + s X A_{i,b}^T B_{i,b}^T
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

    Xr = X.detach().float().requires_grad_(True)
    Ar = [a.detach().float().requires_grad_(True) for a in A]
    Br = [b.detach().float().requires_grad_(True) for b in B]
    Wr = W.float()
    rows = []
    for i in range(2):
        a, e, ri = int(p.off[i]), int(p.off[i + 1]), int(r[i])
        xi = Xr[a:e]
        cols, c0 = [], 0
        for b, w in enumerate(widths):
            Ab, Bb = Ar[i][b * ri:(b + 1) * ri], Br[i][c0:c0 + w]
            cols.append(xi @ Wr[c0:c0 + w].t() + float(p.scales[i]) * (xi @ Ab.t()) @ Bb.t())
            c0 += w
        rows.append(torch.cat(cols, dim=1))
    Yr = torch.cat(rows)
    (Yr * dY.float()).sum().backward()

    assert rel_err(Y.float().detach().cpu().numpy(), Yr.detach().cpu().numpy()) <= BF16_TOL
    assert rel_err(X.grad.float().cpu().numpy(), Xr.grad.cpu().numpy()) <= BF16_TOL
    for i in range(2):
        assert rel_err(A[i].grad.float().cpu().numpy(), Ar[i].grad.cpu().numpy()) <= BF16_TOL
        assert rel_err(B[i].grad.float().cpu().numpy(), Br[i].grad.cpu().numpy()) <= BF16_TOL
    eng.close()
