"""GPU parity of the packed AdamW step (plora_adamw_step) against the fp64 oracle step.

Tolerance: max|err|/max|ref| <= 1e-5 per tensor (fp32 arithmetic) for the parameters and
both moments; the bf16 parameter copy must be exactly the round-to-nearest-even of the
GPU's own fp32 result."""
import numpy as np
import pytest

import oracle
import plora_workloads as wl
from plora_testlib import rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402

TOL = 1e-5
HP = [dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, step=1),
      dict(lr=2e-2, beta1=0.8, beta2=0.99, eps=1e-6, weight_decay=0.0, step=7),
      dict(lr=5e-4, beta1=0.0, beta2=0.5, eps=1e-3, weight_decay=0.1, step=1000),
      dict(lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.02, step=3)]


def _draw(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_adamw_step_matches_oracle(dtype):
    d_in, d_out = 264, 392
    ranks = [1, 16, 64, 3]
    rng = np.random.default_rng(11)
    dev = "cuda"
    eng = pl.PackedLoRA(d_in, d_out, dtype, max_adapters=4, max_rank=64, max_tokens=16)
    host = []
    A16, B16, Am, Bm, mA, vA, mB, vB, dA, dB = ([] for _ in range(10))
    for r in ranks:
        h = dict(A=_draw(rng, (r, d_in), 0.05), B=_draw(rng, (d_out, r), 0.05),
                 mA=_draw(rng, (r, d_in), 1e-3), vA=np.abs(_draw(rng, (r, d_in), 1e-4)),
                 mB=_draw(rng, (d_out, r), 1e-3), vB=np.abs(_draw(rng, (d_out, r), 1e-4)),
                 gA=_draw(rng, (r, d_in), 1e-2), gB=_draw(rng, (d_out, r), 1e-2))
        host.append(h)
        t = lambda a: torch.from_numpy(a).to(dev)
        if dtype == "bf16":
            A16.append(torch.empty((r, d_in), dtype=torch.bfloat16, device=dev))
            B16.append(torch.empty((d_out, r), dtype=torch.bfloat16, device=dev))
            Am.append(t(h["A"])); Bm.append(t(h["B"]))
        else:
            A16.append(t(h["A"])); B16.append(t(h["B"]))
        mA.append(t(h["mA"])); vA.append(t(h["vA"])); mB.append(t(h["mB"])); vB.append(t(h["vB"]))
        dA.append(t(h["gA"])); dB.append(t(h["gB"]))
    tab = eng.table([1.0] * 4, A16, B16, dA, dB)
    st = pl.make_adamw_states(HP, [x.data_ptr() for x in Am] if dtype == "bf16" else None,
                              [x.data_ptr() for x in Bm] if dtype == "bf16" else None,
                              [x.data_ptr() for x in mA], [x.data_ptr() for x in vA],
                              [x.data_ptr() for x in mB], [x.data_ptr() for x in vB])
    pl.plora_adamw_step(eng.h, 4, tab, st, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert pl.plora_check(eng.h, 0) == pl.PLORA_OK
    for i, h in enumerate(host):
        hp = HP[i]
        for name, g, m, v, p_dev, copy in (("A", h["gA"], mA[i], vA[i], Am[i] if dtype == "bf16" else A16[i], A16[i]),
                                           ("B", h["gB"], mB[i], vB[i], Bm[i] if dtype == "bf16" else B16[i], B16[i])):
            p_ref, m_ref, v_ref = oracle.adamw(h[name], h["m" + name], h["v" + name], g, **hp)
            p_got = p_dev.float().cpu().numpy().astype(np.float64)
            assert rel_err(p_got, p_ref) <= TOL, (i, name)
            assert rel_err(m.cpu().numpy(), m_ref) <= TOL, (i, name)
            assert rel_err(v.cpu().numpy(), v_ref) <= TOL, (i, name)
            if dtype == "bf16":
                want = wl.f32_to_bf16_bits(p_dev.cpu().numpy())
                assert np.array_equal(copy.view(torch.uint16).cpu().numpy(), want), (i, name)
    eng.close()


def test_adamw_rejects_bad_state():
    eng = pl.PackedLoRA(64, 64, "bf16", max_adapters=1, max_rank=8, max_tokens=16)
    A = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((64, 8), dtype=torch.bfloat16, device="cuda")
    f = lambda s: torch.zeros(s, dtype=torch.float32, device="cuda")
    dA, dB, Am, Bm = f((8, 64)), f((64, 8)), f((8, 64)), f((64, 8))
    mA, vA, mB, vB = f((8, 64)), f((8, 64)), f((64, 8)), f((64, 8))
    tab = eng.table([1.0], [A], [B], [dA], [dB])
    bad = [dict(lr=1e-3, beta1=1.0, step=1), dict(lr=1e-3, step=0), dict(lr=1e-3, eps=0.0, step=1)]
    for hp in bad:
        st = pl.make_adamw_states([hp], [Am.data_ptr()], [Bm.data_ptr()], [mA.data_ptr()], [vA.data_ptr()],
                                  [mB.data_ptr()], [vB.data_ptr()])
        assert pl.plora_adamw_step(eng.h, 1, tab, st, 0, check=False) == pl.PLORA_ERR_INVALID_ARG
    # a bf16 handle needs fp32 master copies
    st = pl.make_adamw_states([dict(lr=1e-3, step=1)], None, None, [mA.data_ptr()], [vA.data_ptr()],
                              [mB.data_ptr()], [vB.data_ptr()])
    assert pl.plora_adamw_step(eng.h, 1, tab, st, 0, check=False) == pl.PLORA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert not torch.any(Am) and not torch.any(A)       # nothing written
    eng.close()


def test_adamw_step_with_output_blocks():
    # with P output blocks A (and its master, moments, gradient) is [P r][d_in]; the update is
    # elementwise, so it matches the oracle step on the whole stacked tensor
    d_in, widths, ranks = 136, [256, 256], [8, 16]
    rng = np.random.default_rng(12)
    eng = pl.PackedLoRA(d_in, sum(widths), "bf16", max_adapters=2, max_rank=16, max_tokens=16, out_blocks=widths)
    t = lambda a: torch.from_numpy(a).to("cuda")
    hp = [HP[0], HP[1]]
    A16, B16, Am, Bm, mA, vA, mB, vB, dA, dB, host = ([] for _ in range(11))
    for r in ranks:
        h = dict(A=_draw(rng, (2 * r, d_in), 0.05), B=_draw(rng, (sum(widths), r), 0.05),
                 mA=_draw(rng, (2 * r, d_in), 1e-3), vA=np.abs(_draw(rng, (2 * r, d_in), 1e-4)),
                 mB=_draw(rng, (sum(widths), r), 1e-3), vB=np.abs(_draw(rng, (sum(widths), r), 1e-4)),
                 gA=_draw(rng, (2 * r, d_in), 1e-2), gB=_draw(rng, (sum(widths), r), 1e-2))
        host.append(h)
        A16.append(torch.empty((2 * r, d_in), dtype=torch.bfloat16, device="cuda"))
        B16.append(torch.empty((sum(widths), r), dtype=torch.bfloat16, device="cuda"))
        Am.append(t(h["A"])); Bm.append(t(h["B"]))
        mA.append(t(h["mA"])); vA.append(t(h["vA"])); mB.append(t(h["mB"])); vB.append(t(h["vB"]))
        dA.append(t(h["gA"])); dB.append(t(h["gB"]))
    tab = eng.table([1.0, 1.0], A16, B16, dA, dB)
    st = pl.make_adamw_states(hp, [x.data_ptr() for x in Am], [x.data_ptr() for x in Bm],
                              [x.data_ptr() for x in mA], [x.data_ptr() for x in vA],
                              [x.data_ptr() for x in mB], [x.data_ptr() for x in vB])
    pl.plora_adamw_step(eng.h, 2, tab, st, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert pl.plora_check(eng.h, 0) == pl.PLORA_OK
    for i, h in enumerate(host):
        for name, g, m, v, pdev, copy in (("A", h["gA"], mA[i], vA[i], Am[i], A16[i]),
                                          ("B", h["gB"], mB[i], vB[i], Bm[i], B16[i])):
            p_ref, m_ref, v_ref = oracle.adamw(h[name], h["m" + name], h["v" + name], g, **hp[i])
            assert rel_err(pdev.cpu().numpy(), p_ref) <= TOL, (i, name)
            assert rel_err(m.cpu().numpy(), m_ref) <= TOL and rel_err(v.cpu().numpy(), v_ref) <= TOL, (i, name)
            assert np.array_equal(copy.view(torch.uint16).cpu().numpy(), wl.f32_to_bf16_bits(pdev.cpu().numpy()))
    eng.close()
