"""Layer calls (plora_layer_*): several projections over one segment map run as one launch set: one
persistent launch per memory-bound product kind over all of them, one base-GEMM launch per projection.  A small LLaMA-like layer -- q|k|v and gate|up as
projections with output blocks, o and down as plain ones -- with ragged segments, an empty adapter and
a rank-1 adapter.  Checked: every projection's Y, dX, dA, dB equal bit for bit those of separate
plora_forward / plora_backward calls (the same kernels compute every tile; only the launches are
shared); each projection matches the fp64 oracle (per output block, as in the output-block tests),
max|err|/max|ref| <= 2e-2; a forward takes 3 launches plus one per projection, a backward 2 plus one
per projection."""
import dataclasses

import numpy as np
import pytest

import oracle
import plora_workloads as wl
from plora_testlib import BF16_TOL, DeviceProblem, compare, from_dev, rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402
from test_out_blocks import blocked_problem  # noqa: E402

RANKS = [8, 16, 1, 40]
COUNTS = [300, 0, 129, 700]


def layer_problems():
    """(name, stacked problem, per-block problems or None, out_blocks or None) per projection."""
    r = np.asarray(RANKS)
    qkv, qkv_blocks = blocked_problem(1301, 384, [512, 256], RANKS, COUNTS)
    o = wl.make_problem("o", "bf16", 512, 384, r, COUNTS, 2.0 * r, wl.init_llm(512), 1302)
    gu, gu_blocks = blocked_problem(1303, 384, [512, 512], RANKS, COUNTS)
    down = wl.make_problem("down", "bf16", 1024, 384, r, COUNTS, 2.0 * r, wl.init_llm(1024), 1304)
    return [("qkv", qkv, qkv_blocks, [512, 256]), ("o", o, None, None), ("gate_up", gu, gu_blocks, [512, 512]),
            ("down", down, None, None)]


def test_layer_call_equals_separate_calls_and_the_oracle():
    projs = layer_problems()
    T = projs[0][1].T
    off = projs[0][1].off
    scales = projs[0][1].scales
    dev = [DeviceProblem(p) for _, p, _, _ in projs]
    io = [{"X": d.X, "W": d.W, "A": d.A, "B": d.B, "dY": d.dY} for d in dev]
    layer = pl.PackedLoRALayer([(p.d_in, p.d_out) + ((blk,) if blk else ()) for _, p, _, blk in projs],
                               max_adapters=len(RANKS), max_rank=max(RANKS), max_tokens=T)
    pl.plora_profile_read(layer.handle(0))
    pl.plora_profile_enable(layer.handle(0), True)
    fw = layer.forward(io, off, scales)
    bw = layer.backward(io, off, scales, [s for _, s in fw])
    torch.cuda.synchronize()
    assert layer.check() == pl.PLORA_OK
    prof = pl.plora_profile_read(layer.handle(0))
    launches = {k: v[0] for k, v in prof.items() if v[0]}
    assert launches == {"stage_copy": 2, "pack_ab": 1, "shrink_x": 1, "base_fwd": len(projs), "shrink_dy+wgrad_b": 1,
                        "base_dx+wgrad_a": len(projs)}, launches
    for k, (name, p, blocks, blk) in enumerate(projs):
        Y, saved = fw[k]
        dX, dA, dB = bw[k]
        g = {"Y": from_dev(Y), "dX": from_dev(dX), "dA": [from_dev(x) for x in dA], "dB": [from_dev(x) for x in dB]}
        # separate calls on a handle of their own: the same bits
        eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=len(RANKS), max_rank=max(RANKS), max_tokens=T,
                            out_blocks=blk)
        d = dev[k]
        Y1, saved1 = eng.forward(d.X, d.W, off, scales, d.A, d.B)
        dX1, dA1, dB1 = eng.backward(d.X, d.W, d.dY, off, scales, d.A, d.B, saved1)
        torch.cuda.synchronize()
        assert pl.plora_check(eng.h, 0) == pl.PLORA_OK
        assert torch.equal(Y, Y1) and torch.equal(dX, dX1), name
        for i in range(len(RANKS)):
            assert torch.equal(dA[i], dA1[i]) and torch.equal(dB[i], dB1[i]), (name, i)
        eng.close()
        # the oracle, per projection (per output block for the stacked ones)
        if blocks is None:
            errs, bad = compare(p, g, oracle.full(p, nthreads=oracle.num_procs()), BF16_TOL)
            assert not bad, (name, bad)
            continue
        dX_ref = 0.0
        for b, (cols, pb) in enumerate(blocks):
            ob = oracle.full(pb, nthreads=oracle.num_procs())
            assert rel_err(g["Y"][:, cols], ob["Y"]) <= BF16_TOL, (name, "Y", b)
            dX_ref = dX_ref + ob["dX"]
            for i, r in enumerate(RANKS):
                assert rel_err(g["dA"][i][b * r:(b + 1) * r], ob["dA"][i]) <= BF16_TOL, (name, "dA", b, i)
                assert rel_err(g["dB"][i][cols], ob["dB"][i]) <= BF16_TOL, (name, "dB", b, i)
        assert rel_err(g["dX"], dX_ref) <= BF16_TOL, name
    layer.close()


def test_layer_call_rejects_a_bad_projection_and_writes_nothing():
    projs = layer_problems()[1:2] * 2   # two plain projections
    p = projs[0][1]
    d = DeviceProblem(p)
    layer = pl.PackedLoRALayer([(p.d_in, p.d_out), (p.d_in, p.d_out)], max_adapters=4, max_rank=64, max_tokens=p.T)
    Y = [torch.full((p.T, p.d_out), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    tab = pl.make_table([b.shape[1] for b in d.B], p.scales, [a.data_ptr() for a in d.A], [b.data_ptr() for b in d.B])
    saved = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
    items = [{"X": d.X.data_ptr(), "W": d.W.data_ptr(), "Y": Y[0].data_ptr(), "tab": tab, "saved": saved.data_ptr()},
             {"X": d.X.data_ptr() + 2, "W": d.W.data_ptr(), "Y": Y[1].data_ptr(), "tab": tab,
              "saved": saved.data_ptr()}]      # projection 1: X misaligned
    st = pl.load().plora_layer_forward(layer.L, p.n_adapters, np.ascontiguousarray(p.off).ctypes.data,
                                       pl.make_projs(items), 0)
    assert st == pl.PLORA_ERR_INVALID_ARG
    assert pl.load().plora_layer_last_error(layer.L).decode().startswith("projection 1:")
    torch.cuda.synchronize()
    assert all(bool(torch.all(y == 7.0)) for y in Y)
    layer.close()


def test_layer_call_with_different_ranks_per_projection_and_a_skipped_dX():
    """Each projection has its own adapter table: here the same adapters carry ranks up to 16 in one
    projection and up to 200 in the other (so the shared narrow ring must hold the wider pitch), and
    the second projection's backward skips dX.  Results equal separate calls bit for bit."""
    counts = [257, 1, 0, 640]
    r1, r2 = np.array([4, 16, 8, 1]), np.array([200, 3, 64, 33])
    p1 = wl.make_problem("l1", "bf16", 320, 512, r1, counts, 2.0 * r1, wl.init_llm(320), 1401)
    p2 = wl.make_problem("l2", "bf16", 768, 264, r2, counts, 2.0 * r2, wl.init_llm(768), 1402)
    d1, d2 = DeviceProblem(p1), DeviceProblem(p2)
    layer = pl.PackedLoRALayer([(320, 512), (768, 264)], max_adapters=4, max_rank=200, max_tokens=p1.T)
    io = [{"X": d.X, "W": d.W, "A": d.A, "B": d.B, "dY": d.dY} for d in (d1, d2)]
    scales = [p1.scales, p2.scales]          # alpha / r per adapter differs between the projections
    fw = layer.forward(io, p1.off, scales)
    bw1 = layer.backward(io, p1.off, scales, [s for _, s in fw])
    torch.cuda.synchronize()
    assert layer.check() == pl.PLORA_OK
    for k, (p, d) in enumerate(((p1, d1), (p2, d2))):
        eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=4, max_rank=200, max_tokens=p.T)
        Y1, s1 = eng.forward(d.X, d.W, p1.off, p.scales, d.A, d.B)
        dX1, dA1, dB1 = eng.backward(d.X, d.W, d.dY, p1.off, p.scales, d.A, d.B, s1)
        torch.cuda.synchronize()
        assert torch.equal(fw[k][0], Y1), k
        assert torch.equal(bw1[k][0], dX1), k
        for i in range(4):
            assert torch.equal(bw1[k][1][i], dA1[i]) and torch.equal(bw1[k][2][i], dB1[i]), (k, i)
        eng.close()
    # a backward that skips every dX gives the same weight gradients
    bw2 = layer.backward(io, p1.off, scales, [s for _, s in fw], want_dX=False)
    torch.cuda.synchronize()
    assert layer.check() == pl.PLORA_OK
    for k in range(2):
        assert bw2[k][0] is None
        for i in range(4):
            assert torch.equal(bw2[k][1][i], bw1[k][1][i]) and torch.equal(bw2[k][2][i], bw1[k][2][i]), (k, i)
    layer.close()
