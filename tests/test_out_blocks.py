"""GPU parity of output blocks: P shared-input projections (q, k, v, say) stacked in one W and run
as one packed call, against the fp64 oracle run on each projection alone.  For block p the
definition is the plain one over its slice: Y[:, block p] = X W_p^T + s X A_p^T B_p^T, and dX is
the sum of the blocks' input gradients.  Tolerance as in test_parity: max|err|/max|ref| <= 2e-2
per tensor (bf16 inputs, fp32 accumulation)."""
import dataclasses

import numpy as np
import pytest

import oracle
import plora_workloads as wl
from plora_testlib import BF16_TOL, DeviceProblem, rel_err, run

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402


def blocked_problem(seed, d_in, widths, ranks, counts):
    """The stacked problem (A_i with one rank-r block per projection) and each projection's own."""
    r = np.asarray(ranks)
    d_out = int(sum(widths))
    base = wl.make_problem(f"blk{seed}", "bf16", d_in, d_out, r, counts, 2.0 * r, wl.init_llm(d_in), seed)
    extra = [wl.make_problem(f"blk{seed}a{b}", "bf16", d_in, d_out, r, counts, 2.0 * r, wl.init_llm(d_in),
                             seed + 100 * b) for b in range(1, len(widths))]
    A_blocks = [base.A] + [e.A for e in extra]          # A_blocks[b][i]: [r_i][d_in]
    stacked = dataclasses.replace(base, A=[np.concatenate([A_blocks[b][i] for b in range(len(widths))])
                                           for i in range(len(r))])
    per_block, c0 = [], 0
    for b, w in enumerate(widths):
        cols = slice(c0, c0 + w)
        per_block.append((cols, dataclasses.replace(base, d_out=w, W=base.W[cols], dY=base.dY[:, cols],
                                                    A=A_blocks[b], B=[x[cols] for x in base.B])))
        c0 += w
    return stacked, per_block


CASES = [
    # d_in, block widths, ranks, counts (ragged tails, rank 1 and a rank whose padding differs, an
    # empty and a 1-token segment)
    (384, [512, 256, 256], [1, 16, 24, 64, 3], [300, 129, 0, 1000, 1]),
    (1024, [1024, 256, 256], [8, 32, 80], [700, 1, 513]),
    (264, [256, 256], [128, 5], [260, 97]),
]


@pytest.mark.parametrize("k", range(len(CASES)))
def test_output_blocks_match_each_projection_alone(k):
    d_in, widths, ranks, counts = CASES[k]
    stacked, per_block = blocked_problem(900 + k, d_in, widths, ranks, counts)
    eng = pl.PackedLoRA(d_in, sum(widths), "bf16", max_adapters=len(ranks), max_rank=max(ranks),
                        max_tokens=stacked.T, out_blocks=widths)
    g = run(stacked, engine=eng)
    eng.close()
    dX_ref = 0.0
    for b, (cols, pb) in enumerate(per_block):
        o = oracle.full(pb, nthreads=oracle.num_procs())
        assert rel_err(g["Y"][:, cols], o["Y"]) <= BF16_TOL, ("Y", b)
        dX_ref = dX_ref + o["dX"]
        for i, r in enumerate(ranks):
            assert rel_err(g["dA"][i][b * r:(b + 1) * r], o["dA"][i]) <= BF16_TOL, ("dA", b, i)
            assert rel_err(g["dB"][i][cols], o["dB"][i]) <= BF16_TOL, ("dB", b, i)
    assert rel_err(g["dX"], dX_ref) <= BF16_TOL


def test_output_blocks_saved_activation_per_block():
    # the saved H'_i = s_i X_i A_i^T comes back with block b's rank columns at b r .. b r + r - 1
    d_in, widths, ranks, counts = CASES[0]
    stacked, per_block = blocked_problem(950, d_in, widths, ranks, counts)
    eng = pl.PackedLoRA(d_in, sum(widths), "bf16", max_adapters=len(ranks), max_rank=max(ranks),
                        max_tokens=stacked.T, out_blocks=widths)
    d = DeviceProblem(stacked)
    Y, saved = eng.forward(d.X, d.W, stacked.off, stacked.scales, d.A, d.B)
    tab = eng.table(stacked.scales, d.A, d.B)
    refs = [oracle.forward(pb, want_H=True)["H"] for _, pb in per_block]   # X A_b^T, fp64, all rows
    for i, r in enumerate(ranks):
        n = int(counts[i])
        H = torch.zeros((max(n, 1), len(widths) * r), dtype=torch.float32, device="cuda")
        pl.plora_debug_unpack_saved(eng.h, len(ranks), stacked.off, tab, saved.data_ptr(), i, H.data_ptr())
        torch.cuda.synchronize()
        if n == 0:
            continue
        got = H.cpu().numpy().astype(np.float64)[:n]
        a, e = int(stacked.off[i]), int(stacked.off[i + 1])
        for b in range(len(widths)):
            ref = float(stacked.scales[i]) * refs[b][a:e, :r]
            assert rel_err(got[:, b * r:(b + 1) * r], ref) <= BF16_TOL, (i, b)
    eng.close()


def test_output_blocks_equal_separate_calls_bit_for_bit():
    # Every output column accumulates on its own, and the block-diagonal zeros add exact zeros, so
    # the fused call reproduces each projection's own call exactly in Y, dA and dB; dX (a sum over
    # the blocks) agrees within the bf16 tolerance with the sum of the separate dX.
    d_in, widths, ranks, counts = CASES[1]
    stacked, per_block = blocked_problem(970, d_in, widths, ranks, counts)
    eng = pl.PackedLoRA(d_in, sum(widths), "bf16", max_adapters=len(ranks), max_rank=max(ranks),
                        max_tokens=stacked.T, out_blocks=widths)
    g = run(stacked, engine=eng)
    eng.close()
    dX_sum = 0.0
    for b, (cols, pb) in enumerate(per_block):
        h = run(pb, max_tokens=stacked.T)
        assert np.array_equal(g["Y"][:, cols], h["Y"]), b
        for i, r in enumerate(ranks):
            assert np.array_equal(g["dA"][i][b * r:(b + 1) * r], h["dA"][i]), (b, i)
            assert np.array_equal(g["dB"][i][cols], h["dB"][i]), (b, i)
        dX_sum = dX_sum + h["dX"]
    assert rel_err(g["dX"], dX_sum) <= BF16_TOL
