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


def test_output_blocks_llama_qkv_sampled():
    # LLaMA-3-8B q|k|v (4096 -> 4096 + 1024 + 1024), 16 adapters, r ~ U{16,32,64}, long-tail segment
    # lengths; each block against the oracle on sampled rows of Y / dX and sampled columns of dA / dB
    d_in, widths = 4096, [4096, 1024, 1024]
    rng = np.random.default_rng(31)
    ranks = rng.choice(np.array([16, 32, 64]), size=16)
    counts = np.round(np.exp(rng.uniform(np.log(256), np.log(2048), size=16))).astype(np.int64)
    r = np.asarray(ranks)
    d_out = sum(widths)
    base = wl.make_problem("qkv", "bf16", d_in, d_out, r, counts, 2.0 * r, wl.init_llm(d_in), 1201)
    # the k and v blocks' A factors (A depends on d_in and the ranks only; a 1-token draw suffices)
    extra = [wl.make_problem(f"qkv{b}", "bf16", d_in, 8, r, [1] * 16, 2.0 * r, wl.init_llm(d_in), 1201 + 100 * b).A
             for b in (1, 2)]
    A_blocks = [base.A] + extra
    stacked = dataclasses.replace(base, A=[np.concatenate([A_blocks[b][i] for b in range(3)]) for i in range(16)])
    eng = pl.PackedLoRA(d_in, d_out, "bf16", max_adapters=16, max_rank=64, max_tokens=stacked.T, out_blocks=widths)
    g = run(stacked, engine=eng)
    eng.close()
    rows = wl.sample_rows(stacked, per_segment=2)
    cols_a = np.unique(rng.integers(0, d_in, 48))
    nt = oracle.num_procs()
    dX_ref, c0 = 0.0, 0
    for b, w in enumerate(widths):
        cols = slice(c0, c0 + w)
        pb = dataclasses.replace(base, d_out=w, W=base.W[cols], dY=base.dY[:, cols], A=A_blocks[b],
                                 B=[x[cols] for x in base.B])
        cols_b = np.unique(rng.integers(0, w, 48))
        assert rel_err(g["Y"][rows][:, cols], oracle.forward(pb, rows=rows, nthreads=nt)["Y"]) <= BF16_TOL, b
        dX_ref = dX_ref + oracle.input_grad(pb, rows=rows, nthreads=nt)["dX"]
        o = oracle.weight_grads(pb, nthreads=nt, cols_a=cols_a, cols_b=cols_b)
        for i, ri in enumerate(r):
            ri = int(ri)
            assert rel_err(g["dA"][i][b * ri:(b + 1) * ri][:, cols_a], o["dA"][i][:, cols_a]) <= BF16_TOL, (b, i)
            assert rel_err(g["dB"][i][cols][cols_b], o["dB"][i][cols_b]) <= BF16_TOL, (b, i)
        c0 += w
    assert rel_err(g["dX"][rows], dX_ref) <= BF16_TOL
