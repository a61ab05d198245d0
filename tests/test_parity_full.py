"""GPU parity at the stated full sizes, with checks that see the low-rank branch.

At full size Y and dX are dominated by the frozen base term X W (entries of size ~1 against a LoRA
term of 0.01-0.2), so a max|err|/max|ref| <= 2e-2 check of Y and dX alone would not notice a
dropped or misrouted low-rank fold.  These tests therefore also run the same inputs with W = 0,
where Y and dX hold only the LoRA terms (X_i A_i B_i s_i and s_i dY_i B_i^T A_i^T), and compare
them with the fp64 oracle at full sensitivity.  The largest stated shapes are covered: the
LLaMA-3-8B layer's down projection (14336 -> 4096) and its gate|up pair (4096 -> 2 x 14336, one
call with output blocks) at 16 adapters x 8192 tokens = 131072 rows, where byte offsets into X and
dY pass 2^31, and a bit-exact segment signature over more than 65536 rows.

Y and dX are compared on sampled rows (the first, last and random rows of every segment, gathered
on the device); dA and dB on sampled hidden columns, for a few adapters, through the oracle run on
each adapter alone.  Tolerance: max|err|/max|ref| <= 2e-2 per tensor (bf16 inputs, fp32
accumulation); the signature is exact."""
import dataclasses

import numpy as np
import pytest

import oracle
import plora_workloads as wl
from plora_testlib import BF16_TOL, adapter_subproblem, cached_problem, rel_err, row_subproblem, run, run_sampled

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

NT = None


def nthreads():
    global NT
    if NT is None:
        NT = oracle.num_procs()
    return NT


def check_rows(p, g, rows, what):
    """Sampled rows of Y and dX against the oracle on the row sub-problem."""
    sub = row_subproblem(p, rows)
    oy = oracle.forward(sub, nthreads=nthreads())["Y"]
    ox = oracle.input_grad(sub, nthreads=nthreads())["dX"]
    ey, ex = rel_err(g["Y"], oy), rel_err(g["dX"], ox)
    assert ey <= BF16_TOL and ex <= BF16_TOL, (what, ey, ex)
    return ey, ex


def check_weight_grads(p, g, adapters, ncols=32, seed=11, blocks=None):
    """dA_i and dB_i of the listed adapters on sampled hidden columns, against the oracle run on
    each adapter alone (per output block when `blocks` lists the blocks' column ranges)."""
    rng = np.random.default_rng(seed)
    cols_a = np.unique(rng.integers(0, p.d_in, ncols))
    for i in adapters:
        r = int(p.ranks[i])
        for b, cols in enumerate(blocks or [slice(0, p.d_out)]):
            width = cols.stop - cols.start
            cols_b = np.unique(rng.integers(0, width, ncols))
            q = adapter_subproblem(p, i, out_cols=cols, A_rows=slice(b * r, (b + 1) * r) if blocks else None)
            o = oracle.weight_grads(q, nthreads=nthreads(), cols_a=cols_a, cols_b=cols_b)
            ga = g["dA"][i][b * r:(b + 1) * r] if blocks else g["dA"][i]
            gb = g["dB"][i][cols]
            ea = rel_err(ga[:, cols_a], o["dA"][0][:, cols_a])
            eb = rel_err(gb[cols_b], o["dB"][0][cols_b])
            assert ea <= BF16_TOL and eb <= BF16_TOL, (i, b, ea, eb)


# ----------------------------------------------------------------------------- the LoRA branch at full size
@pytest.mark.parametrize("path", ["tc", "tc_pair"])
def test_config3_lora_branch_with_zero_base(path):
    """The benchmark workload (LLaMA-3-8B up_proj, 32 long-tail adapters, 438 base tiles) with W = 0:
    every folded expand of the base GEMMs, every overlap record and the K-major row-padded B at
    d_out = 14336 are checked at full sensitivity."""
    p = wl.with_zero_W(cached_problem("config3", wl.config3))
    rows = wl.sample_rows(p, per_segment=2)
    g = run_sampled(p, rows, base_pair=(path == "tc_pair"))
    check_rows(p, g, rows, path)


def test_config5_mix_ii_lora_branch_with_zero_base():
    """1-token adapters next to 8192-token adapters (4096 -> 4096, rank 16) with W = 0: base tiles that
    straddle a 1-token segment fold two or three adapters."""
    p = wl.with_zero_W(wl.config5_mix("ii"))
    rows = wl.sample_rows(p, per_segment=6)
    g = run_sampled(p, rows)
    check_rows(p, g, rows, "mix ii")


# ----------------------------------------------------------------------------- config 4 at its stated size
def test_config4_down_projection_full_size():
    """The layer's down projection, 14336 -> 4096, 16 adapters x 8192 tokens = 131072 rows (X holds
    3.76 GB): sampled rows with the frozen W and again with W = 0, and the weight gradients of
    three adapters."""
    p = wl.config4_projection(6)
    assert p.name == "cfg4_llama_down" and p.T == 131072 and p.d_in == 14336
    rows = wl.sample_rows(p, per_segment=2)
    g = run_sampled(p, rows)
    check_rows(p, g, rows, "down")
    check_weight_grads(p, g, [0, 7, 15])
    z = wl.with_zero_W(p)
    check_rows(z, run_sampled(z, rows), rows, "down, W = 0")


def test_config4_gate_up_output_blocks_full_size():
    """The layer's gate and up projections, which read the same input, as one call with two output
    blocks (4096 -> 2 x 14336; dY holds 7.5 GB), 16 adapters x 8192 tokens: each block's sampled rows
    of Y against the oracle on that projection alone, dX against the sum of both projections' input
    gradients, and the per-block weight gradients of two adapters."""
    ranks = wl.config4_ranks()
    widths = [14336, 14336]
    base = wl.make_problem("cfg4_llama_gate_up", "bf16", 4096, sum(widths), ranks, [8192] * 16, 2.0 * ranks,
                           wl.init_llm(4096), 1004 * 16 + 4)
    extra = wl.make_problem("cfg4_llama_gate_up_a1", "bf16", 4096, 256, ranks, [8192] * 16, 2.0 * ranks,
                            wl.init_llm(4096), 1004 * 16 + 5, draw_tokens=False)
    p = dataclasses.replace(base, A=[np.concatenate([base.A[i], extra.A[i]]) for i in range(16)])
    blocks = [slice(0, widths[0]), slice(widths[0], sum(widths))]
    rows = wl.sample_rows(p, per_segment=2)
    g = run_sampled(p, rows, out_blocks=widths)
    sub = row_subproblem(p, rows)
    dX_ref = 0.0
    for b, cols in enumerate(blocks):
        pb = dataclasses.replace(sub, d_out=widths[b], W=np.ascontiguousarray(p.W[cols]),
                                 dY=np.ascontiguousarray(sub.dY[:, cols]),
                                 A=[np.ascontiguousarray(a[b * int(r):(b + 1) * int(r)]) for a, r in zip(p.A, ranks)],
                                 B=[np.ascontiguousarray(x[cols]) for x in p.B])
        ey = rel_err(g["Y"][:, cols], oracle.forward(pb, nthreads=nthreads())["Y"])
        assert ey <= BF16_TOL, ("Y block", b, ey)
        dX_ref = dX_ref + oracle.input_grad(pb, nthreads=nthreads())["dX"]
    assert rel_err(g["dX"], dX_ref) <= BF16_TOL
    check_weight_grads(p, g, [1, 14], blocks=blocks)


# ----------------------------------------------------------------------------- exact, beyond 65536 rows
@pytest.mark.parametrize("path", ["tc", "tc_pair"])
def test_segment_signature_beyond_64k_rows(path):
    """Y[t][c] = s_adapter(t) exactly and dA_i[0][0] = dB_i[0][0] = s_i n_i exactly, over 70135 rows
    (a 70000-token adapter between a 1-token and a 129-token one, an empty one and a 5-token one)."""
    from test_oracle import signature_problem
    counts = [1, 70000, 129, 0, 5]
    p = signature_problem(counts, dtype="bf16", d_in=256, d_out=256, rank=3)
    g = run(p, base_pair=(path == "tc_pair"))
    seg = np.repeat(np.arange(len(counts)), counts)
    assert np.array_equal(g["Y"], np.broadcast_to((seg + 1)[:, None].astype(np.float64), g["Y"].shape))
    for i, n in enumerate(counts):
        e = np.zeros_like(g["dB"][i]); e[0, 0] = (i + 1) * n
        assert np.array_equal(g["dB"][i], e), i
        e = np.zeros_like(g["dA"][i]); e[0, 0] = (i + 1) * n
        assert np.array_equal(g["dA"][i], e), i
