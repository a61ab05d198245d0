"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Tolerances: max|err|/max|ref| per output tensor <= 2e-2
for bf16 inputs with fp32 accumulation, <= 1e-5 for the fp32 path.  Integer
and indexing results (segment signature, B = 0, packed == alone, repeat runs)
must match bit for bit."""
import dataclasses

import numpy as np
import pytest

import oracle
import plora_workloads as wl
from plora_testlib import BF16_TOL, FP32_TOL, DeviceProblem, cached_problem, compare, rel_err, run

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402


def tol(p):
    return BF16_TOL if p.dtype == "bf16" else FP32_TOL


def full_oracle(p):
    return oracle.full(p, nthreads=oracle.num_procs())


def mix(seed, dtype, d_in, d_out, ranks, counts):
    r = np.asarray(ranks)
    init = wl.init_small(d_in) if dtype == "fp32" else wl.init_llm(d_in)
    return wl.make_problem(f"mix{seed}", dtype, d_in, d_out, r, counts, 2.0 * r, init, seed)


# ----------------------------------------------------------------------------- small, full comparison
def test_config1_fp32():
    p = wl.config1()
    errs, bad = compare(p, run(p), full_oracle(p), FP32_TOL)
    assert not bad, bad


MIXES = [
    # d_in, d_out, ranks, counts  (ragged tails, rank 1 and 256, empty and 1-token segments,
    # hidden sizes that are not multiples of the 128/256 tiles)
    (256, 256, [4, 8, 8, 16], [64, 128, 32, 96]),
    (520, 328, [1, 3, 17, 64, 100], [1, 127, 129, 0, 300]),
    (384, 1032, [256, 1, 16], [200, 77, 256]),
    (136, 72, [8, 2, 33, 5, 64, 7], [5, 0, 140, 1, 66, 250]),
    (1024, 512, [32, 32, 128], [513, 0, 1000]),
]


@pytest.mark.parametrize("k", range(len(MIXES)))
@pytest.mark.parametrize("path", ["tc", "tc_pair", "tc_unfused", "simt", "fp32"])
def test_small_mixes(k, path):
    d_in, d_out, ranks, counts = MIXES[k]
    p = mix(100 + k, "fp32" if path == "fp32" else "bf16", d_in, d_out, ranks, counts)
    g = run(p, simt=(path == "simt"), unfused=(path == "tc_unfused"), base_pair=(path == "tc_pair"))
    errs, bad = compare(p, g, full_oracle(p), tol(p))
    assert not bad, (bad, errs)


@pytest.mark.parametrize("unfused", [False, True])
def test_lora_delta_with_zero_base(unfused):
    """W = 0: Y and dX hold only the LoRA terms, so the bf16 check sees them at full sensitivity."""
    for k in (1, 2, 3):
        d_in, d_out, ranks, counts = MIXES[k]
        p = wl.with_zero_W(mix(200 + k, "bf16", d_in, d_out, ranks, counts))
        errs, bad = compare(p, run(p, unfused=unfused), full_oracle(p), BF16_TOL)
        assert not bad, (bad, errs)


@pytest.mark.parametrize("base_pair", [False, True])
def test_many_adapters_in_one_tile(base_pair):
    """1- and 2-token adapters: a base-GEMM tile overlaps many adapters."""
    counts = [1, 2, 1, 0, 3, 1, 130, 1, 1, 5, 1, 2, 250, 1]
    ranks = [1, 8, 16, 4, 64, 3, 32, 256, 2, 17, 1, 8, 100, 5]
    p = wl.with_zero_W(mix(250, "bf16", 264, 392, ranks, counts))
    errs, bad = compare(p, run(p, base_pair=base_pair), full_oracle(p), BF16_TOL)
    assert not bad, (bad, errs)


def test_weight_grad_split_path():
    """Adapters longer than the split size exercise the split partials and their fixed-order reduction."""
    p = mix(300, "bf16", 256, 384, [16, 96, 8], [34000, 16385, 300])
    errs, bad = compare(p, run(p), full_oracle(p), BF16_TOL)
    assert not bad, (bad, errs)


def test_narrow_last_n_tile_over_many_tiles():
    """Outputs whose last n-tile is narrower than 256 columns (d_out = 392: a 136-column last tile; dX:
    136 columns) store an odd number of 64-column chunks per 128-row half, and 100 000 rows give every
    SM several 256-row tiles in a row: the epilogue's staging buffers must alternate across calls, not
    restart per call.  Full comparison with the oracle, and two runs bit-identical."""
    p = mix(330, "bf16", 136, 392, [8, 16, 32, 4, 64], [40000, 1, 30000, 129, 29870])
    g = run(p)
    errs, bad = compare(p, g, full_oracle(p), BF16_TOL)
    assert not bad, (bad, errs)
    h = run(p)
    assert np.array_equal(g["Y"], h["Y"]) and np.array_equal(g["dX"], h["dX"])


@pytest.mark.parametrize("counts", [[1], [0, 129], [128, 127], [256], [200, 57], [1, 384]])
@pytest.mark.parametrize("path", ["tc", "tc_unfused"])
def test_row_counts_at_the_256_row_tile_edges(counts, path):
    """Packed row counts at and around a base-GEMM tile (256 rows) and its 128-row halves: a half with no
    rows, a single row, a full tile, one row past it.  d_in = 64 gives Y's tiles a single base k-block
    (the whole tile fits the ring at once), d_out = 448 gives dX's seven (first, middle and last
    k-blocks), and dX's 64 columns are one output chunk.  Full oracle comparison, with W as drawn and
    with W = 0 (Y and dX then hold only the low-rank terms)."""
    ranks = [16, 40][:len(counts)]
    p = mix(340 + sum(counts), "bf16", 64, 448, ranks, counts)
    for q in (p, wl.with_zero_W(p)):
        errs, bad = compare(q, run(q, unfused=(path == "tc_unfused")), full_oracle(q), BF16_TOL)
        assert not bad, (bad, errs)


def test_no_dX_gives_same_weight_grads():
    p = mix(310, "bf16", 520, 328, [1, 3, 17, 64, 100], [1, 127, 129, 0, 300])
    a, b = run(p), run(p, want_dX=False)
    for i in range(p.n_adapters):
        assert np.array_equal(a["dA"][i], b["dA"][i]) and np.array_equal(a["dB"][i], b["dB"][i])


# ----------------------------------------------------------------------------- exact checks
def signature_problem(counts, d_in=256, d_out=256, rank=3, dtype="bf16"):
    from test_oracle import signature_problem as sp
    return sp(counts, dtype=dtype, d_in=d_in, d_out=d_out, rank=rank)


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_segment_signature_bit_exact(path):
    counts = [1, 0, 8192, 127, 128, 129, 5]
    p = signature_problem(counts)
    g = run(p, simt=(path == "simt"))
    seg = np.repeat(np.arange(len(counts)), counts)
    assert np.array_equal(g["Y"], np.broadcast_to((seg + 1)[:, None].astype(np.float64), g["Y"].shape))
    for i, n in enumerate(counts):
        eB = np.zeros_like(g["dB"][i]); eB[0, 0] = (i + 1) * n
        eA = np.zeros_like(g["dA"][i]); eA[0, 0] = (i + 1) * n
        assert np.array_equal(g["dB"][i], eB), i
        assert np.array_equal(g["dA"][i], eA), i


def test_B_zero_gives_base_and_zero_dA_exactly():
    d_in, d_out, ranks, counts = MIXES[1]
    p = wl.with_zero_B(mix(400, "bf16", d_in, d_out, ranks, counts))
    q = dataclasses.replace(p, A=[np.zeros_like(a) for a in p.A])
    g, h = run(p), run(q)
    assert np.array_equal(g["Y"], h["Y"])
    assert np.array_equal(g["dX"], h["dX"])
    for i in range(p.n_adapters):
        assert not np.any(g["dA"][i])
    errs, bad = compare(p, g, full_oracle(p), BF16_TOL)
    assert not bad, bad


@pytest.mark.parametrize("path", ["tc", "tc_pair", "tc_unfused", "simt"])
def test_packed_equals_alone_bit_exact(path):
    d_in, d_out, ranks, counts = (384, 520, [1, 16, 100, 64, 8], [300, 129, 0, 16500, 1])
    p = mix(500, "bf16", d_in, d_out, ranks, counts)
    g = run(p, simt=(path == "simt"), unfused=(path == "tc_unfused"), base_pair=(path == "tc_pair"))
    for i in range(p.n_adapters):
        a, b = int(p.off[i]), int(p.off[i + 1])
        q = dataclasses.replace(p, off=np.array([0, b - a], np.int64), ranks=p.ranks[i:i + 1],
                                alphas=p.alphas[i:i + 1], scales=p.scales[i:i + 1], X=p.X[a:b],
                                A=[p.A[i]], B=[p.B[i]], dY=p.dY[a:b])
        h = run(q, simt=(path == "simt"), unfused=(path == "tc_unfused"), base_pair=(path == "tc_pair"))
        assert np.array_equal(h["Y"], g["Y"][a:b]), i
        assert np.array_equal(h["dX"], g["dX"][a:b]), i
        assert np.array_equal(h["dA"][0], g["dA"][i]), i
        assert np.array_equal(h["dB"][0], g["dB"][i]), i


def test_repeat_runs_bit_identical():
    p = mix(600, "bf16", 520, 328, [1, 3, 17, 64, 100], [1, 127, 129, 0, 17000])
    dev = DeviceProblem(p)
    a, b = run(p, dev=dev), run(p, dev=dev)
    for k in ("Y", "dX"):
        assert np.array_equal(a[k], b[k])
    for i in range(p.n_adapters):
        assert np.array_equal(a["dA"][i], b["dA"][i]) and np.array_equal(a["dB"][i], b["dB"][i])


def test_saved_activations_match_oracle_H():
    d_in, d_out, ranks, counts = MIXES[1]
    p = mix(700, "bf16", d_in, d_out, ranks, counts)
    eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=8, max_rank=256, max_tokens=p.T)
    d = DeviceProblem(p)
    Y, saved = eng.forward(d.X, d.W, p.off, p.scales, d.A, d.B)
    tab = eng.table(p.scales, d.A, d.B)
    o = oracle.forward(p, want_H=True)
    for i in range(p.n_adapters):
        n, r = int(p.counts[i]), int(p.ranks[i])
        H = torch.zeros((max(n, 1), r), dtype=torch.float32, device="cuda")
        pl.plora_debug_unpack_saved(eng.h, p.n_adapters, p.off, tab, saved.data_ptr(), i, H.data_ptr())
        torch.cuda.synchronize()
        if n:
            ref = float(p.scales[i]) * o["H"][p.off[i]:p.off[i + 1], :r]   # saved holds s_i X_i A_i
            assert rel_err(H.cpu().numpy()[:n], ref) <= BF16_TOL
    eng.close()


def test_empty_calls():
    p = mix(800, "bf16", 256, 256, [4, 8], [0, 0])
    g = run(p, max_tokens=16)
    for i in range(2):
        assert not np.any(g["dA"][i]) and not np.any(g["dB"][i])


def test_invalid_call_writes_nothing():
    p = mix(900, "bf16", 256, 256, [4, 8], [10, 20])
    eng = pl.PackedLoRA(256, 256, "bf16", max_adapters=2, max_rank=8, max_tokens=30)
    d = DeviceProblem(p)
    Y = torch.full((p.T, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    tab = eng.table(p.scales, d.A, d.B)
    saved = torch.empty(eng.saved_bytes(p.off, tab), dtype=torch.uint8, device="cuda")
    bad_off = np.array([0, 20, 10], np.int64)
    s = pl.plora_forward(eng.h, d.X.data_ptr(), d.W.data_ptr(), Y.data_ptr(), 2, bad_off, tab, saved.data_ptr(),
                         0, check=False)
    assert s == pl.PLORA_ERR_INVALID_ARG and "decrease" in pl.plora_last_error(eng.h)
    s = pl.plora_forward(eng.h, d.X.data_ptr() + 2, d.W.data_ptr(), Y.data_ptr(), 2, p.off, tab,
                         saved.data_ptr(), 0, check=False)
    assert s == pl.PLORA_ERR_INVALID_ARG
    # a host pointer: refused by the extent check, nothing launched
    host_X = np.zeros((p.T, 256), np.uint16)
    s = pl.plora_forward(eng.h, host_X.ctypes.data, d.W.data_ptr(), Y.data_ptr(), 2, p.off, tab, saved.data_ptr(),
                         0, check=False)
    assert s == pl.PLORA_ERR_INVALID_ARG and "X is not a device buffer" in pl.plora_last_error(eng.h)
    torch.cuda.synchronize()
    assert bool(torch.all(Y == 7.0))
    assert pl.plora_check(eng.h, 0) == pl.PLORA_OK
    eng.close()


# ----------------------------------------------------------------------------- full-size workloads
def test_config2_qwen_q_proj():
    p = wl.config2()
    g = run(p)
    rows = wl.sample_rows(p, per_segment=4)
    cols = np.unique(np.random.default_rng(5).integers(0, p.d_in, 96))
    nt = oracle.num_procs()
    o = {"Y": oracle.forward(p, rows=rows, nthreads=nt)["Y"],
         "dX": oracle.input_grad(p, rows=rows, nthreads=nt)["dX"]}
    o.update(oracle.weight_grads(p, nthreads=nt, cols_a=cols, cols_b=cols))
    errs, bad = compare(p, g, o, BF16_TOL, rows=rows, cols_a=cols, cols_b=cols)
    assert not bad, (bad, errs)


@pytest.mark.parametrize("path", ["tc", "tc_pair"])
def test_config3_llama_up_proj_32_adapters(path):
    """The benchmark workload (LLaMA-3-8B up_proj, 32 long-tail adapters) on sampled outputs, with the
    base GEMMs on single SMs (the default) and on SM pairs."""
    p = cached_problem("config3", wl.config3)
    g = run(p, base_pair=(path == "tc_pair"))
    rows = wl.sample_rows(p, per_segment=2)
    rng = np.random.default_rng(6)
    cols_a = np.unique(rng.integers(0, p.d_in, 64))
    cols_b = np.unique(rng.integers(0, p.d_out, 64))
    nt = oracle.num_procs()
    o = {"Y": oracle.forward(p, rows=rows, nthreads=nt)["Y"],
         "dX": oracle.input_grad(p, rows=rows, nthreads=nt)["dX"]}
    o.update(oracle.weight_grads(p, nthreads=nt, cols_a=cols_a, cols_b=cols_b))
    errs, bad = compare(p, g, o, BF16_TOL, rows=rows, cols_a=cols_a, cols_b=cols_b)
    assert not bad, (bad, errs)


def sampled_check(p, g, per_segment=2, ncols=48, seed=8):
    rows = wl.sample_rows(p, per_segment=per_segment)
    rng = np.random.default_rng(seed)
    cols_a = np.unique(rng.integers(0, p.d_in, ncols))
    cols_b = np.unique(rng.integers(0, p.d_out, ncols))
    nt = oracle.num_procs()
    o = {"Y": oracle.forward(p, rows=rows, nthreads=nt)["Y"],
         "dX": oracle.input_grad(p, rows=rows, nthreads=nt)["dX"]}
    o.update(oracle.weight_grads(p, nthreads=nt, cols_a=cols_a, cols_b=cols_b))
    return compare(p, g, o, BF16_TOL, rows=rows, cols_a=cols_a, cols_b=cols_b)


@pytest.mark.parametrize("which", ["i", "ii", "iii", "iv"])
def test_config5_degenerate_mixes(which):
    """Full-size degenerate mixes: rank 1 next to rank 256, 1-token next to 8192-token segments,
    mixed ranks over equal segments, and an adapter with no tokens."""
    p = wl.config5_mix(which)
    errs, bad = sampled_check(p, run(p))
    assert not bad, (which, bad, errs)


def test_config5_scaling_32_adapters():
    p = wl.config5_scaling(32)
    errs, bad = sampled_check(p, run(p))
    assert not bad, (bad, errs)


@pytest.mark.parametrize("proj", range(7))
def test_config4_layer_projection_shapes(proj):
    """Each of the LLaMA-3-8B layer's seven projection shapes (q, k, v, o, gate, up, down; the down
    projection reads 14336-wide inputs), 16 adapters r ~ U{16,32,64}, at 512 tokens per adapter."""
    nm, di, do = wl.LLAMA3_LAYER[proj]
    ranks = wl.rng_for(1004, 1).choice(np.array([16, 32, 64]), size=16)
    p = wl.make_problem(f"cfg4s_{nm}", "bf16", di, do, ranks, [512] * 16, 2.0 * ranks, wl.init_llm(di),
                        1004 * 16 + proj)
    errs, bad = sampled_check(p, run(p))
    assert not bad, (nm, bad, errs)
