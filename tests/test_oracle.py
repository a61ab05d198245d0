"""Pins for the fp64 oracle: properties the mathematics fixes, checked on the CPU.

Each test checks the oracle against something other than itself: a library
matmul on the merged weight, closed forms, invariants, exact finite
differences, or a hand-derived example.  A dropped term, a wrong sign, a wrong
index or a transposed operand anywhere in ``oracle.c`` fails at least one.
"""
import dataclasses
import json
import os

import numpy as np
import pytest

import oracle
import plora_workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small(seed, dtype="fp32", d_in=24, d_out=20, ranks=(1, 3, 8, 5), counts=(7, 0, 12, 5)):
    r = np.asarray(ranks)
    return wl.make_problem("small", dtype, d_in, d_out, r, counts, 2.0 * r + 1.0,
                           wl.init_small(d_in), seed)


def f64(p, a):
    return wl.to_f64(a, p.dtype)


def merged_reference(p):
    """Y and dX through the merged weight W_eff = W + s_i A_i B_i, one library matmul per segment.
    Merging the low-rank patch into the base weight gives the full weight ('LLM+LoRA微调加速技术原理解析',
    深入理解LoRA：基本原理与PEFT实现: the released LoRA weight is a patch merged into the original)."""
    Wt = f64(p, p.W).T                      # W[j][c]
    Y = np.zeros((p.T, p.d_out))
    dX = np.zeros((p.T, p.d_in))
    X, dY = f64(p, p.X), f64(p, p.dY)
    for i in range(p.n_adapters):
        a, b = p.off[i], p.off[i + 1]
        A = f64(p, p.A[i]).T                # A_i[j][k]
        B = f64(p, p.B[i]).T                # B_i[k][c]
        Weff = Wt + float(p.scales[i]) * (A @ B)
        Y[a:b] = X[a:b] @ Weff
        dX[a:b] = dY[a:b] @ Weff.T
    return Y, dX


def rel(a, b):
    den = np.max(np.abs(b)) if np.size(b) else 0.0
    return float(np.max(np.abs(a - b)) / den) if den > 0 else float(np.max(np.abs(a - b), initial=0.0))


@pytest.mark.parametrize("seed", [1, 2, 3])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_forward_and_input_grad_match_merged_weight(seed, dtype):
    p = small(seed, dtype)
    Y, dX = merged_reference(p)
    o = oracle.forward(p)
    g = oracle.input_grad(p)
    assert rel(o["Y"], Y) < 1e-12
    assert rel(g["dX"], dX) < 1e-12


def test_config1_matches_merged_weight():
    p = wl.config1()
    Y, dX = merged_reference(p)
    assert rel(oracle.forward(p)["Y"], Y) < 1e-12
    assert rel(oracle.input_grad(p)["dX"], dX) < 1e-12


def test_hand_derived_integer_example():
    g = json.load(open(os.path.join(GOLDEN, "tiny_integer_example.json")))
    r = np.asarray(g["ranks"], dtype=np.int32)
    al = np.asarray(g["alphas"], dtype=np.float64)
    p = wl.Problem("golden", "fp32", g["d_in"], g["d_out"], np.asarray(g["off"], dtype=np.int64), r, al,
                   (al / r).astype(np.float32), np.asarray(g["X"], np.float32),
                   np.asarray(g["W_store"], np.float32), [np.asarray(a, np.float32) for a in g["A_store"]],
                   [np.asarray(b, np.float32) for b in g["B_store"]], np.asarray(g["dY"], np.float32))
    o = oracle.full(p)
    e = g["expect"]
    assert np.array_equal(o["Y"], np.asarray(e["Y"], float))
    assert np.array_equal(o["dX"], np.asarray(e["dX"], float))
    for i in range(2):
        assert np.array_equal(o["dA"][i], np.asarray(e["dA_store"][i], float))
        assert np.array_equal(o["dB"][i], np.asarray(e["dB_store"][i], float))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_B_zero_gives_base_exactly_and_zero_dA(dtype):
    """B = 0 (the LoRA init of B): Y = X W exactly, dA = 0 exactly, dB = s H^T dY."""
    p = wl.with_zero_B(small(11, dtype))
    q = dataclasses.replace(p, A=[np.zeros_like(a) for a in p.A])     # branch removed another way
    o, oq = oracle.full(p), oracle.full(q)
    assert np.array_equal(o["Y"], oq["Y"])
    assert np.array_equal(o["dX"], oq["dX"])
    base = f64(p, p.X) @ f64(p, p.W).T
    assert rel(o["Y"], base) < 1e-12
    assert rel(o["dX"], f64(p, p.dY) @ f64(p, p.W)) < 1e-12
    X, dY = f64(p, p.X), f64(p, p.dY)
    for i in range(p.n_adapters):
        assert not np.any(o["dA"][i])
        a, b = p.off[i], p.off[i + 1]
        H = X[a:b] @ f64(p, p.A[i]).T
        dB = float(p.scales[i]) * (dY[a:b].T @ H)
        assert rel(o["dB"][i], dB) < 1e-12 or (b == a and not np.any(o["dB"][i]))


def test_rank1_outer_product_closed_forms():
    """Rank 1: A = a, B = b^T.  Y - XW = s (X a) b^T; dB = s dY^T (X a); dA = s X^T (dY b)."""
    p = small(21, "fp32", ranks=(1, 1, 1), counts=(9, 4, 6))
    o = oracle.full(p)
    pb = wl.with_zero_B(p)
    base = oracle.forward(pb)["Y"]
    base_dx = oracle.input_grad(pb)["dX"]
    X, dY = f64(p, p.X), f64(p, p.dY)
    for i in range(3):
        a, b = p.off[i], p.off[i + 1]
        av = f64(p, p.A[i])[0]              # a[j]
        bv = f64(p, p.B[i])[:, 0]           # b[c]
        s = float(p.scales[i])
        assert rel(o["Y"][a:b] - base[a:b], s * np.outer(X[a:b] @ av, bv)) < 1e-12
        assert rel(o["dX"][a:b] - base_dx[a:b], s * np.outer(dY[a:b] @ bv, av)) < 1e-12
        assert rel(o["dB"][i][:, 0], s * (dY[a:b].T @ (X[a:b] @ av))) < 1e-12
        assert rel(o["dA"][i][0], s * (X[a:b].T @ (dY[a:b] @ bv))) < 1e-12


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_packed_equals_each_adapter_alone(dtype):
    """Packing does not change any adapter's result: bit-exact in the oracle."""
    p = small(31, dtype)
    o = oracle.full(p)
    for i in range(p.n_adapters):
        a, b = int(p.off[i]), int(p.off[i + 1])
        q = dataclasses.replace(p, off=np.array([0, b - a], np.int64), ranks=p.ranks[i:i + 1],
                                alphas=p.alphas[i:i + 1], scales=p.scales[i:i + 1], X=p.X[a:b],
                                A=[p.A[i]], B=[p.B[i]], dY=p.dY[a:b])
        oq = oracle.full(q)
        assert np.array_equal(oq["Y"], o["Y"][a:b])
        assert np.array_equal(oq["dX"], o["dX"][a:b])
        assert np.array_equal(oq["dA"][0], o["dA"][i])
        assert np.array_equal(oq["dB"][0], o["dB"][i])


def test_linear_in_scale():
    """dA and dB scale exactly by 2 with s -> 2s; Y - XW and dX - dY W^T scale by 2 up to roundoff."""
    p = small(41, "fp32")
    q = dataclasses.replace(p, scales=(2 * p.scales).astype(np.float32))
    o, oq = oracle.full(p), oracle.full(q)
    for i in range(p.n_adapters):
        assert np.array_equal(oq["dA"][i], 2 * o["dA"][i])
        assert np.array_equal(oq["dB"][i], 2 * o["dB"][i])
    pb = oracle.full(wl.with_zero_B(p))
    assert rel(oq["Y"] - pb["Y"], 2 * (o["Y"] - pb["Y"])) < 1e-12
    assert rel(oq["dX"] - pb["dX"], 2 * (o["dX"] - pb["dX"])) < 1e-12


def _loss(p):
    """L = <dY, Y>: its gradients are exactly dX, dA, dB."""
    return float(np.sum(f64(p, p.dY) * oracle.forward(p)["Y"]))


def test_gradients_match_central_finite_differences():
    """L is linear in X, in A and in B separately, so the central difference with the
    actually representable perturbation is exact up to fp64 roundoff."""
    r = np.asarray([1, 2, 3])
    p = wl.make_problem("fd", "fp32", 8, 6, r, [2, 0, 3], 2.0 * r + 1.0, wl.init_small(8), 51)
    o = oracle.full(p)
    h = np.float32(0.0625)

    def fd(get, put, idx):
        base = get()
        up, dn = base.copy(), base.copy()
        up[idx] = base[idx] + h
        dn[idx] = base[idx] - h
        put(up)
        lp = _loss(p)
        put(dn)
        lm = _loss(p)
        put(base)
        return (lp - lm) / (float(up[idx]) - float(dn[idx]))

    scale = max(np.max(np.abs(o["dX"])), 1.0)
    for t in range(p.T):
        for j in range(p.d_in):
            g = fd(lambda: p.X, lambda v: setattr(p, "X", v), (t, j))
            assert abs(g - o["dX"][t, j]) <= 1e-10 * scale
    for i in range(p.n_adapters):
        for k in range(int(r[i])):
            for j in range(p.d_in):
                g = fd(lambda: p.A[i], lambda v: p.A.__setitem__(i, v), (k, j))
                assert abs(g - o["dA"][i][k, j]) <= 1e-10 * scale
            for c in range(p.d_out):
                g = fd(lambda: p.B[i], lambda v: p.B.__setitem__(i, v), (c, k))
                assert abs(g - o["dB"][i][c, k]) <= 1e-10 * scale
    assert not np.any(o["dA"][1]) and not np.any(o["dB"][1])      # the empty segment


def signature_problem(counts, dtype="fp32", d_in=16, d_out=24, rank=3):
    """Segment signature: W = 0, X[t][0] = 1, A_store_i[0][0] = 1, B_store_i[c][0] = 1, s_i = i + 1,
    dY[t][0] = 1.  Then Y[t][c] = s_adapter(t), dB_store_i[0][0] = dA_store_i[0][0] = s_i n_i."""
    n = len(counts)
    off = np.zeros(n + 1, np.int64)
    off[1:] = np.cumsum(counts)
    T = int(off[-1])
    one = wl.from_f64(np.ones(1), dtype)[0]
    zero = wl.from_f64(np.zeros(1), dtype)[0]

    def z(shape):
        return np.full(shape, zero)
    X = z((T, d_in)); X[:, 0] = one
    dY = z((T, d_out)); dY[:, 0] = one
    A, B = [], []
    for i in range(n):
        a = z((rank, d_in)); a[0, 0] = one; A.append(a)
        b = z((d_out, rank)); b[:, 0] = one; B.append(b)
    ranks = np.full(n, rank, np.int32)
    scales = np.arange(1, n + 1, dtype=np.float32)
    return wl.Problem("signature", dtype, d_in, d_out, off, ranks, scales.astype(np.float64) * rank,
                      scales, X, z((d_out, d_in)), A, B, dY)


def signature_expect(p):
    seg = np.repeat(np.arange(p.n_adapters), p.counts)
    Y = np.zeros((p.T, p.d_out))
    Y[:, :] = (seg + 1)[:, None]
    return Y


def test_segment_signature_exact():
    p = signature_problem([5, 1, 0, 9, 2])
    o = oracle.full(p)
    assert np.array_equal(o["Y"], signature_expect(p))
    for i in range(p.n_adapters):
        e = np.zeros_like(o["dB"][i]); e[0, 0] = (i + 1) * p.counts[i]
        assert np.array_equal(o["dB"][i], e)
        e = np.zeros_like(o["dA"][i]); e[0, 0] = (i + 1) * p.counts[i]
        assert np.array_equal(o["dA"][i], e)


def test_rows_api_matches_full_rows():
    p = small(61, "bf16")
    rows = np.array([0, 3, 6, 7, 18, 23], np.int64)
    fo, fg = oracle.forward(p), oracle.input_grad(p)
    so, sg = oracle.forward(p, rows=rows), oracle.input_grad(p, rows=rows)
    assert np.array_equal(so["Y"], fo["Y"][rows])
    assert np.array_equal(sg["dX"], fg["dX"][rows])
    with pytest.raises(ValueError):
        oracle.forward(p, rows=np.array([p.T], np.int64))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_column_subset_api_matches_full_columns(dtype):
    """The column-subset mode of the weight gradients (the full-size parity tests check sampled
    hidden columns of dA and rows of dB) gives exactly the full call's values on the requested
    columns, for every adapter including the empty one, and leaves every other column untouched.
    The requested columns come unsorted and include both ends."""
    p = small(62, dtype)
    full = oracle.weight_grads(p)
    cols_a = np.array([p.d_in - 1, 3, 0, 11], np.int64)
    cols_b = np.array([7, p.d_out - 1, 0, 2, 15], np.int64)
    sub = oracle.weight_grads(p, cols_a=cols_a, cols_b=cols_b)
    for i in range(p.n_adapters):
        assert np.array_equal(sub["dA"][i][:, cols_a], full["dA"][i][:, cols_a]), i
        assert np.array_equal(sub["dB"][i][cols_b], full["dB"][i][cols_b]), i
        rest_a = np.setdiff1d(np.arange(p.d_in), cols_a)
        rest_b = np.setdiff1d(np.arange(p.d_out), cols_b)
        assert not np.any(sub["dA"][i][:, rest_a]) and not np.any(sub["dB"][i][rest_b]), i
    # the subsets are not all zero: the comparison above has something to see
    assert any(np.any(sub["dA"][i][:, cols_a]) for i in range(p.n_adapters))
    assert any(np.any(sub["dB"][i][cols_b]) for i in range(p.n_adapters))


def test_row_and_adapter_subproblems_give_the_full_problems_rows():
    """The full-size parity tests run the oracle on small derived problems: the sampled rows
    (each adapter's sampled rows as its segment), and one adapter alone (optionally one output
    block's columns).  Both reproduce the full problem's values bit for bit."""
    from plora_testlib import adapter_subproblem, row_subproblem
    p = small(63, "bf16", counts=(9, 0, 14, 6))
    full = oracle.full(p)
    rows = np.array([0, 4, 8, 9, 15, 22, 23, 28], np.int64)
    sub = oracle.full(row_subproblem(p, rows))
    assert np.array_equal(sub["Y"], full["Y"][rows]) and np.array_equal(sub["dX"], full["dX"][rows])
    for i in range(p.n_adapters):
        alone = oracle.weight_grads(adapter_subproblem(p, i))
        assert np.array_equal(alone["dA"][0], full["dA"][i]) and np.array_equal(alone["dB"][0], full["dB"][i])
    # one output block: columns [8, 20) of W, dY, B; the weight gradients of that block alone
    cols = slice(8, 20)
    blk = dataclasses.replace(p, d_out=12, W=p.W[cols], dY=np.ascontiguousarray(p.dY[:, cols]),
                              B=[np.ascontiguousarray(b[cols]) for b in p.B])
    fb = oracle.weight_grads(blk)
    for i in range(p.n_adapters):
        alone = oracle.weight_grads(adapter_subproblem(p, i, out_cols=cols))
        assert np.array_equal(alone["dA"][0], fb["dA"][i]) and np.array_equal(alone["dB"][0], fb["dB"][i])


def test_threads_do_not_change_results():
    p = small(71, "bf16")
    a, b = oracle.full(p, nthreads=1), oracle.full(p, nthreads=4)
    assert np.array_equal(a["Y"], b["Y"]) and np.array_equal(a["dX"], b["dX"])
    for i in range(p.n_adapters):
        assert np.array_equal(a["dA"][i], b["dA"][i]) and np.array_equal(a["dB"][i], b["dB"][i])


def test_input_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e-3], np.float32)
    b = wl.f32_to_bf16_bits(x)
    back = wl.bf16_bits_to_f32(b)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2 ** -6
    assert back[3] == -2.5
    assert abs(back[4] - 3.0e-3) <= 3.0e-3 * 2 ** -8


# ----------------------------------------------------------------------------- AdamW step
ADAMW_CASES = [dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
               dict(lr=3e-2, beta1=0.8, beta2=0.99, eps=1e-6, weight_decay=0.0),
               dict(lr=5e-4, beta1=0.0, beta2=0.5, eps=1e-3, weight_decay=0.1)]


@pytest.mark.parametrize("hp", ADAMW_CASES)
def test_adamw_matches_torch_adamw_in_float64(hp):
    """Special case = library routine: torch.optim.AdamW on float64 tensors, several steps."""
    torch = pytest.importorskip("torch")
    g = np.random.default_rng(5)
    p0 = g.standard_normal((7, 13))
    tp = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=hp["lr"], betas=(hp["beta1"], hp["beta2"]), eps=hp["eps"],
                            weight_decay=hp["weight_decay"])
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t in range(1, 6):
        grad = g.standard_normal(p0.shape) * (0.1 * t)
        tp.grad = torch.tensor(grad, dtype=torch.float64)
        opt.step()
        p, m, v = oracle.adamw(p, m, v, grad, step=t, **hp)
        st = opt.state[tp]
        assert np.max(np.abs(p - tp.detach().numpy())) <= 1e-12 * max(1.0, np.max(np.abs(p)))
        assert np.max(np.abs(m - st["exp_avg"].numpy())) <= 1e-14
        assert np.max(np.abs(v - st["exp_avg_sq"].numpy())) <= 1e-14


def test_adamw_first_step_closed_form():
    """From zero moments, step 1: m_hat = g and sqrt(v_hat) = |g|, so p1 = p0 (1 - lr wd) - lr g / (|g| + eps)."""
    g = np.random.default_rng(6)
    p0, grad = g.standard_normal(50), g.standard_normal(50)
    lr, wd, eps = 0.01, 0.05, 1e-4
    p1, m1, v1 = oracle.adamw(p0, np.zeros(50), np.zeros(50), grad, lr=lr, weight_decay=wd, eps=eps, step=1)
    assert np.allclose(p1, p0 * (1 - lr * wd) - lr * grad / (np.abs(grad) + eps), rtol=1e-13, atol=1e-15)
    assert np.allclose(m1, 0.1 * grad, rtol=1e-15) and np.allclose(v1, 0.001 * grad * grad, rtol=1e-12)


def test_adamw_zero_gradient_is_pure_decay():
    p0 = np.random.default_rng(7).standard_normal(40)
    p1, m1, v1 = oracle.adamw(p0, np.zeros(40), np.zeros(40), np.zeros(40), lr=0.1, weight_decay=0.2, step=3)
    assert np.array_equal(p1, p0 * (1 - 0.1 * 0.2)) and not np.any(m1) and not np.any(v1)


def test_output_blocks_equal_one_block_diagonal_adapter():
    """Stacking P projections that read the same input (q|k|v), each adapter holding one rank-r pair
    per projection, is the same layer as one adapter of rank P r over the stacked W whose B is
    block-diagonal.  The oracle run on each projection's slice and on that block-diagonal embedding
    agree: Y and dX, the row blocks of dA and the diagonal blocks of dB (the reading that output
    blocks implement)."""
    widths, ranks, counts, d_in = [8, 4, 4], [2, 3], [5, 7], 12
    P, r = len(widths), np.asarray(ranks)
    base = wl.make_problem("blk", "fp32", d_in, sum(widths), r, counts, 2.0 * r, wl.init_small(d_in), 41)
    extra = [wl.make_problem(f"blk{b}", "fp32", d_in, 8, r, [1, 1], 2.0 * r, wl.init_small(d_in), 41 + b).A
             for b in range(1, P)]
    A_blocks = [base.A] + extra
    bounds = np.concatenate([[0], np.cumsum(widths)])
    A_bd, B_bd = [], []
    for i, ri in enumerate(ranks):
        A_bd.append(np.concatenate([A_blocks[b][i] for b in range(P)]))
        Bi = np.zeros((sum(widths), P * ri), dtype=base.B[i].dtype)
        for b in range(P):
            Bi[bounds[b]:bounds[b + 1], b * ri:(b + 1) * ri] = base.B[i][bounds[b]:bounds[b + 1]]
        B_bd.append(Bi)
    bd = dataclasses.replace(base, ranks=P * r, A=A_bd, B=B_bd)   # same scales s_i = alpha_i / r_i
    o_bd = oracle.full(bd)
    dX = 0.0
    for b in range(P):
        cols = slice(bounds[b], bounds[b + 1])
        pb = dataclasses.replace(base, d_out=widths[b], W=base.W[cols], dY=base.dY[:, cols], A=A_blocks[b],
                                 B=[x[cols] for x in base.B])
        o = oracle.full(pb)
        assert rel(o_bd["Y"][:, cols], o["Y"]) < 1e-12
        dX = dX + o["dX"]
        for i, ri in enumerate(ranks):
            assert rel(o_bd["dA"][i][b * ri:(b + 1) * ri], o["dA"][i]) < 1e-12
            assert rel(o_bd["dB"][i][cols, b * ri:(b + 1) * ri], o["dB"][i]) < 1e-12
    assert rel(o_bd["dX"], dX) < 1e-12
