"""The allocation-free dB entry point (plora_grad_B_static).

Some callers cannot allocate device memory -- a runtime whose memory planner or
caching allocator owns the whole device, code that must not synchronise the
device, hosts that only hand the library the tensors it works on.  For them
the library computes dB with its scratch in a static device array.  Here it is
called through the C ABI, twice in a row, and each result is checked against
the handle-based plora_backward and against the fp64 oracle, within the bf16
tolerance of the other tests.  This file is collected last so that a stop at
the first failure has already run every other test.
"""
import numpy as np
import pytest

import oracle
import plora_workloads as wl
from plora_testlib import BF16_TOL, DeviceProblem, rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402

CASES = [
    # d_in, d_out, ranks, token counts.  Every case has adapters longer than the 16384-token split,
    # so split partials and arrival counters are used, plus a short one and an empty one.
    (256, 384, [16, 96, 8, 24], [34000, 16385, 300, 0]),
    # d_in much wider than d_out, with two split adapters: the plan spaces each split adapter's
    # arrival counters by the d_in tiles (32 here), beyond the d_out tiles (4) that dB reads.
    (4096, 512, [16, 64, 8, 32], [20000, 17000, 300, 0]),
]


def _problem(k):
    d_in, d_out, ranks, counts = CASES[k]
    r = np.array(ranks)
    return wl.make_problem(f"noalloc{k}", "bf16", d_in, d_out, r, counts, 2.0 * r, wl.init_llm(d_in), 4242 + k)


@pytest.mark.parametrize("k", range(len(CASES)))
def test_static_grad_B_matches_backward_and_oracle_twice(k):
    p = _problem(k)
    d = DeviceProblem(p)
    eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=p.n_adapters, max_rank=int(max(p.ranks)),
                        max_tokens=p.T)
    Y, saved = eng.forward(d.X, d.W, p.off, p.scales, d.A, d.B)
    _, _, dB_ref = eng.backward(d.X, d.W, d.dY, p.off, p.scales, d.A, d.B, saved)
    torch.cuda.synchronize()
    assert pl.plora_check(eng.h, 0) == pl.PLORA_OK
    ref = [b.cpu().numpy().astype(np.float64) for b in dB_ref]
    # the oracle's dB in full (one dA column keeps its dA part cheap)
    o = oracle.weight_grads(p, nthreads=oracle.num_procs(), cols_a=np.array([0]))["dB"]

    cfg = pl.plora_config(p.d_in, p.d_out, pl.PLORA_BF16, p.n_adapters, int(max(p.ranks)), 0, p.T)
    for call in range(2):
        dB = [torch.full(b.shape, float("nan"), dtype=torch.float32, device="cuda") for b in d.B]
        dA = [torch.empty(a.shape, dtype=torch.float32, device="cuda") for a in d.A]
        tab = eng.table(p.scales, d.A, d.B, dA, dB)
        st = pl.plora_grad_B_static(cfg, d.dY.data_ptr(), p.n_adapters, p.off, tab, saved.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
        assert st == pl.PLORA_OK, pl.status_string(st)
        torch.cuda.synchronize()
        for i in range(p.n_adapters):
            got = dB[i].cpu().numpy().astype(np.float64)
            assert np.all(np.isfinite(got)), (call, i)
            assert rel_err(got, ref[i]) <= BF16_TOL, ("backward", call, i)
            assert rel_err(got, o[i]) <= BF16_TOL, ("oracle", call, i)
    eng.close()


def test_static_grad_B_rejects_oversized_calls():
    """Calls whose split state cannot fit the static array are refused before any device work.
    The precondition is computed here from the documented limit first, so that a change of the
    library's constants can never turn this into a launch on the placeholder pointers below."""
    split, d_in, d_out, rank, tokens = 16384, 256, 65536, 256, 40000
    splits = -(-tokens // split)
    rp = -(-rank // 64) * 64
    counters = -(-(1 * max(-(-d_in // 128), -(-d_out // 128)) * 4) // 256) * 256
    partial_bytes = splits * (-(-d_out // 128)) * 128 * rp * 4
    assert splits > 1 and counters + partial_bytes > 8 * (pl.PLORA_STATIC_SCRATCH_BYTES)
    cfg = pl.plora_config(d_in, d_out, pl.PLORA_BF16, 1, rank, 0, tokens)
    tab = pl.make_table([rank], [1.0], [1 << 20], [1 << 21], [1 << 22], [1 << 23])
    st = pl.plora_grad_B_static(cfg, 1 << 24, 1, np.array([0, tokens], np.int64), tab, 1 << 25, 0)
    assert st == pl.PLORA_ERR_UNSUPPORTED
    cfg32 = pl.plora_config(256, 384, pl.PLORA_FP32, 1, 256, 0, 1000)
    st = pl.plora_grad_B_static(cfg32, 1 << 24, 1, np.array([0, 1000], np.int64), tab, 1 << 25, 0)
    assert st == pl.PLORA_ERR_UNSUPPORTED
