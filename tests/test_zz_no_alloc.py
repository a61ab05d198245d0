"""The allocation-free dB entry point (plora_grad_B_static).

Some callers cannot allocate device memory -- a runtime whose memory planner or
caching allocator owns the whole device, code that must not synchronise the
device, hosts that only hand the library the tensors it works on.  For them
the library computes dB with its scratch in a static device array.  Here it is
called through the C ABI, twice in a row, and each result is checked against
the handle-based plora_backward within the bf16 tolerance of the other tests.
This file is collected last so that a stop at the first failure has already
run every other test.
"""
import numpy as np
import pytest

import plora_workloads as wl
from plora_testlib import BF16_TOL, DeviceProblem, rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402


def _problem():
    # Two adapters longer than the 16384-token split (so split partials and arrival
    # counters are used), a short one and an empty one.
    r = np.array([16, 96, 8, 24])
    return wl.make_problem("noalloc", "bf16", 256, 384, r, [34000, 16385, 300, 0], 2.0 * r,
                           wl.init_llm(256), 4242)


def test_static_grad_B_matches_backward_twice():
    p = _problem()
    d = DeviceProblem(p)
    eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=p.n_adapters, max_rank=int(max(p.ranks)),
                        max_tokens=p.T)
    Y, saved = eng.forward(d.X, d.W, p.off, p.scales, d.A, d.B)
    _, _, dB_ref = eng.backward(d.X, d.W, d.dY, p.off, p.scales, d.A, d.B, saved)
    torch.cuda.synchronize()
    assert pl.plora_check(eng.h, 0) == pl.PLORA_OK
    ref = [b.cpu().numpy().astype(np.float64) for b in dB_ref]

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
            assert rel_err(got, ref[i]) <= BF16_TOL, (call, i)
    eng.close()


def test_static_grad_B_rejects_oversized_calls():
    """Calls whose split partials cannot fit the static array are refused before any device work.
    The precondition is computed here from the documented limit first, so that a change of the
    library's constants can never turn this into a launch on the placeholder pointers below."""
    split, d_out, rank, tokens = 16384, 65536, 256, 40000
    splits = -(-tokens // split)
    partial_bytes = splits * (-(-d_out // 128)) * (4 + 128 * rank * 4)
    assert splits > 1 and partial_bytes > 8 * (pl.PLORA_STATIC_SCRATCH_BYTES)
    cfg = pl.plora_config(256, d_out, pl.PLORA_BF16, 1, rank, 0, tokens)
    tab = pl.make_table([rank], [1.0], [1 << 20], [1 << 21], [1 << 22], [1 << 23])
    st = pl.plora_grad_B_static(cfg, 1 << 24, 1, np.array([0, tokens], np.int64), tab, 1 << 25, 0)
    assert st == pl.PLORA_ERR_UNSUPPORTED
    cfg32 = pl.plora_config(256, 384, pl.PLORA_FP32, 1, 256, 0, 1000)
    st = pl.plora_grad_B_static(cfg32, 1 << 24, 1, np.array([0, 1000], np.int64), tab, 1 << 25, 0)
    assert st == pl.PLORA_ERR_UNSUPPORTED
