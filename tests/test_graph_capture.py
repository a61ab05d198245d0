"""CUDA graph capture of the packed step: a captured forward + backward replays to the same bits as
the eager calls, an eager call between replays leaves the graph's schedules intact, and a call
captured without a reserved slot fails without enqueuing anything."""
import numpy as np
import pytest

import plora_workloads as wl
from plora_testlib import DeviceProblem

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402


def setup_step(seed=88):
    r = np.array([4, 16, 1, 64])
    p = wl.make_problem("cap", "bf16", 384, 520, r, [300, 129, 0, 700], 2.0 * r, wl.init_llm(384), seed)
    eng = pl.PackedLoRA(p.d_in, p.d_out, "bf16", max_adapters=4, max_rank=64, max_tokens=p.T)
    d = DeviceProblem(p)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    out = dict(Y=torch.empty((p.T, p.d_out), **bf), dX=torch.empty((p.T, p.d_in), **bf),
               dA=[torch.empty(a.shape, dtype=torch.float32, device="cuda") for a in d.A],
               dB=[torch.empty(b.shape, dtype=torch.float32, device="cuda") for b in d.B])
    tf = eng.table(p.scales, d.A, d.B)
    tb = eng.table(p.scales, d.A, d.B, out["dA"], out["dB"])
    saved = torch.empty(eng.saved_bytes(p.off, tf), dtype=torch.uint8, device="cuda")

    def step(stream):
        pl.plora_forward(eng.h, d.X.data_ptr(), d.W.data_ptr(), out["Y"].data_ptr(), p.n_adapters, p.off, tf,
                         saved.data_ptr(), stream)
        pl.plora_backward(eng.h, d.X.data_ptr(), d.W.data_ptr(), d.dY.data_ptr(), out["dX"].data_ptr(),
                          p.n_adapters, p.off, tb, saved.data_ptr(), stream)

    tensors = [out["Y"], out["dX"]] + out["dA"] + out["dB"]
    return eng, step, tensors


def test_captured_step_replays_bit_exactly():
    eng, step, tensors = setup_step()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step(s.cuda_stream)
    torch.cuda.synchronize()
    ref = [t.clone() for t in tensors]
    pl.plora_capture_reserve(eng.h, 2)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s.cuda_stream)
    for rnd in range(2):
        for t in tensors:
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(tensors, ref):
            assert torch.equal(a, b), rnd
        # an eager call (it uses the handle's ring) between replays
        step(torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
    assert pl.plora_check(eng.h, 0) == pl.PLORA_OK
    del g
    pl.plora_capture_release(eng.h)
    eng.close()


def test_capture_without_reserved_slot_fails_cleanly():
    eng, step, tensors = setup_step(89)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step(s.cuda_stream)          # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with pytest.raises(pl.PloraError) as err:
        with torch.cuda.graph(g, stream=s):
            tensors[0].add_(0)       # keeps the graph non-empty
            step(s.cuda_stream)
    assert err.value.status == pl.PLORA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    eng.close()
