"""Failure detection without a GPU fault: a bounded device wait that nothing satisfies runs
out, the kernel reports PLORA_ERR_TIMEOUT through the handle's error flag and returns, and the
context stays usable for the next call."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import packed_lora_fine_b200 as pl  # noqa: E402
import plora_workloads as wl  # noqa: E402
from plora_testlib import run  # noqa: E402


def test_bounded_wait_reports_timeout_and_context_survives():
    eng = pl.PackedLoRA(64, 64, "bf16", max_adapters=1, max_rank=8, max_tokens=16)
    assert pl.plora_check(eng.h, 0) == pl.PLORA_OK
    assert pl.plora_debug_timeout_probe(eng.h, 50_000_000, 0) == pl.PLORA_OK     # 50 ms limit
    assert pl.plora_check(eng.h, 0) == pl.PLORA_ERR_TIMEOUT
    assert "ran out of time" in pl.plora_last_error(eng.h)
    assert pl.plora_check(eng.h, 0) == pl.PLORA_OK                              # flag cleared
    assert pl.plora_debug_timeout_probe(eng.h, 10, 0) == pl.PLORA_ERR_INVALID_ARG
    eng.close()
    # the context is still usable: a normal packed step runs and passes its own check
    r = np.array([4, 8])
    p = wl.make_problem("after", "bf16", 64, 64, r, [10, 20], 2.0 * r, wl.init_llm(64), 3)
    run(p)
