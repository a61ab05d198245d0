"""The PLORA_DEBUG build (libplora_debug.so): every kernel checks each index it forms from a call's
schedule against the extent of the buffer it addresses, records PLORA_ERR_BOUNDS on a failure and
skips the access, so a wrong schedule shows up as an error status, not as a fault.  This test runs the
small-mix parity tests (every path: 1-SM and SM-pair tensor cores, unfused, SIMT bf16, fp32), the
weight-gradient split path, many adapters in one tile, narrow last n-tiles over many tiles, row counts
at the base tile's edges, output blocks, layer calls and the allocation-free dB
entry point once more, in a child process that loads the debug build: on valid inputs no check
fires (each run's plora_check returns PLORA_OK) and every result still matches the oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suite_under_the_debug_build():
    from packed_lora_fine_b200 import build as plbuild
    assert os.path.exists(plbuild.DEBUG_LIB), "libplora_debug.so is not built"
    env = dict(os.environ, PLORA_LIBRARY=plbuild.DEBUG_LIB)
    which = subprocess.run([sys.executable, "-c", "import packed_lora_fine_b200 as pl; "
                            "print(pl.load().plora_debug_build())"], cwd=ROOT, env=env, capture_output=True,
                           text=True, timeout=300)
    assert which.returncode == 0 and which.stdout.strip() == "1", which.stderr
    sel = ("small_mixes or weight_grad_split or many_adapters_in_one_tile or lora_delta_with_zero_base or "
           "narrow_last_n_tile or tile_edges or output_blocks_match_each_projection_alone or static_grad_B or "
           "layer_call")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider", "-k", sel,
                        "tests/test_parity.py", "tests/test_out_blocks.py", "tests/test_layer.py",
                        "tests/test_zz_no_alloc.py"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = "\n".join(r.stdout.splitlines()[-15:])
    assert r.returncode == 0, tail
    assert " passed" in tail and "failed" not in tail, tail
