"""Host-side tests of the C ABI: it loads, exports what include/plora.h declares,
rejects bad configurations and tables, and its schedule covers every token of
every adapter exactly once.  No kernel is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

import packed_lora_fine_b200 as pl
from packed_lora_fine_b200 import build as plbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    plbuild.build()
    pl.load()


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "plora.h")).read()
    return sorted(set(re.findall(r"PLORA_API\s+[\w\s\*]+?\b(plora_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 11
    lib = ctypes.CDLL(pl.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(pl.EXPORTED)


def test_debug_build_loads_and_exports_the_same_symbols():
    """The PLORA_DEBUG build (device-side bounds checks) is a drop-in for the release library: it loads
    without a GPU, exports every declared function and says which build it is."""
    from packed_lora_fine_b200 import build as plbuild
    rel = ctypes.CDLL(plbuild.LIB)
    dbg = ctypes.CDLL(plbuild.DEBUG_LIB)
    for n in declared_functions():
        assert hasattr(dbg, n), n
    rel.plora_debug_build.restype = dbg.plora_debug_build.restype = ctypes.c_int32
    assert rel.plora_debug_build() == 0 and dbg.plora_debug_build() == 1
    dbg.plora_status_string.restype = ctypes.c_char_p
    assert dbg.plora_status_string(6) == b"PLORA_ERR_BOUNDS"


def test_status_strings_and_version():
    for code, name in [(0, "PLORA_OK"), (1, "PLORA_ERR_INVALID_ARG"), (2, "PLORA_ERR_UNSUPPORTED"),
                       (3, "PLORA_ERR_OOM"), (4, "PLORA_ERR_CUDA"), (5, "PLORA_ERR_TIMEOUT"),
                       (6, "PLORA_ERR_BOUNDS")]:
        assert pl.status_string(code) == name
    assert pl.plora_version() >= 100


def cfg(d_in=64, d_out=64, dtype=pl.PLORA_BF16, max_adapters=8, max_rank=64, max_tokens=4096, flags=0):
    return pl.plora_config(d_in, d_out, dtype, max_adapters, max_rank, flags, max_tokens)


@pytest.mark.parametrize("c, want", [
    (cfg(d_in=60), pl.PLORA_ERR_UNSUPPORTED),
    (cfg(d_out=4), pl.PLORA_ERR_UNSUPPORTED),
    (cfg(d_in=1 << 17), pl.PLORA_ERR_UNSUPPORTED),
    (cfg(dtype=7), pl.PLORA_ERR_UNSUPPORTED),
    (cfg(max_adapters=0), pl.PLORA_ERR_INVALID_ARG),
    (cfg(max_rank=257), pl.PLORA_ERR_INVALID_ARG),
    (cfg(max_rank=0), pl.PLORA_ERR_INVALID_ARG),
    (cfg(max_tokens=0), pl.PLORA_ERR_INVALID_ARG),
    (cfg(flags=8), pl.PLORA_ERR_INVALID_ARG),
])
def test_create_rejects_bad_config(c, want):
    s, h = pl.plora_create_status(c)
    assert s == want and not h


def blocked_cfg(widths, d_out=None, **kw):
    c = cfg(d_out=d_out if d_out is not None else sum(widths), **kw)
    end = 0
    c.n_out_blocks = len(widths)
    for b, w in enumerate(widths[:pl.PLORA_MAX_OUT_BLOCKS]):
        end += w
        c.out_block_end[b] = end
    return c


@pytest.mark.parametrize("c, want", [
    (blocked_cfg([200, 312]), pl.PLORA_ERR_INVALID_ARG),                 # a block end not a multiple of 256
    (blocked_cfg([256, 512], d_out=512), pl.PLORA_ERR_INVALID_ARG),      # ends past d_out
    (blocked_cfg([256, 256, 256], max_rank=96), pl.PLORA_ERR_INVALID_ARG),  # 3 x 96 padded ranks > 256
    (blocked_cfg([256] * 9), pl.PLORA_ERR_INVALID_ARG),                  # more than 8 blocks
    (blocked_cfg([256, 256], dtype=pl.PLORA_FP32), pl.PLORA_ERR_UNSUPPORTED),
    (blocked_cfg([256, 256], flags=pl.PLORA_FLAG_SIMT), pl.PLORA_ERR_UNSUPPORTED),
    (blocked_cfg([256, 256], flags=pl.PLORA_FLAG_UNFUSED), pl.PLORA_ERR_UNSUPPORTED),
    (blocked_cfg([256, 256], flags=pl.PLORA_FLAG_BASE_PAIR), pl.PLORA_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_output_blocks(c, want):
    s, h = pl.plora_create_status(c)
    assert s == want and not h


def test_output_blocks_widen_the_padded_rank():
    # rank 24 per block: each block's columns of H' are 32 wide (24 rounded up to 16), so three
    # blocks need 96 columns and the saved / G pitch RP rounds that up to 128
    off = np.array([0, 100], np.int64)
    c1, c3 = cfg(d_out=768, max_rank=64), blocked_cfg([256, 256, 256], max_rank=64)
    for c, want in ((c1, 64), (c3, 128)):
        s, v = pl.plora_debug_schedule(c, 1, off, fake_table([24]), False, 3)
        assert s == pl.PLORA_OK and v[0] == want
    s, v = pl.plora_debug_schedule(c3, 1, off, fake_table([24]), False, 2)
    assert s == pl.PLORA_OK and list(v[3:5]) == [96, 128]        # H/G width 3 x 32, rounded to 64
    s, v = pl.plora_debug_schedule(c1, 1, off, fake_table([24]), False, 2)
    assert s == pl.PLORA_OK and list(v[3:5]) == [32, 64]


def test_create_without_gpu_fails_loudly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    s, h = pl.plora_create_status(cfg())
    assert s == pl.PLORA_ERR_CUDA and not h


def test_null_handle_calls_are_rejected():
    import ctypes
    lib = pl.load()
    out = (ctypes.c_int32 * 3)()
    cnt = ctypes.c_int32(-1)
    assert lib.plora_device_info(None, ctypes.cast(out, ctypes.c_void_p), 3, ctypes.byref(cnt)) == pl.PLORA_ERR_INVALID_ARG
    assert cnt.value == -1
    assert lib.plora_profile_enable(None, 1) == pl.PLORA_ERR_INVALID_ARG
    assert lib.plora_capture_reserve(None, 1) == pl.PLORA_ERR_INVALID_ARG
    assert lib.plora_capture_release(None) == pl.PLORA_ERR_INVALID_ARG
    assert lib.plora_check(None, None) == pl.PLORA_ERR_INVALID_ARG


def fake_table(ranks, aligned=True, grads=True):
    base = 0x7f0000000000
    n = len(ranks)
    A = [base + 4096 * (4 * i) for i in range(n)]
    B = [base + 4096 * (4 * i + 1) for i in range(n)]
    dA = [base + 4096 * (4 * i + 2) for i in range(n)] if grads else None
    dB = [base + 4096 * (4 * i + 3) for i in range(n)] if grads else None
    if not aligned:
        A[0] += 8
    return pl.make_table(ranks, [2.0] * n, A, B, dA, dB)


def schedule(c, off, ranks, which, grads=False, tab=None):
    s, v = pl.plora_debug_schedule(c, len(off) - 1, off, tab if tab is not None else fake_table(ranks), grads,
                                   which)
    assert s == pl.PLORA_OK, pl.status_string(s)
    return v


@pytest.mark.parametrize("off, ranks, want", [
    ([1, 5], [4], pl.PLORA_ERR_INVALID_ARG),              # off[0] != 0
    ([0, 9, 5], [4, 4], pl.PLORA_ERR_INVALID_ARG),        # decreasing
    ([0, 5000], [4], pl.PLORA_ERR_INVALID_ARG),           # > max_tokens
    ([0, 5], [0], pl.PLORA_ERR_INVALID_ARG),              # rank 0
    ([0, 5], [65], pl.PLORA_ERR_INVALID_ARG),             # rank > max_rank
    ([0] * 10, [4] * 9, pl.PLORA_ERR_INVALID_ARG),        # n > max_adapters
])
def test_bad_tables_rejected(off, ranks, want):
    s, _ = pl.plora_debug_schedule(cfg(), len(off) - 1, off, fake_table(ranks), False, 0)
    assert s == want


def test_null_and_misaligned_pointers_rejected():
    c = cfg()
    s, _ = pl.plora_debug_schedule(c, 1, [0, 5], fake_table([4], aligned=False), False, 0)
    assert s == pl.PLORA_ERR_INVALID_ARG
    s, _ = pl.plora_debug_schedule(c, 1, [0, 5], fake_table([4], grads=False), True, 0)
    assert s == pl.PLORA_ERR_INVALID_ARG            # backward needs dA, dB
    s, _ = pl.plora_debug_schedule(c, 1, [0, 5], fake_table([4], grads=False), False, 0)
    assert s == pl.PLORA_OK                         # forward ignores them
    t = fake_table([4])
    t[0].scale = float("nan")
    s, _ = pl.plora_debug_schedule(c, 1, [0, 5], t, False, 0)
    assert s == pl.PLORA_ERR_INVALID_ARG


def random_segments(seed, n, lo, hi, zero_frac=0.2):
    g = np.random.default_rng(seed)
    counts = g.integers(lo, hi + 1, size=n)
    counts[g.random(n) < zero_frac] = 0
    off = np.zeros(n + 1, np.int64)
    off[1:] = np.cumsum(counts)
    ranks = g.choice([1, 3, 8, 16, 17, 64, 100, 256], size=n)
    return off, ranks


@pytest.mark.parametrize("seed", range(6))
def test_token_tiles_cover_every_row_once(seed):
    off, ranks = random_segments(seed, 40, 0, 700)
    c = cfg(max_adapters=64, max_rank=256, max_tokens=int(off[-1]) + 1)
    tiles = schedule(c, off, ranks, 0).reshape(-1, 4)
    ad = schedule(c, off, ranks, 2).reshape(-1, 5)
    RP, h_rows = schedule(c, off, ranks, 3)
    owner = np.full(int(off[-1]), -1)
    for a, rows, x, hrow in tiles:
        assert 1 <= rows <= 128
        assert np.all(owner[x:x + rows] == -1)
        owner[x:x + rows] = a
        assert off[a] <= x and x + rows <= off[a + 1]
        assert hrow - ad[a, 2] == x - off[a]               # same offset inside the adapter's block
        assert (x - off[a]) % 128 == 0
    assert np.array_equal(owner, np.repeat(np.arange(len(ranks)), np.diff(off)))   # bit-exact map
    # H/G blocks: every adapter with tokens owns 256 zero rows, its rows rounded up to 128 and
    # 256 zero rows, packed in order; the first H/G row of its data follows the leading pad.
    n = np.diff(off)
    blocks = np.where(n > 0, ((n + 127) // 128) * 128 + 512, 0)
    starts = np.concatenate([[0], np.cumsum(blocks)[:-1]])
    assert np.array_equal(ad[n > 0, 2], starts[n > 0] + 256)
    assert h_rows == blocks.sum()
    # adapters overlapping each global 256-row tile of the base GEMMs
    mto = schedule(c, off, ranks, 4)
    mtl = schedule(c, off, ranks, 5)
    T = int(off[-1])
    assert len(mto) == (T + 255) // 256 + 1 and mto[0] == 0 and mto[-1] == len(mtl)
    for mb in range((T + 255) // 256):
        m0, m1 = 256 * mb, min(T, 256 * mb + 256)
        want = [j for j in range(len(ranks)) if n[j] > 0 and off[j] < m1 and off[j + 1] > m0]
        assert list(mtl[mto[mb]:mto[mb + 1]]) == want
    assert RP == ((max(ranks) + 63) // 64) * 64
    assert np.array_equal(ad[:, 3], ((ranks + 15) // 16) * 16)
    assert np.array_equal(ad[:, 4], ((ranks + 63) // 64) * 64)


@pytest.mark.parametrize("seed", range(4))
def test_weight_grad_splits_cover_tokens_and_depend_only_on_count(seed):
    off, ranks = random_segments(seed, 24, 0, 40000)
    c = cfg(max_adapters=64, max_rank=256, max_tokens=int(off[-1]) + 1)
    red = schedule(c, off, ranks, 1, grads=True).reshape(-1, 8)
    ks = red[:, 3]
    assert np.all(ks[:-1] >= ks[1:])                       # longest first
    n = np.diff(off)
    for i in range(len(ranks)):
        e = red[red[:, 0] == i]
        if n[i] == 0:
            assert len(e) == 0
            continue
        e = e[np.argsort(e[:, 4])]
        S = (n[i] + 16383) // 16384
        assert len(e) == S and np.all(e[:, 5] == S) and np.array_equal(e[:, 4], np.arange(S))
        assert np.array_equal(e[:, 1], off[i] + 16384 * np.arange(S))
        lens = np.minimum(16384, n[i] - 16384 * np.arange(S))
        assert np.array_equal(e[:, 3], (lens + 63) // 64)
        assert (S == 1) == (e[0, 6] == -1)
        # the same adapter alone gets the same splits
        alone = schedule(c, [0, n[i]], [ranks[i]], 1, grads=True).reshape(-1, 8)
        alone = alone[np.argsort(alone[:, 4])]
        assert np.array_equal(alone[:, 3:6], e[:, 3:6])
        assert np.array_equal(alone[:, 1], e[:, 1] - off[i])


def test_empty_call_is_valid():
    v = schedule(cfg(), [0], [], 0)
    assert len(v) == 0
    v = schedule(cfg(), [0, 0, 0], [3, 5], 1, grads=True)
    assert len(v) == 0


def test_make_config_writes_cumulative_block_ends():
    c = pl.make_config(4096, 6144, pl.PLORA_BF16, 16, 64, 1 << 16, 0, out_blocks=[4096, 1024, 1024])
    assert c.n_out_blocks == 3 and list(c.out_block_end[:3]) == [4096, 5120, 6144] and c.reserved == 0
    assert pl.make_config(64, 64, pl.PLORA_BF16, 1, 8, 8, 0, out_blocks=[64]).n_out_blocks == 0
    off = np.array([0, 10], np.int64)
    s, v = pl.plora_debug_schedule(c, 1, off, fake_table([16]), False, 3)
    assert s == pl.PLORA_OK and v[0] == 3 * 16 + 16        # RP: 3 blocks x 16, rounded up to 64


def test_layer_create_refuses_bad_layers_without_a_device():
    """plora_layer_create checks the projection count and each configuration's path before it creates
    any handle, so these refusals need no GPU."""
    lib = pl.load()
    L = ctypes.c_void_p()
    cfg = pl.make_config(256, 256, pl.PLORA_BF16, 4, 16, 1024)
    cfgs = (pl.plora_config * 9)(*([cfg] * 9))
    assert lib.plora_layer_create(ctypes.byref(L), 0, cfgs) == pl.PLORA_ERR_INVALID_ARG
    assert lib.plora_layer_create(ctypes.byref(L), 9, cfgs) == pl.PLORA_ERR_INVALID_ARG
    assert lib.plora_layer_create(ctypes.byref(L), 2, None) == pl.PLORA_ERR_INVALID_ARG
    for flags in (pl.PLORA_FLAG_SIMT, pl.PLORA_FLAG_UNFUSED, pl.PLORA_FLAG_BASE_PAIR):
        bad = (pl.plora_config * 2)(cfg, pl.make_config(256, 256, pl.PLORA_BF16, 4, 16, 1024, flags))
        assert lib.plora_layer_create(ctypes.byref(L), 2, bad) == pl.PLORA_ERR_UNSUPPORTED
    f32 = (pl.plora_config * 1)(pl.make_config(256, 256, pl.PLORA_FP32, 4, 16, 1024))
    assert lib.plora_layer_create(ctypes.byref(L), 1, f32) == pl.PLORA_ERR_UNSUPPORTED
    assert L.value is None
    assert lib.plora_layer_destroy(None) == pl.PLORA_OK
