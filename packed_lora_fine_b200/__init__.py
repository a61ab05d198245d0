"""Packed LoRA fine-tuning for NVIDIA B200 (sm_100a): Python binding of the C ABI.

This module only marshals arguments into ``libplora.so`` (built from
``csrc/`` by ``packed_lora_fine_b200.build``); every step of the computation
runs in the library's CUDA kernels.  The functions keep the C names of
``include/plora.h``: ``plora_create``, ``plora_forward``, ``plora_backward``,
``plora_check``, ``plora_saved_bytes``, ``plora_debug_unpack_saved``,
``plora_destroy``.  Tensors are passed as device pointers (ints); PyTorch is
only a convenient owner of device memory and streams.

There is no fallback: if the library is missing, importing the binding
raises ``ImportError``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# PLORA_LIBRARY may name another build of the library (the PLORA_DEBUG build with device-side bounds
# checks, libplora_debug.so); a missing file still raises ImportError.
LIB_PATH = os.environ.get("PLORA_LIBRARY") or os.path.join(_HERE, "libplora.so")

PLORA_OK = 0
PLORA_ERR_INVALID_ARG = 1
PLORA_ERR_UNSUPPORTED = 2
PLORA_ERR_OOM = 3
PLORA_ERR_CUDA = 4
PLORA_ERR_TIMEOUT = 5
PLORA_ERR_BOUNDS = 6
PLORA_BF16 = 0
PLORA_FP32 = 1
PLORA_FLAG_SIMT = 1
PLORA_FLAG_UNFUSED = 2
PLORA_FLAG_BASE_PAIR = 4
PLORA_MAX_RANK = 256
PLORA_MAX_ADAPTERS = 4096
PLORA_MAX_OUT_BLOCKS = 8
PLORA_STATIC_SCRATCH_BYTES = 16 << 20

EXPORTED = ("plora_create", "plora_destroy", "plora_saved_bytes", "plora_forward", "plora_backward",
            "plora_check", "plora_status_string", "plora_last_error", "plora_debug_unpack_saved",
            "plora_version", "plora_debug_schedule", "plora_profile_enable", "plora_profile_read",
            "plora_grad_B_static", "plora_adamw_step", "plora_debug_timeout_probe", "plora_device_info",
            "plora_capture_reserve", "plora_capture_release", "plora_partition", "plora_debug_build",
            "plora_layer_create", "plora_layer_destroy", "plora_layer_handle", "plora_layer_saved_bytes",
            "plora_layer_forward", "plora_layer_backward", "plora_layer_check", "plora_layer_last_error")


class plora_config(ctypes.Structure):
    _fields_ = [("d_in", ctypes.c_int64), ("d_out", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("max_adapters", ctypes.c_int32), ("max_rank", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("max_tokens", ctypes.c_int64), ("n_out_blocks", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("out_block_end", ctypes.c_int64 * PLORA_MAX_OUT_BLOCKS)]


def make_config(d_in, d_out, dtype, max_adapters, max_rank, max_tokens, flags=0, out_blocks=None):
    """plora_config; out_blocks: the output widths of P >= 2 shared-input projections stacked in W
    (their sum is d_out), or None for one projection."""
    cfg = plora_config(d_in, d_out, dtype, max_adapters, max_rank, flags, max_tokens)
    if out_blocks is not None and len(out_blocks) > 1:
        cfg.n_out_blocks = len(out_blocks)
        end = 0
        for b, w in enumerate(out_blocks):
            end += int(w)
            cfg.out_block_end[b] = end
    return cfg


class plora_adapter(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32), ("scale", ctypes.c_float), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("dA", ctypes.c_void_p), ("dB", ctypes.c_void_p)]


class plora_adamw_state(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int32),
                ("A_master", ctypes.c_void_p), ("B_master", ctypes.c_void_p), ("mA", ctypes.c_void_p),
                ("vA", ctypes.c_void_p), ("mB", ctypes.c_void_p), ("vB", ctypes.c_void_p)]


class PloraError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{status_string(status)}: {message}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Load libplora.so (raises ImportError if it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libplora.so not built at {path}; run packed_lora_fine_b200.build.build()")
    lib = ctypes.CDLL(path)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    H = ctypes.c_void_p
    lib.plora_create.argtypes = [ctypes.POINTER(H), ctypes.POINTER(plora_config)]
    lib.plora_destroy.argtypes = [H]
    lib.plora_saved_bytes.argtypes = [H, I32, P, P, ctypes.POINTER(ctypes.c_size_t)]
    lib.plora_forward.argtypes = [H, P, P, P, I32, P, P, P, P]
    lib.plora_backward.argtypes = [H, P, P, P, P, I32, P, P, P, P]
    lib.plora_check.argtypes = [H, P]
    lib.plora_status_string.argtypes = [ctypes.c_int]
    lib.plora_status_string.restype = ctypes.c_char_p
    lib.plora_last_error.argtypes = [H]
    lib.plora_last_error.restype = ctypes.c_char_p
    lib.plora_debug_unpack_saved.argtypes = [H, I32, P, P, P, I32, P, P]
    lib.plora_debug_schedule.argtypes = [ctypes.POINTER(plora_config), I32, P, P, I32, I32, P, I64,
                                         ctypes.POINTER(ctypes.c_int64)]
    lib.plora_debug_schedule.restype = ctypes.c_int
    lib.plora_profile_enable.argtypes = [H, I32]
    lib.plora_profile_enable.restype = ctypes.c_int
    lib.plora_profile_read.argtypes = [H, I32, ctypes.POINTER(I32), P, P, P]
    lib.plora_profile_read.restype = ctypes.c_int
    lib.plora_capture_reserve.argtypes = [H, I32]
    lib.plora_capture_reserve.restype = ctypes.c_int
    lib.plora_capture_release.argtypes = [H]
    lib.plora_capture_release.restype = ctypes.c_int
    lib.plora_device_info.argtypes = [H, P, I32, ctypes.POINTER(I32)]
    lib.plora_device_info.restype = ctypes.c_int
    lib.plora_debug_timeout_probe.argtypes = [H, I64, P]
    lib.plora_debug_timeout_probe.restype = ctypes.c_int
    lib.plora_adamw_step.argtypes = [H, I32, P, P, P]
    lib.plora_adamw_step.restype = ctypes.c_int
    lib.plora_grad_B_static.argtypes = [ctypes.POINTER(plora_config), P, I32, P, P, P, P]
    lib.plora_grad_B_static.restype = ctypes.c_int
    lib.plora_version.argtypes = []
    lib.plora_version.restype = ctypes.c_int32
    lib.plora_debug_build.argtypes = []
    lib.plora_debug_build.restype = ctypes.c_int32
    lib.plora_layer_create.argtypes = [ctypes.POINTER(H), I32, P]
    lib.plora_layer_destroy.argtypes = [H]
    lib.plora_layer_handle.argtypes = [H, I32, ctypes.POINTER(H)]
    lib.plora_layer_saved_bytes.argtypes = [H, I32, P, P, P]
    lib.plora_layer_forward.argtypes = [H, I32, P, P, P]
    lib.plora_layer_backward.argtypes = [H, I32, P, P, P]
    lib.plora_layer_check.argtypes = [H, P]
    lib.plora_layer_last_error.argtypes = [H]
    lib.plora_layer_last_error.restype = ctypes.c_char_p
    for fn in ("plora_layer_create", "plora_layer_destroy", "plora_layer_handle", "plora_layer_saved_bytes",
               "plora_layer_forward", "plora_layer_backward", "plora_layer_check"):
        getattr(lib, fn).restype = ctypes.c_int
    lib.plora_partition.argtypes = [I32, P, P, I64, I64, ctypes.c_double, ctypes.c_double, I32, P, P]
    lib.plora_partition.restype = ctypes.c_int
    for fn in ("plora_create", "plora_destroy", "plora_saved_bytes", "plora_forward", "plora_backward",
               "plora_check", "plora_debug_unpack_saved"):
        getattr(lib, fn).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(s: int) -> str:
    return load().plora_status_string(int(s)).decode()


def _raise(h, s: int):
    if s != PLORA_OK:
        msg = load().plora_last_error(h).decode() if h else ""
        raise PloraError(s, msg)


def _offsets(off) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(off, dtype=np.int64))


def make_table(ranks: Sequence[int], scales: Sequence[float], A: Sequence[int], B: Sequence[int],
               dA: Optional[Sequence[int]] = None, dB: Optional[Sequence[int]] = None):
    """Build a host plora_adapter[] from ranks, scales and device pointers (ints)."""
    n = len(ranks)
    tab = (plora_adapter * max(1, n))()
    for i in range(n):
        tab[i].rank = int(ranks[i])
        tab[i].scale = float(scales[i])
        tab[i].A = int(A[i])
        tab[i].B = int(B[i])
        tab[i].dA = int(dA[i]) if dA is not None else None
        tab[i].dB = int(dB[i]) if dB is not None else None
    return tab


# ---------------------------------------------------------------- C names
def plora_create(d_in: int, d_out: int, dtype: int, max_adapters: int, max_rank: int, max_tokens: int,
                 flags: int = 0, out_blocks=None) -> int:
    lib = load()
    cfg = make_config(d_in, d_out, dtype, max_adapters, max_rank, max_tokens, flags, out_blocks)
    h = ctypes.c_void_p()
    s = lib.plora_create(ctypes.byref(h), ctypes.byref(cfg))
    if s != PLORA_OK:
        raise PloraError(s, "plora_create")
    return h.value


def plora_create_status(cfg: plora_config):
    """Raw form: returns (status, handle-or-None)."""
    h = ctypes.c_void_p()
    s = load().plora_create(ctypes.byref(h), ctypes.byref(cfg))
    return s, h.value


def plora_destroy(h: int) -> None:
    _raise(None, load().plora_destroy(h))


def plora_saved_bytes(h: int, n: int, off, tab) -> int:
    off = _offsets(off)
    out = ctypes.c_size_t(0)
    _raise(h, load().plora_saved_bytes(h, n, off.ctypes.data, ctypes.addressof(tab), ctypes.byref(out)))
    return int(out.value)


def plora_forward(h: int, X: int, W: int, Y: int, n: int, off, tab, saved: int, stream: int = 0,
                  check: bool = True) -> int:
    off = _offsets(off)
    s = load().plora_forward(h, X, W, Y, n, off.ctypes.data, ctypes.addressof(tab), saved, stream)
    if check:
        _raise(h, s)
    return s


def plora_backward(h: int, X: int, W: int, dY: int, dX: Optional[int], n: int, off, tab, saved: int,
                   stream: int = 0, check: bool = True) -> int:
    off = _offsets(off)
    s = load().plora_backward(h, X, W, dY, dX or None, n, off.ctypes.data, ctypes.addressof(tab), saved, stream)
    if check:
        _raise(h, s)
    return s


def plora_check(h: int, stream: int = 0) -> int:
    return load().plora_check(h, stream)


def plora_last_error(h: int) -> str:
    return load().plora_last_error(h).decode()


def plora_debug_unpack_saved(h: int, n: int, off, tab, saved: int, i: int, H_out: int, stream: int = 0) -> None:
    off = _offsets(off)
    _raise(h, load().plora_debug_unpack_saved(h, n, off.ctypes.data, ctypes.addressof(tab), saved, i, H_out,
                                              stream))


def plora_debug_schedule(cfg: plora_config, n: int, off, tab, grads: bool, which: int):
    """Returns (status, int32 numpy array) of the host schedule; see include/plora.h."""
    lib = load()
    off = _offsets(off)
    cnt = ctypes.c_int64(0)
    tptr = ctypes.addressof(tab) if tab is not None else None
    s = lib.plora_debug_schedule(ctypes.byref(cfg), n, off.ctypes.data, tptr, int(grads), which, None, 0,
                                 ctypes.byref(cnt))
    if s != PLORA_OK:
        return s, None
    buf = np.zeros(max(1, cnt.value), dtype=np.int32)
    s = lib.plora_debug_schedule(ctypes.byref(cfg), n, off.ctypes.data, tptr, int(grads), which,
                                 buf.ctypes.data, cnt.value, ctypes.byref(cnt))
    return s, buf[:cnt.value]


def plora_profile_enable(h: int, enable: bool) -> None:
    _raise(h, load().plora_profile_enable(h, int(bool(enable))))


def plora_profile_read(h: int) -> dict:
    """{kernel kind: (launches, total device ms)} since the last read."""
    lib = load()
    cap = 32
    n = ctypes.c_int32(0)
    names = (ctypes.c_char_p * cap)()
    launches = (ctypes.c_int64 * cap)()
    ms = (ctypes.c_double * cap)()
    _raise(h, lib.plora_profile_read(h, cap, ctypes.byref(n), names, launches, ms))
    return {names[k].decode(): (int(launches[k]), float(ms[k])) for k in range(min(n.value, cap))}


def plora_capture_reserve(h: int, n: int) -> None:
    """Reserve n schedule slots for calls captured into CUDA graphs (one per captured call)."""
    _raise(h, load().plora_capture_reserve(h, int(n)))


def plora_capture_release(h: int) -> None:
    """Free the capture slots (only once no graph holding this handle's captured calls replays)."""
    _raise(h, load().plora_capture_release(h))


def plora_device_info(h: int) -> dict:
    """SMs of the handle's device, the co-resident 2-SM clusters of the pair base GEMMs, and this
    build's single-SM base-GEMM tile rows and rasterisation windows."""
    out = (ctypes.c_int32 * 6)()
    cnt = ctypes.c_int32(0)
    _raise(h, load().plora_device_info(h, ctypes.cast(out, ctypes.c_void_p), 6, ctypes.byref(cnt)))
    return {"sms": int(out[0]), "pairs_fwd": int(out[1]), "pairs_dx": int(out[2]), "base_rows": int(out[3]),
            "window_rows": int(out[4]), "dx_window_rows": int(out[5])}


# Nominal B200 peaks for the partition cost model (dense bf16 tensor FLOP/s, HBM bytes/s); only their
# ratio matters for the balance.
PARTITION_FLOPS = 2.25e15
PARTITION_BYTES = 8.0e12


def plora_partition(counts, ranks, d_in: int, d_out: int, n_parts: int, flops_per_s: float = PARTITION_FLOPS,
                    bytes_per_s: float = PARTITION_BYTES):
    """Assign each adapter to one of n_parts GPUs (longest processing time first over the per-adapter
    cost of include/plora.h).  Returns (owner int32[n], part_cost float64[n_parts]); raises PloraError."""
    counts = np.ascontiguousarray(counts, dtype=np.int64)
    ranks = np.ascontiguousarray(ranks, dtype=np.int32)
    n = len(counts)
    owner = np.full(n, -1, np.int32)
    cost = np.zeros(max(1, int(n_parts)), np.float64)
    st = load().plora_partition(n, counts.ctypes.data, ranks.ctypes.data, int(d_in), int(d_out), float(flops_per_s),
                                float(bytes_per_s), int(n_parts), owner.ctypes.data, cost.ctypes.data)
    if st != PLORA_OK:
        raise PloraError(st, "plora_partition")
    return owner, cost[:n_parts]


def shard(owner, off, part: int):
    """Part `part`'s share of a packed adapter set: (adapter ids in increasing order, their local
    offsets int64[k+1] into the part's own packed token buffer, and the global row ranges
    [(off[i], off[i+1])] to gather that buffer from).  Index bookkeeping only."""
    owner = np.asarray(owner)
    off = np.asarray(off, dtype=np.int64)
    ids = np.nonzero(owner == part)[0].astype(np.int64)
    counts = off[ids + 1] - off[ids]
    local = np.zeros(len(ids) + 1, np.int64)
    local[1:] = np.cumsum(counts)
    return ids, local, [(int(off[i]), int(off[i + 1])) for i in ids]


def plora_grad_B_static(cfg: plora_config, dY: int, n: int, off, tab, saved: int, stream: int = 0) -> int:
    """dB of every adapter without allocating (scratch in a static device array). Returns the status."""
    off = _offsets(off)
    return int(load().plora_grad_B_static(ctypes.byref(cfg), dY, n, off.ctypes.data, ctypes.addressof(tab),
                                          saved, stream))


def make_adamw_states(hparams, A_master, B_master, mA, vA, mB, vB):
    """Host plora_adamw_state[] from per-adapter dicts (lr, beta1, beta2, eps, weight_decay, step) and device
    pointers (ints; A_master / B_master may be None for an fp32 handle)."""
    n = len(hparams)
    st = (plora_adamw_state * max(1, n))()
    for i, hp in enumerate(hparams):
        st[i].lr = float(hp["lr"])
        st[i].beta1 = float(hp.get("beta1", 0.9))
        st[i].beta2 = float(hp.get("beta2", 0.999))
        st[i].eps = float(hp.get("eps", 1e-8))
        st[i].weight_decay = float(hp.get("weight_decay", 0.01))
        st[i].step = int(hp["step"])
        st[i].A_master = A_master[i] if A_master is not None else None
        st[i].B_master = B_master[i] if B_master is not None else None
        st[i].mA, st[i].vA, st[i].mB, st[i].vB = mA[i], vA[i], mB[i], vB[i]
    return st


def plora_adamw_step(h: int, n: int, tab, states, stream: int = 0, check: bool = True) -> int:
    s = load().plora_adamw_step(h, n, ctypes.addressof(tab), ctypes.addressof(states), stream)
    if check:
        _raise(h, s)
    return s


def plora_debug_timeout_probe(h: int, timeout_ns: int, stream: int = 0) -> int:
    return int(load().plora_debug_timeout_probe(h, int(timeout_ns), stream))


def plora_version() -> int:
    return int(load().plora_version())


# ---------------------------------------------------------------- torch convenience
class PackedLoRA:
    """Owns a handle; runs the packed forward/backward on torch CUDA tensors.

    ``A[i]`` is ``[r_i][d_in]`` (lora_A.weight), ``B[i]`` is ``[d_out][r_i]``
    (lora_B.weight), ``W`` is ``[d_out][d_in]`` (nn.Linear.weight), ``X`` is
    the packed ``[T][d_in]`` token buffer, ``off`` the host segment offsets.
    With ``out_blocks`` (the widths of P shared-input projections stacked in W, e.g.
    q, k, v), ``A[i]`` is the P projections' lora_A weights stacked, ``[P r_i][d_in]``,
    and ``B[i]`` their lora_B weights stacked, ``[d_out][r_i]``.
    """

    def __init__(self, d_in, d_out, dtype="bf16", max_adapters=64, max_rank=PLORA_MAX_RANK,
                 max_tokens=1 << 16, simt=False, unfused=False, base_pair=False, out_blocks=None):
        self.d_in, self.d_out = int(d_in), int(d_out)
        self.dtype = dtype
        self.out_blocks = list(out_blocks) if out_blocks is not None else None
        self.h = plora_create(self.d_in, self.d_out, PLORA_BF16 if dtype == "bf16" else PLORA_FP32,
                              max_adapters, max_rank, max_tokens,
                              (PLORA_FLAG_SIMT if simt else 0) | (PLORA_FLAG_UNFUSED if unfused else 0)
                              | (PLORA_FLAG_BASE_PAIR if base_pair else 0), out_blocks)

    def close(self):
        if self.h:
            plora_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def table(self, scales, A, B, dA=None, dB=None):
        ranks = [b.shape[1] for b in B]
        return make_table(ranks, scales, [a.data_ptr() for a in A], [b.data_ptr() for b in B],
                          None if dA is None else [x.data_ptr() for x in dA],
                          None if dB is None else [x.data_ptr() for x in dB])

    def saved_bytes(self, off, tab) -> int:
        return plora_saved_bytes(self.h, len(off) - 1, off, tab)

    def forward(self, X, W, off, scales, A, B, Y=None, saved=None, stream=None):
        import torch
        n = len(off) - 1
        tab = self.table(scales, A, B)
        if Y is None:
            Y = torch.empty((X.shape[0], self.d_out), dtype=X.dtype, device=X.device)
        nbytes = self.saved_bytes(off, tab)
        if saved is None:
            saved = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=X.device)
        st = (stream or torch.cuda.current_stream()).cuda_stream
        plora_forward(self.h, X.data_ptr(), W.data_ptr(), Y.data_ptr(), n, off, tab, saved.data_ptr(), st)
        return Y, saved

    def backward(self, X, W, dY, off, scales, A, B, saved, dX=None, dA=None, dB=None, want_dX=True, stream=None):
        import torch
        n = len(off) - 1
        if dA is None:
            dA = [torch.empty(a.shape, dtype=torch.float32, device=X.device) for a in A]
        if dB is None:
            dB = [torch.empty(b.shape, dtype=torch.float32, device=X.device) for b in B]
        if want_dX and dX is None:
            dX = torch.empty_like(X)
        tab = self.table(scales, A, B, dA, dB)
        st = (stream or torch.cuda.current_stream()).cuda_stream
        plora_backward(self.h, X.data_ptr(), W.data_ptr(), dY.data_ptr(), dX.data_ptr() if want_dX else None,
                       n, off, tab, saved.data_ptr(), st)
        return dX, dA, dB


# ---------------------------------------------------------------- layer calls
class plora_proj(ctypes.Structure):
    _fields_ = [("X", ctypes.c_void_p), ("W", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("dY", ctypes.c_void_p),
                ("dX", ctypes.c_void_p), ("tab", ctypes.c_void_p), ("saved", ctypes.c_void_p)]


def make_projs(items) -> "ctypes.Array":
    """plora_proj[n] from dicts with keys X, W, Y, dY, dX (device pointers or None), tab (a table from
    make_table) and saved (device pointer or None)."""
    arr = (plora_proj * len(items))()
    keep = []
    for k, it in enumerate(items):
        tab = it.get("tab")
        keep.append(tab)
        arr[k] = plora_proj(it.get("X"), it.get("W"), it.get("Y"), it.get("dY"), it.get("dX"),
                            ctypes.addressof(tab) if tab is not None else None, it.get("saved"))
    arr._keep = keep
    return arr


class PackedLoRALayer:
    """A layer call: several projections over one segment map (the same adapters over the same packed
    token rows) run as one launch set, one persistent launch per product kind over all of them.

    ``projections`` lists each projection as ``(d_in, d_out)`` or ``(d_in, d_out, out_blocks)``.
    ``forward(io, off, scales)`` takes one dict per projection with its ``X``, ``W``, ``A``, ``B``
    torch tensors and returns ``[(Y, saved)]``; ``backward(io, off, scales, saved)`` takes the same
    dicts with ``dY`` added and returns ``[(dX, dA, dB)]``.  ``scales`` is one list of per-adapter
    scales for every projection, or one such list per projection (an adapter's alpha / r differs
    between projections where its rank does).  Results equal separate calls bit for bit.
    """

    def __init__(self, projections, max_adapters=64, max_rank=PLORA_MAX_RANK, max_tokens=1 << 16):
        self.proj = [tuple(p) for p in projections]
        cfgs = (plora_config * len(self.proj))()
        for k, p in enumerate(self.proj):
            cfgs[k] = make_config(p[0], p[1], PLORA_BF16, max_adapters, max_rank, max_tokens, 0,
                                  p[2] if len(p) > 2 else None)
        h = ctypes.c_void_p()
        st = load().plora_layer_create(ctypes.byref(h), len(self.proj), cfgs)
        if st != PLORA_OK:
            raise PloraError(st, "plora_layer_create")
        self.L = h.value

    def handle(self, p: int) -> int:
        h = ctypes.c_void_p()
        st = load().plora_layer_handle(self.L, p, ctypes.byref(h))
        if st != PLORA_OK:
            raise PloraError(st, "plora_layer_handle")
        return h.value

    def close(self):
        if self.L:
            load().plora_layer_destroy(self.L)
            self.L = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _err(self, st, what):
        if st != PLORA_OK:
            raise PloraError(st, f"{what}: {load().plora_layer_last_error(self.L).decode()}")

    @staticmethod
    def _scales(scales, k):
        """Projection k's per-adapter scales from one shared list or a list per projection."""
        first = scales[0] if len(scales) else None
        return scales[k] if isinstance(first, (list, tuple, np.ndarray)) else scales

    @staticmethod
    def _table(scales, A, B, dA=None, dB=None):
        return make_table([b.shape[1] for b in B], scales, [a.data_ptr() for a in A], [b.data_ptr() for b in B],
                          None if dA is None else [x.data_ptr() for x in dA],
                          None if dB is None else [x.data_ptr() for x in dB])

    def forward(self, io, off, scales, stream=None):
        import torch
        off = np.ascontiguousarray(off, dtype=np.int64)
        n = len(off) - 1
        items, outs = [], []
        for k, d in enumerate(io):
            tab = self._table(self._scales(scales, k), d["A"], d["B"])
            Y = torch.empty((d["X"].shape[0], self.proj[k][1]), dtype=d["X"].dtype, device=d["X"].device)
            items.append({"X": d["X"].data_ptr(), "W": d["W"].data_ptr(), "Y": Y.data_ptr(), "tab": tab})
            outs.append(Y)
        projs = make_projs(items)
        sizes = (ctypes.c_size_t * len(io))()
        self._err(load().plora_layer_saved_bytes(self.L, n, off.ctypes.data, projs, sizes), "plora_layer_saved_bytes")
        saved = [torch.empty(max(int(b), 256), dtype=torch.uint8, device=d["X"].device) for b, d in zip(sizes, io)]
        for k in range(len(io)):
            projs[k].saved = saved[k].data_ptr()
        st = (stream or torch.cuda.current_stream()).cuda_stream
        self._err(load().plora_layer_forward(self.L, n, off.ctypes.data, projs, st), "plora_layer_forward")
        return list(zip(outs, saved))

    def backward(self, io, off, scales, saved, want_dX=True, stream=None):
        import torch
        off = np.ascontiguousarray(off, dtype=np.int64)
        n = len(off) - 1
        items, outs = [], []
        for k, d in enumerate(io):
            dA = [torch.empty(a.shape, dtype=torch.float32, device=a.device) for a in d["A"]]
            dB = [torch.empty(b.shape, dtype=torch.float32, device=b.device) for b in d["B"]]
            dX = torch.empty_like(d["X"]) if want_dX else None
            tab = self._table(self._scales(scales, k), d["A"], d["B"], dA, dB)
            items.append({"X": d["X"].data_ptr(), "W": d["W"].data_ptr(), "dY": d["dY"].data_ptr(),
                          "dX": dX.data_ptr() if want_dX else None, "tab": tab, "saved": saved[k].data_ptr()})
            outs.append((dX, dA, dB))
        projs = make_projs(items)
        st = (stream or torch.cuda.current_stream()).cuda_stream
        self._err(load().plora_layer_backward(self.L, n, off.ctypes.data, projs, st), "plora_layer_backward")
        return outs

    def check(self, stream=None) -> int:
        return int(load().plora_layer_check(self.L, stream))


# ---------------------------------------------------------------- autograd
def packed_lora(engine: "PackedLoRA", X, W, off, scales, A, B):
    """Y = X W + s_i (X_i A_i) B_i for every packed adapter, differentiable in X, A_i and B_i
    (W is the frozen base weight and gets no gradient).  A[i] is lora_A.weight ([r_i][d_in]),
    B[i] is lora_B.weight ([d_out][r_i]), W is nn.Linear.weight ([d_out][d_in]); `off` holds
    the host segment offsets of the packed rows of X.  The backward runs plora_backward; the
    fp32 weight gradients are returned in each parameter's dtype."""
    import torch

    class _PackedLoRAFn(torch.autograd.Function):
        @staticmethod
        def forward(ctx, X_, W_, *AB):
            n = len(off) - 1
            A_, B_ = list(AB[:n]), list(AB[n:])
            Y, saved = engine.forward(X_.contiguous(), W_.contiguous(), off, scales, A_, B_)
            ctx.save_for_backward(X_, W_, saved, *AB)
            return Y

        @staticmethod
        def backward(ctx, dY):
            X_, W_, saved, *AB = ctx.saved_tensors
            n = len(off) - 1
            A_, B_ = list(AB[:n]), list(AB[n:])
            dX, dA, dB = engine.backward(X_, W_, dY.contiguous(), off, scales, A_, B_, saved,
                                         want_dX=ctx.needs_input_grad[0])
            gA = [g.to(a.dtype) for g, a in zip(dA, A_)]
            gB = [g.to(b.dtype) for g, b in zip(dB, B_)]
            return (dX, None, *gA, *gB)

    if W.requires_grad:
        raise ValueError("packed_lora: the base weight W is frozen; pass W with requires_grad=False")
    return _PackedLoRAFn.apply(X, W, *A, *B)
