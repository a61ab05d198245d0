"""Seeded synthetic inputs for packed LoRA fine-tuning workloads.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the LoRA arithmetic: the oracle (``oracle/``) and the CUDA
path (``packed_lora_fine_b200``) both consume what it produces, and neither
shares any other code with the other.

Storage layouts (row-major, the PyTorch / PEFT module layouts):

* ``X[T][d_in]``        packed token buffer, adapter i owns rows off[i]..off[i+1]
* ``W[d_out][d_in]``    frozen base weight, ``nn.Linear.weight``
* ``A[i][r_i][d_in]``   ``lora_A.weight`` of adapter i
* ``B[i][d_out][r_i]``  ``lora_B.weight`` of adapter i
* ``dY[T][d_out]``      upstream gradient

bf16 tensors are held as ``uint16`` bit patterns, fp32 tensors as ``float32``.
Every value is drawn from numpy's PCG64 and rounded once, round-to-nearest-even,
to the storage dtype; both sides then read exactly the same numbers.

The workload shapes follow the LoRA fine-tuning setups the PLoRA summary page
evaluates (Qwen-2.5 and LLaMA-3 projection layers, up to 32 packed adapters;
gist.science/zh/paper/2508.02932, 技术摘要 › 结果), and the long-tail mix of
sequence lengths across tenants reported on the LobRA announcement
(scholat.com/orgPost.html?id=2494, 图1).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, List, Optional, Sequence

import numpy as np

# Stream ids: each tensor comes from its own PCG64 stream, keyed by (seed, id).
_S_OFF, _S_RANK, _S_ALPHA, _S_W, _S_X, _S_DY = 0, 1, 2, 3, 4, 5
_S_ADAPTER = 100  # adapter i uses 100 + 2*i (A) and 101 + 2*i (B)
_CHUNK = 1 << 22


def rng_for(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(stream)])))


# ----------------------------------------------------------------------------
# dtype helpers (rounding and exact widening; no LoRA arithmetic)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of a storage array to float64."""
    if dtype == "bf16":
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def from_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype (via fp32, then RNE to bf16)."""
    a32 = np.asarray(a, dtype=np.float64).astype(np.float32)
    return f32_to_bf16_bits(a32) if dtype == "bf16" else a32


def _draw(rng: np.random.Generator, shape, dtype: str, kind: str, p: float) -> np.ndarray:
    """Draw `shape` values and round to `dtype`.

    kind "normal": N(0, p) (p is the standard deviation);
    kind "uniform": U(-p, p).
    Large tensors are drawn in fixed-size chunks, in order, from one stream.
    """
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        if kind == "normal":
            v = rng.standard_normal(m, dtype=np.float32 if dtype == "bf16" else np.float64)
            v = v * np.asarray(p, dtype=v.dtype)
        elif kind == "uniform":
            v = rng.random(m, dtype=np.float32 if dtype == "bf16" else np.float64)
            v = (v * 2 - 1) * np.asarray(p, dtype=v.dtype)
        else:
            raise ValueError(kind)
        out[s:s + m] = f32_to_bf16_bits(v.astype(np.float32)) if dtype == "bf16" else v.astype(np.float32)
    return out.reshape(shape)


# ----------------------------------------------------------------------------
# Problem description
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Init:
    """Distributions. Each entry is (kind, parameter); see `_draw`."""
    X: tuple
    W: tuple
    A: tuple
    B: tuple
    dY: tuple


def init_llm(d_in: int) -> Init:
    """W ~ N(0, 0.02); A He-uniform U(+-sqrt(6/d_in)); B ~ N(0, 0.01); X, dY ~ N(0, 1)."""
    return Init(X=("normal", 1.0), W=("normal", 0.02), A=("uniform", math.sqrt(6.0 / d_in)),
                B=("normal", 0.01), dY=("normal", 1.0))


def init_small(d_in: int) -> Init:
    """X, W, A ~ N(0,1)/sqrt(d_in); B ~ N(0, 0.02); dY ~ N(0, 1)."""
    s = 1.0 / math.sqrt(d_in)
    return Init(X=("normal", s), W=("normal", s), A=("normal", s), B=("normal", 0.02), dY=("normal", 1.0))


@dataclasses.dataclass
class Problem:
    name: str
    dtype: str                  # "bf16" or "fp32": storage dtype of X, W, A, B, Y, dY, dX
    d_in: int
    d_out: int
    off: np.ndarray             # int64 [N+1], off[0] = 0, monotone
    ranks: np.ndarray           # int32 [N]
    alphas: np.ndarray          # float64 [N]
    scales: np.ndarray          # float32 [N], alpha / rank rounded to fp32
    X: np.ndarray
    W: np.ndarray
    A: List[np.ndarray]
    B: List[np.ndarray]
    dY: np.ndarray
    seed: int = 0

    @property
    def n_adapters(self) -> int:
        return int(len(self.ranks))

    @property
    def T(self) -> int:
        return int(self.off[-1])

    @property
    def counts(self) -> np.ndarray:
        return np.diff(self.off)

    def describe(self) -> dict:
        return {"name": self.name, "dtype": self.dtype, "d_in": self.d_in, "d_out": self.d_out,
                "adapters": self.n_adapters, "tokens": self.T,
                "ranks": [int(r) for r in self.ranks], "seed": self.seed}


def make_problem(name: str, dtype: str, d_in: int, d_out: int, ranks: Sequence[int],
                 counts: Sequence[int], alphas: Sequence[float], init: Init, seed: int,
                 draw_tokens: bool = True) -> Problem:
    ranks = np.asarray(ranks, dtype=np.int32)
    counts = np.asarray(counts, dtype=np.int64)
    alphas = np.asarray(alphas, dtype=np.float64)
    assert ranks.shape == counts.shape == alphas.shape
    off = np.zeros(len(counts) + 1, dtype=np.int64)
    off[1:] = np.cumsum(counts)
    T = int(off[-1])
    scales = (alphas / ranks.astype(np.float64)).astype(np.float32)
    W = _draw(rng_for(seed, _S_W), (d_out, d_in), dtype, *init.W)
    if draw_tokens:
        X = _draw(rng_for(seed, _S_X), (T, d_in), dtype, *init.X)
        dY = _draw(rng_for(seed, _S_DY), (T, d_out), dtype, *init.dY)
    else:
        X = dY = None
    A, B = [], []
    for i, r in enumerate(ranks):
        A.append(_draw(rng_for(seed, _S_ADAPTER + 2 * i), (int(r), d_in), dtype, *init.A))
        B.append(_draw(rng_for(seed, _S_ADAPTER + 2 * i + 1), (d_out, int(r)), dtype, *init.B))
    return Problem(name, dtype, d_in, d_out, off, ranks, alphas, scales, X, W, A, B, dY, seed)


def random_problem(seed: int, dtype: str, d_in: int, d_out: int, n_adapters: int,
                   rank_choices: Sequence[int], count_range: tuple, name: str = "random",
                   init: Optional[Init] = None) -> Problem:
    """Small random mix used by tests: ranks uniform over `rank_choices`,
    token counts uniform in [count_range[0], count_range[1]], alpha = 2*rank."""
    g = rng_for(seed, _S_RANK)
    ranks = g.choice(np.asarray(rank_choices), size=n_adapters)
    counts = rng_for(seed, _S_OFF).integers(count_range[0], count_range[1] + 1, size=n_adapters)
    return make_problem(name, dtype, d_in, d_out, ranks, counts, 2.0 * ranks,
                        init or (init_small(d_in) if dtype == "fp32" else init_llm(d_in)), seed)


# ----------------------------------------------------------------------------
# The five workload configurations
# ----------------------------------------------------------------------------

def config1(seed: int = 1001) -> Problem:
    """Single 256x256 fp32 layer, 4 adapters, ranks {4,8,8,16}, alpha = 2r, segments {64,128,32,96}."""
    r = [4, 8, 8, 16]
    return make_problem("cfg1_fp32_256", "fp32", 256, 256, r, [64, 128, 32, 96],
                        [2.0 * x for x in r], init_small(256), seed)


def config2(seed: int = 1002) -> Problem:
    """Qwen-2.5-7B q_proj 3584->3584, bf16, 8 adapters ranks {8,8,16,16,32,32,64,64}, 2x1024 tokens each."""
    r = [8, 8, 16, 16, 32, 32, 64, 64]
    return make_problem("cfg2_qwen_qproj", "bf16", 3584, 3584, r, [2048] * 8,
                        [2.0 * x for x in r], init_llm(3584), seed)


def config3_shape(seed: int = 1003):
    """Ranks, token counts and alphas of the LLaMA-3-8B up_proj 32-adapter long-tail mix."""
    n = 32
    ranks = rng_for(seed, _S_RANK).choice(np.array([8, 16, 32, 64, 128]), size=n)
    u = rng_for(seed, _S_OFF).uniform(math.log(512.0), math.log(4096.0), size=n)
    counts = np.rint(np.exp(u)).astype(np.int64)
    alphas = rng_for(seed, _S_ALPHA).choice(np.array([8.0, 16.0, 32.0]), size=n)
    return ranks, counts, alphas


def config3(seed: int = 1003, draw_tokens: bool = True) -> Problem:
    """LLaMA-3-8B up_proj 4096->14336, bf16, 32 adapters, r ~ U{8..128}, n ~ logU[512,4096], alpha ~ U{8,16,32}."""
    ranks, counts, alphas = config3_shape(seed)
    return make_problem("cfg3_llama_up_proj", "bf16", 4096, 14336, ranks, counts, alphas,
                        init_llm(4096), seed, draw_tokens)


LLAMA3_LAYER = [("q", 4096, 4096), ("k", 4096, 1024), ("v", 4096, 1024), ("o", 4096, 4096),
                ("gate", 4096, 14336), ("up", 4096, 14336), ("down", 14336, 4096)]


def config4_ranks(seed: int = 1004) -> np.ndarray:
    """The 16 adapter ranks of the one-layer workload, U{16,32,64}."""
    return rng_for(seed, _S_RANK).choice(np.array([16, 32, 64]), size=16)


def config4_projection(index: int, seed: int = 1004, draw_tokens: bool = True) -> Problem:
    """Projection `index` of LLAMA3_LAYER in the one-layer workload: 16 adapters r ~ U{16,32,64},
    4x2048 tokens each, with its own W, X, dY and per-adapter A, B (independent streams)."""
    nm, di, do = LLAMA3_LAYER[index]
    ranks = config4_ranks(seed)
    return make_problem(f"cfg4_llama_{nm}", "bf16", di, do, ranks, [8192] * 16, 2.0 * ranks, init_llm(di),
                        seed * 16 + index, draw_tokens)


def config4(seed: int = 1004, draw_tokens: bool = True) -> List[Problem]:
    """One LLaMA-3-8B layer's seven LoRA targets (config4_projection for each of LLAMA3_LAYER)."""
    return [config4_projection(k, seed, draw_tokens) for k in range(len(LLAMA3_LAYER))]


def config5_scaling(k: int, seed: int = 1005) -> Problem:
    """4096->4096, bf16, k adapters of rank 16 with 2048 tokens each."""
    return make_problem(f"cfg5_scale_k{k}", "bf16", 4096, 4096, [16] * k, [2048] * k,
                        [32.0] * k, init_llm(4096), seed)


def config5_mix(which: str, seed: int = 1005) -> Problem:
    """Degenerate mixes on 4096->4096, bf16.
    i:   8 adapters alternating rank 1 and rank 256, 2048 tokens each
    ii:  8 adapters with 1 and 8192 tokens alternating, rank 16
    iii: 16 equal segments of 2048 tokens, rank ~ U{1,16,256}
    iv:  mix iii with a 0-token adapter inserted (an added edge case: an adapter with no tokens)"""
    if which == "i":
        r = [1, 256] * 4
        c = [2048] * 8
    elif which == "ii":
        r = [16] * 8
        c = [1, 8192] * 4
    elif which in ("iii", "iv"):
        r = list(rng_for(seed, _S_RANK).choice(np.array([1, 16, 256]), size=16))
        c = [2048] * 16
        if which == "iv":
            r.insert(5, 16)
            c.insert(5, 0)
    else:
        raise ValueError(which)
    r = [int(x) for x in r]
    return make_problem(f"cfg5_mix_{which}", "bf16", 4096, 4096, r, c, [2.0 * x for x in r],
                        init_llm(4096), seed)


def with_zero_B(p: Problem) -> Problem:
    """Same problem with every B_i = 0 (the LoRA init of the B factor)."""
    q = dataclasses.replace(p)
    q.B = [np.zeros_like(b) for b in p.B]
    return q


def with_zero_W(p: Problem) -> Problem:
    """Same problem with W = 0, so Y and dX hold only the LoRA terms."""
    q = dataclasses.replace(p)
    q.W = np.zeros_like(p.W)
    return q


def take_adapters(p: Problem, ids) -> Problem:
    """The adapters `ids` of p (in that order) as a problem of their own: their rows of X and dY packed
    contiguously with local offsets, their factors, the same W.  Data selection only (one GPU's share
    of an adapter set split across GPUs)."""
    ids = [int(i) for i in ids]
    counts = np.array([p.off[i + 1] - p.off[i] for i in ids], dtype=np.int64)
    off = np.zeros(len(ids) + 1, dtype=np.int64)
    off[1:] = np.cumsum(counts)

    def rows(a):
        if a is None:
            return None
        parts = [a[p.off[i]:p.off[i + 1]] for i in ids]
        return np.ascontiguousarray(np.concatenate(parts)) if parts else a[:0].copy()
    return dataclasses.replace(p, name=f"{p.name}_part", off=off, ranks=p.ranks[ids], alphas=p.alphas[ids],
                               scales=p.scales[ids], X=rows(p.X), dY=rows(p.dY), A=[p.A[i] for i in ids],
                               B=[p.B[i] for i in ids])


def sample_rows(p: Problem, per_segment: int = 6, seed: int = 7) -> np.ndarray:
    """First, last and `per_segment` random rows of every non-empty segment (sorted, unique)."""
    g = np.random.default_rng(seed)
    rows = []
    for i in range(p.n_adapters):
        a, b = int(p.off[i]), int(p.off[i + 1])
        if b <= a:
            continue
        rows += [a, b - 1]
        rows += list(g.integers(a, b, size=min(per_segment, b - a)))
    return np.unique(np.asarray(rows, dtype=np.int64))
