"""Seeded synthetic inputs for the MoE-layer forward workloads.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark. It holds no arithmetic of the method itself (no routing, no
permutation, no FFN): only the workload table and the random draws.

Recipe (every workload):
  * draws are standard normals from numpy's PCG64, one independent stream per
    (seed, tensor, chunk) made by ``numpy.random.SeedSequence``; chunks are
    drawn on a thread pool, so the values do not depend on the thread count;
  * order of tensors: x, W_r, W_gate, W_up, W_down (logits first, then x, for
    the dispatch/combine-only sweep);
  * x ~ N(0, 1); weights ~ N(0, 0.02) with 0.02 read as the standard
    deviation; values drawn in fp32, then rounded to bf16 (round to nearest
    even, by torch) for the bf16 workloads;
  * the skewed workload adds a fixed Zipf(s=1.2) router bias whose scale was
    fitted by ``oracle/fit_zipf_bias.py`` and is read from
    ``tests/golden/zipf_bias_alpha.json``.

The shapes mirror the model rows of the SonicMoE explainer (gitcode.csdn.net
page, section 2: Mixtral 8 experts / top-2, Qwen3-30B-A3B 128 / top-8,
gpt-oss 32 / top-4).
"""
from __future__ import annotations

import json
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
ZIPF_ALPHA_FILE = os.path.join(_HERE, "tests", "golden", "zipf_bias_alpha.json")

# tensor keys for the seed sequence (stable across versions: never renumber)
_KEY_X, _KEY_WR, _KEY_WG, _KEY_WU, _KEY_WD, _KEY_LOGITS = 1, 2, 3, 4, 5, 6

_CHUNK = 1 << 22  # elements per independent stream


@dataclass(frozen=True)
class MoEConfig:
    """One workload: T tokens of width d, E experts, top-K, expert width n."""

    name: str
    T: int
    d: int
    E: int
    K: int
    n: int
    dtype: str  # "f32" or "bf16" (activations and weights)
    capacity_factor: float = 0.0  # <= 0: no limit
    zipf_s: float = 0.0  # > 0: add the Zipf-ranked router bias
    logits_given: bool = False  # dispatch/combine-only: seeded fp32 logits
    identity_experts: bool = False
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    logits_std: float = 1.0

    @property
    def A(self) -> int:
        return self.T * self.K

    def with_T(self, T: int) -> "MoEConfig":
        return replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")


# The five workloads (sizes exactly as stated for the layer forward).
TINY_FP32 = MoEConfig("tiny_fp32", T=256, d=128, E=8, K=2, n=256, dtype="f32")
MIXTRAL_BF16 = MoEConfig("mixtral_bf16", T=4096, d=4096, E=8, K=2, n=14336, dtype="bf16")
FINE_GRAINED_BF16 = MoEConfig("fine_grained_bf16", T=16384, d=2048, E=128, K=8, n=768,
                              dtype="bf16")
SKEWED_CAPACITY_BF16 = MoEConfig("skewed_capacity_bf16", T=8192, d=2880, E=32, K=4, n=2880,
                                 dtype="bf16", capacity_factor=1.25, zipf_s=1.2)
DISPATCH_COMBINE = MoEConfig("dispatch_combine", T=4096, d=4096, E=64, K=6, n=0,
                             dtype="bf16", logits_given=True, identity_experts=True)
DISPATCH_COMBINE_T = (64, 256, 1024, 4096, 16384, 65536)

CONFIGS = {c.name: c for c in (TINY_FP32, MIXTRAL_BF16, FINE_GRAINED_BF16,
                               SKEWED_CAPACITY_BF16, DISPATCH_COMBINE)}


def zipf_alpha() -> float:
    """Scale of the Zipf router bias for the skewed workload (fitted, frozen)."""
    with open(ZIPF_ALPHA_FILE) as f:
        return float(json.load(f)["alpha"])


def zipf_bias(E: int, s: float, alpha: float) -> torch.Tensor:
    """bias_e = alpha * (e + 1) ** (-s): expert 0 is the hottest (rank = id)."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    return (alpha * ranks.pow(-s)).to(torch.float32)


def _draw_chunk(seed: int, key: int, sub: int, chunk: int, count: int) -> np.ndarray:
    ss = np.random.SeedSequence([seed, key, sub, chunk])
    return np.random.Generator(np.random.PCG64(ss)).standard_normal(count, dtype=np.float32)


_POOL: Optional[ThreadPoolExecutor] = None


def _pool() -> ThreadPoolExecutor:
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))
    return _POOL


def normal(shape, std: float, seed: int, key: int, sub: int = 0) -> torch.Tensor:
    """fp32 tensor of N(0, std^2) draws; chunked streams, thread-count independent."""
    numel = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(numel, dtype=np.float32)
    nchunks = max(1, math.ceil(numel / _CHUNK))

    def work(c):
        lo = c * _CHUNK
        hi = min(numel, lo + _CHUNK)
        out[lo:hi] = _draw_chunk(seed, key, sub, c, hi - lo)

    list(_pool().map(work, range(nchunks)))
    t = torch.from_numpy(out).view(*shape)
    if std != 1.0:
        t.mul_(std)
    return t


def _cast(t: torch.Tensor, dtype: str) -> torch.Tensor:
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _expert_stack(E, rows, cols, std, seed, key, dtype) -> torch.Tensor:
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty(E, rows, cols, dtype=tdt)
    for e in range(E):
        out[e] = _cast(normal((rows, cols), std, seed, key, sub=e), dtype)
    return out


@dataclass
class MoEInputs:
    cfg: MoEConfig
    x: torch.Tensor
    w_r: Optional[torch.Tensor] = None
    w_gate: Optional[torch.Tensor] = None
    w_up: Optional[torch.Tensor] = None
    w_down: Optional[torch.Tensor] = None
    bias: Optional[torch.Tensor] = None
    logits: Optional[torch.Tensor] = None
    extra: dict = field(default_factory=dict)

    def to(self, device) -> "MoEInputs":
        def mv(t):
            return None if t is None else t.to(device)
        return MoEInputs(self.cfg, mv(self.x), mv(self.w_r), mv(self.w_gate), mv(self.w_up),
                         mv(self.w_down), mv(self.bias), mv(self.logits), dict(self.extra))


def make_inputs(cfg: MoEConfig, with_experts: bool = True) -> MoEInputs:
    """All host (CPU) tensors of one workload, seeded as in the module docstring."""
    s = cfg.seed
    if cfg.logits_given:
        logits = normal((cfg.T, cfg.E), cfg.logits_std, s, _KEY_LOGITS)
        x = _cast(normal((cfg.T, cfg.d), cfg.x_std, s, _KEY_X), cfg.dtype)
        return MoEInputs(cfg, x=x, logits=logits)
    x = _cast(normal((cfg.T, cfg.d), cfg.x_std, s, _KEY_X), cfg.dtype)
    w_r = _cast(normal((cfg.d, cfg.E), cfg.w_std, s, _KEY_WR), cfg.dtype)
    inp = MoEInputs(cfg, x=x, w_r=w_r)
    if cfg.zipf_s > 0:
        inp.bias = zipf_bias(cfg.E, cfg.zipf_s, zipf_alpha())
    if with_experts and cfg.n > 0:
        inp.w_gate = _expert_stack(cfg.E, cfg.d, cfg.n, cfg.w_std, s, _KEY_WG, cfg.dtype)
        inp.w_up = _expert_stack(cfg.E, cfg.d, cfg.n, cfg.w_std, s, _KEY_WU, cfg.dtype)
        inp.w_down = _expert_stack(cfg.E, cfg.n, cfg.d, cfg.w_std, s, _KEY_WD, cfg.dtype)
    return inp


# --------------------------------------------------------------------------- atomic experts
_KEY_WROW, _KEY_WCOL, _KEY_WIN, _KEY_WOUT, _KEY_PLOGITS = 7, 8, 9, 10, 11


@dataclass(frozen=True)
class OmniConfig:
    """Fine-grained (rank-1, "atomic") experts behind a Cartesian-product router:
    N = n_rows * n_cols experts, each a pair of d-vectors (w_in, w_out); top-K
    per token. Sizes of the "Two upstream innovations of MoE: Routing-Free and
    OmniMoE" page, section 4: 102,400 experts per layer on a 320 x 320 grid, K
    from 512 to 4096, 4096 tokens through a ~200M-parameter layer (2 N d =
    210M at d = 1024)."""

    name: str
    T: int
    d: int
    n_rows: int
    n_cols: int
    K: int
    renormalize: bool = True
    logits_given: bool = False  # seeded fp32 row/column logits instead of x W
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    logits_std: float = 1.0

    @property
    def N(self) -> int:
        return self.n_rows * self.n_cols

    @property
    def A(self) -> int:
        return self.T * self.K


OMNI_SMALL = OmniConfig("omni_small", T=256, d=256, n_rows=32, n_cols=32, K=64)
OMNI_102K = OmniConfig("omni_102k", T=4096, d=1024, n_rows=320, n_cols=320, K=512)
OMNI_CONFIGS = {c.name: c for c in (OMNI_SMALL, OMNI_102K)}


@dataclass
class OmniInputs:
    cfg: OmniConfig
    x: torch.Tensor                       # [T, d] bf16
    w_row: Optional[torch.Tensor] = None  # [d, n_rows] bf16
    w_col: Optional[torch.Tensor] = None  # [d, n_cols] bf16
    w_in: Optional[torch.Tensor] = None   # [N, d] bf16
    w_out: Optional[torch.Tensor] = None  # [N, d] bf16
    logits: Optional[torch.Tensor] = None  # [T, n_rows + n_cols] fp32 (logits_given)


def make_omni_inputs(cfg: OmniConfig, with_experts: bool = True) -> OmniInputs:
    """Host tensors of one atomic-expert workload: x ~ N(0, 1), router and expert
    tables ~ N(0, 0.02), drawn in fp32 in the order x, W_row, W_col, W_in, W_out
    and rounded to bf16; or, with ``logits_given``, N(0, 1) fp32 logits."""
    s = cfg.seed
    x = _cast(normal((cfg.T, cfg.d), cfg.x_std, s, _KEY_X), "bf16")
    inp = OmniInputs(cfg, x=x)
    if cfg.logits_given:
        inp.logits = normal((cfg.T, cfg.n_rows + cfg.n_cols), cfg.logits_std, s, _KEY_PLOGITS)
    else:
        inp.w_row = _cast(normal((cfg.d, cfg.n_rows), cfg.w_std, s, _KEY_WROW), "bf16")
        inp.w_col = _cast(normal((cfg.d, cfg.n_cols), cfg.w_std, s, _KEY_WCOL), "bf16")
    if with_experts:
        inp.w_in = _cast(normal((cfg.N, cfg.d), cfg.w_std, s, _KEY_WIN), "bf16")
        inp.w_out = _cast(normal((cfg.N, cfg.d), cfg.w_std, s, _KEY_WOUT), "bf16")
    return inp


def random_small_config(rng: np.random.Generator, dtype: str = "f32", name: str = "rand",
                        max_T: int = 64) -> MoEConfig:
    """A random tiny shape for property tests (both sides get the same draw)."""
    E = int(rng.integers(1, 17))
    K = int(rng.integers(1, E + 1))
    T = int(rng.integers(1, max_T + 1))
    d = int(rng.choice([64, 128]))
    n = int(rng.choice([64, 128, 192]))
    cf = float(rng.choice([0.0, 0.5, 1.0, 2.0]))
    seed = int(rng.integers(0, 2**31 - 1))
    return MoEConfig(name, T=T, d=d, E=E, K=K, n=n, dtype=dtype, capacity_factor=cf, seed=seed)
