"""Seeded synthetic inputs for the token-choice MoE layer.

This module draws numbers and nothing else: it holds none of the layer's
arithmetic (no router product, no top-k, no softmax, no expert FFN). Both the
CUDA path and the CPU oracle take their inputs from here, so it is the only
code the two sides share.

Every tensor has its own random stream, keyed by (seed, stream id, ...) through
numpy's SeedSequence spawn keys and drawn with PCG64, so a tensor (or one
expert's slice of it, or one token row) can be regenerated on its own:

    stream 0  h        token hidden states          N(0, 1)
    stream 1  W_r      router weight [E, d]         N(0, 1/d)
    stream 2  W_gate   [E, F, d], one stream/expert N(0, 1/d)
    stream 3  W_up     [E, F, d], one stream/expert N(0, 1/d)
    stream 4  W_down   [E, d, F], one stream/expert N(0, 1/F)
    stream 5  bias     router bias draws            N(0, 1)
    stream 6  redraw of one token row h_t           key (6, t, attempt)
    stream 7  redraw of one router column W_r[:, c] key (7, c, attempt)
    stream 8  dy       upstream gradient of y (backward) N(0, 1)

Streams 6 and 7 exist for the test-side pass that keeps every token's top-k
router scores at least 1e-3 apart (that pass needs the router arithmetic, so
it lives with the oracle, not here).

bf16 workloads are rounded to bf16 (round to nearest even) once, here; the
oracle reads those exact values widened to fp64.
"""
from __future__ import annotations

import json
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch

STREAM_H, STREAM_WR, STREAM_WG, STREAM_WU, STREAM_WD, STREAM_BIAS = 0, 1, 2, 3, 4, 5
STREAM_REDRAW_H, STREAM_REDRAW_WR_COL = 6, 7
STREAM_DY = 8

_HERE = os.path.dirname(os.path.abspath(__file__))
DERIVED_PATH = os.path.join(_HERE, "derived.json")


@dataclass(frozen=True)
class Workload:
    """One synthetic MoE layer problem.

    bias: "none" | "zipf_3_empty" | "gauss_0.5" | "hot16_empty8"
    capacity: -1 for dropless, else the per-expert cap in assignments.
    expert_kind: "swiglu" | "identity" | "scale"
    tagged: identity-tagged tokens h_t = (t+1) * onehot(t mod d).
    gemm_tiles: "auto" | "single" | "pair" (tile shape of the grouped GEMMs).
    layout: "compact" | "padded" (row layout of the permuted buffers with a
        capacity: kept rows only, or capacity rows per expert).
    """

    name: str
    T: int
    d: int
    E: int
    k: int
    F: int
    dtype: str = "bf16"
    bias: str = "none"
    capacity: int = -1
    expert_kind: str = "swiglu"
    tagged: bool = False
    gemm_tiles: str = "auto"
    layout: str = "compact"
    note: str = ""

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def capacity_factor_cap(T: int, k: int, E: int, num: int = 5, den: int = 4) -> int:
    """floor((num/den) * T * k / E) in exact integer arithmetic (1.25 = 5/4)."""
    return (num * T * k) // (den * E)


# The five problems the layer is measured on. Sizes are the names' sizes.
WORKLOADS = {
    "tiny_f32": Workload(
        "tiny_f32", T=64, d=32, E=4, k=2, F=64, dtype="f32",
        note="tiny fp32 layer T=64 d=32 E=4 k=2 F=64"),
    "mixtral_scaled": Workload(
        "mixtral_scaled", T=4096, d=1024, E=8, k=2, F=3584,
        note="Mixtral-style layer scaled down T=4096 d=1024 E=8 k=2 F=3584, unbiased router"),
    "skewed": Workload(
        "skewed", T=16384, d=2048, E=64, k=6, F=1408, bias="zipf_3_empty",
        note="skewed routing T=16384 d=2048 E=64 k=6 F=1408, b_e=-2ln(e+1), experts 1,31,63 empty"),
    "mixtral_8x7b": Workload(
        "mixtral_8x7b", T=32768, d=4096, E=8, k=2, F=14336, bias="gauss_0.5",
        note="Mixtral 8x7B layer shape T=32768 d=4096 E=8 k=2 F=14336, bias 0.5*N(0,1)"),
    "many_small": Workload(
        "many_small", T=8192, d=2048, E=128, k=8, F=768, bias="hot16_empty8",
        note="many small experts T=8192 d=2048 E=128 k=8 F=768, 16 hot experts take 50%, 8 empty"),
}

# Variants used by tests and the bench.
VARIANTS = {
    "tiny_f32_tagged": WORKLOADS["tiny_f32"].with_(
        name="tiny_f32_tagged", tagged=True, expert_kind="scale",
        note="identity-tagged tokens, scale-by-(e+1) experts"),
    "skewed_capacity": WORKLOADS["skewed"].with_(
        name="skewed_capacity", capacity=capacity_factor_cap(16384, 6, 64),
        note="skewed routing with capacity floor(1.25*T*k/E)=1920, overflow dropped in token order"),
    "skewed_capacity_padded": WORKLOADS["skewed"].with_(
        name="skewed_capacity_padded", capacity=capacity_factor_cap(16384, 6, 64), layout="padded",
        note="skewed routing, capacity 1920, padded layout: every expert computes 1920 rows"),
    "many_small_identity": WORKLOADS["many_small"].with_(
        name="many_small_identity", expert_kind="identity",
        note="many small experts with identity experts: permute + unpermute only"),
}

ALL = {**WORKLOADS, **VARIANTS}

HOT_EXPERTS = 16      # many_small: experts 0..15 get +beta
EMPTY_FROM = 120      # many_small: experts 120..127 get -inf
SKEWED_EMPTY = (1, 31, 63)


def get(name: str) -> Workload:
    return ALL[name]


def rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(key))))


def normal(seed: int, key: tuple, shape, std: float = 1.0) -> np.ndarray:
    a = rng(seed, *key).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def _to(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype)


def derived() -> dict:
    """Constants written by the oracle-side derivation script (stored, not computed here)."""
    with open(DERIVED_PATH) as f:
        return json.load(f)


def draw_h(wl: Workload, seed: int = 0) -> torch.Tensor:
    if wl.tagged:
        h = np.zeros((wl.T, wl.d), np.float32)
        t = np.arange(wl.T)
        h[t, t % wl.d] = (t + 1).astype(np.float32)
        return _to(h, wl.torch_dtype)
    return _to(normal(seed, (STREAM_H,), (wl.T, wl.d)), wl.torch_dtype)


def draw_dy(wl: Workload, seed: int = 0) -> torch.Tensor:
    """Upstream gradient dL/dy [T, d] for the backward pass."""
    return _to(normal(seed, (STREAM_DY,), (wl.T, wl.d)), wl.torch_dtype)


def redraw_h_row(wl: Workload, seed: int, t: int, attempt: int) -> torch.Tensor:
    return _to(normal(seed, (STREAM_REDRAW_H, t, attempt), (wl.d,)), wl.torch_dtype)


def redraw_wr_col(wl: Workload, seed: int, c: int, attempt: int) -> torch.Tensor:
    return _to(normal(seed, (STREAM_REDRAW_WR_COL, c, attempt), (wl.E,), 1.0 / math.sqrt(wl.d)),
               wl.torch_dtype)


def draw_w_router(wl: Workload, seed: int = 0) -> torch.Tensor:
    return _to(normal(seed, (STREAM_WR,), (wl.E, wl.d), 1.0 / math.sqrt(wl.d)), wl.torch_dtype)


def draw_bias(wl: Workload, seed: int = 0, hot_bias: float | None = None) -> torch.Tensor | None:
    """Router bias [E] fp32, or None for an unbiased router."""
    E = wl.E
    if wl.bias == "none":
        return None
    if wl.bias == "zipf_3_empty":
        b = np.array([2.0 * math.log(1.0 / (e + 1)) for e in range(E)], np.float64)
        b[[e for e in SKEWED_EMPTY if e < E]] = -np.inf
        return torch.from_numpy(b.astype(np.float32))
    if wl.bias == "gauss_0.5":
        z = normal(seed, (STREAM_BIAS,), (E,))
        return torch.from_numpy((np.float32(0.5) * z).astype(np.float32))
    if wl.bias == "hot16_empty8":
        beta = derived()["many_small_hot_bias"] if hot_bias is None else hot_bias
        b = np.zeros(E, np.float32)
        b[:HOT_EXPERTS] = np.float32(beta)
        b[EMPTY_FROM:] = -np.inf
        return torch.from_numpy(b)
    raise ValueError(wl.bias)


def _expert_stack(wl: Workload, seed: int, stream: int, shape, std: float, experts=None):
    experts = range(wl.E) if experts is None else experts
    experts = list(experts)
    out = np.empty((len(experts),) + tuple(shape), np.float32)

    def one(i):
        out[i] = normal(seed, (stream, experts[i]), shape, std)

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        list(ex.map(one, range(len(experts))))
    return _to(out, wl.torch_dtype)


def draw_w_gate(wl: Workload, seed: int = 0, experts=None) -> torch.Tensor:
    return _expert_stack(wl, seed, STREAM_WG, (wl.F, wl.d), 1.0 / math.sqrt(wl.d), experts)


def draw_w_up(wl: Workload, seed: int = 0, experts=None) -> torch.Tensor:
    return _expert_stack(wl, seed, STREAM_WU, (wl.F, wl.d), 1.0 / math.sqrt(wl.d), experts)


def draw_w_down(wl: Workload, seed: int = 0, experts=None) -> torch.Tensor:
    return _expert_stack(wl, seed, STREAM_WD, (wl.d, wl.F), 1.0 / math.sqrt(wl.F), experts)


@dataclass
class Inputs:
    wl: Workload
    h: torch.Tensor
    w_router: torch.Tensor
    bias: torch.Tensor | None
    w_gate: torch.Tensor | None = None
    w_up: torch.Tensor | None = None
    w_down: torch.Tensor | None = None
    meta: dict = field(default_factory=dict)


def draw(wl: Workload | str, seed: int = 0, weights: bool = True) -> Inputs:
    """All inputs of one workload, before any test-side margin pass."""
    if isinstance(wl, str):
        wl = get(wl)
    inp = Inputs(wl, draw_h(wl, seed), draw_w_router(wl, seed), draw_bias(wl, seed))
    if weights and wl.expert_kind == "swiglu":
        inp.w_gate = draw_w_gate(wl, seed)
        inp.w_up = draw_w_up(wl, seed)
        inp.w_down = draw_w_down(wl, seed)
    return inp
