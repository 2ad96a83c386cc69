"""Parity cases: seeded inputs with every token's top-k scores kept apart
(test infrastructure only).

The margin pass follows "How Does Mixture-of-Experts Routing Affect LLM
Repeatability?" -- "Boundary Matters": a token whose k-th and (k+1)-th scores
are close can change its expert set under a tiny numerical change. Routing
parity is required bit-exact, so every token's k+1 largest scores are kept at
least MIN_GAP apart (this also fixes the slot order). Offending token rows are
redrawn from their own stream; for identity-tagged tokens (whose rows are
fixed) the router column the token reads is redrawn instead.
"""
from __future__ import annotations

import numpy as np
import torch

import workloads as W
from . import moe_oracle as O

MIN_GAP = 1e-3


def as64(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().double().numpy()
    return np.asarray(x, np.float64)


def enforce_margin(inp: W.Inputs, seed: int = 0, min_gap: float = MIN_GAP, max_attempts: int = 200):
    wl = inp.wl
    bias = as64(inp.bias)
    redrawn = 0
    for attempt in range(1, max_attempts + 1):
        s = O.router_logits(as64(inp.h), as64(inp.w_router), bias)
        bad = np.nonzero(O.min_adjacent_gap(s, wl.k) < min_gap)[0]
        if bad.size == 0:
            inp.meta["margin_redraws"] = redrawn
            inp.meta["min_gap"] = float(O.min_adjacent_gap(s, wl.k).min()) if wl.T else None
            return inp
        redrawn += len(bad)
        if wl.tagged:
            for c in sorted(set(int(t) % wl.d for t in bad)):
                inp.w_router[:, c] = W.redraw_wr_col(wl, seed, c, attempt)
        else:
            for t in bad:
                inp.h[int(t)] = W.redraw_h_row(wl, seed, int(t), attempt)
    raise RuntimeError(f"margin pass did not converge for {wl.name}")


def parity_inputs(wl, seed: int = 0, weights: bool = True) -> W.Inputs:
    """Seeded inputs of a workload after the margin pass."""
    if isinstance(wl, str):
        wl = W.get(wl)
    return enforce_margin(W.draw(wl, seed, weights), seed)


def weights_fn(inp: W.Inputs):
    """Per-expert fp64 weights for the oracle's SwiGLU expert."""
    def f(e):
        return as64(inp.w_gate[e]), as64(inp.w_up[e]), as64(inp.w_down[e])
    return f


def sample_tokens(idx, dest_row, n, seed=0):
    """A seeded token sample covering the first and last kept token of every
    expert segment, padded with random tokens to n (sorted, unique)."""
    idx = np.asarray(idx)
    dest_row = np.asarray(dest_row)
    T = idx.shape[0]
    pick = set()
    for e in np.unique(idx[dest_row >= 0]):
        tt = np.nonzero(((idx == e) & (dest_row >= 0)).any(axis=1))[0]
        pick.add(int(tt[0]))
        pick.add(int(tt[-1]))
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(99,))))
    rest = g.permutation(T)
    for t in rest:
        if len(pick) >= n:
            break
        pick.add(int(t))
    return np.array(sorted(pick), np.int64)
