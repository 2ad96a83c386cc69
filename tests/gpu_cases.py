"""Shared helpers of the GPU parity tests: seeded cases, device copies, and
oracle references (computed on the CPU from the same seeded inputs; nothing
here reads a value back from the CUDA path to build an expectation)."""
from __future__ import annotations

import functools

import torch

import combine_router_gemm_softmax_b200 as M
import oracle as O
import workloads as W
from oracle import cases

DEV = "cuda:0"

# Small problems the oracle finishes in seconds that still span several
# 128-row tiles per expert, a ragged row tail, a half-width column tile
# (d = 384 = 256 + 128) and skewed groups with empty experts.
SMALL = {
    "small_ragged": W.get("mixtral_scaled").with_(
        name="small_ragged", T=1000, d=384, E=8, k=2, F=256, bias="gauss_0.5"),
    "small_skewed": W.get("skewed").with_(
        name="small_skewed", T=777, d=256, E=40, k=4, F=384),
    "small_skewed_capacity": W.get("skewed").with_(
        name="small_skewed_capacity", T=777, d=256, E=40, k=4, F=384,
        capacity=W.capacity_factor_cap(777, 4, 40)),
    "small_many": W.get("many_small").with_(
        name="small_many", T=640, d=256, E=128, k=8, F=256),
    # CTA-pair GEMM tiles: 256-row tiles with a ragged last tile per expert
    # (one CTA of the pair may have no valid rows), and d = 384 gives a
    # half-empty second column tile in the down projection
    "small_pair": W.get("mixtral_scaled").with_(
        name="small_pair", T=2100, d=384, E=4, k=2, F=384, bias="gauss_0.5", gemm_tiles="pair"),
    "small_pair_wide": W.get("mixtral_scaled").with_(
        name="small_pair_wide", T=2100, d=2048, E=4, k=2, F=640, bias="gauss_0.5", gemm_tiles="pair"),
    "small_skewed_pair": W.get("skewed").with_(
        name="small_skewed_pair", T=777, d=256, E=40, k=4, F=384, gemm_tiles="pair"),
    # padded capacity layout: capacity 97 is not a multiple of the 128-row
    # tile, so every expert's last tile is ragged and mixes kept and padding rows
    "small_skewed_padded": W.get("skewed").with_(
        name="small_skewed_padded", T=777, d=256, E=40, k=4, F=384,
        capacity=W.capacity_factor_cap(777, 4, 40), layout="padded"),
}


def workload(name):
    return SMALL[name] if name in SMALL else W.get(name)


def cfg_for(wl) -> M.MoeConfig:
    return M.config(wl.T, wl.d, wl.E, wl.k, wl.F, wl.dtype, wl.expert_kind, wl.capacity, wl.gemm_tiles, wl.layout)


@functools.lru_cache(maxsize=3)
def parity_case(name, seed=0):
    """Margin-passed inputs plus the oracle's routing and dispatch metadata."""
    wl = workload(name)
    inp = cases.parity_inputs(wl, seed)
    h64 = cases.as64(inp.h)
    idx, gate, logits, nan_row = O.route(h64, cases.as64(inp.w_router), cases.as64(inp.bias), wl.k)
    meta = O.dispatch_meta(idx, wl.E, wl.capacity)
    return inp, dict(idx=idx, gate=gate, logits=logits, nan_row=nan_row, **meta)


def oracle_y(name, tokens=None, seed=0):
    inp, ref = parity_case(name, seed)
    wl = inp.wl
    weights = cases.weights_fn(inp) if wl.expert_kind == "swiglu" else None
    return O.combine(cases.as64(inp.h), ref["idx"], ref["gate"], ref["dest_row"], wl.expert_kind, weights, tokens)


class DeviceCase:
    """Device copies of one case's inputs (weights packed for the grouped FFN)."""

    def __init__(self, inp):
        wl = inp.wl
        self.wl = wl
        self.cfg = cfg_for(wl)
        self.h = inp.h.to(DEV)
        self.w_router = inp.w_router.to(DEV)
        self.bias = None if inp.bias is None else inp.bias.to(DEV)
        self.w13 = self.w_down = None
        if wl.expert_kind == "swiglu":
            wg, wu = inp.w_gate.to(DEV), inp.w_up.to(DEV)
            self.w13 = M.moe_pack_weights(self.cfg, wg, wu)
            del wg, wu
            self.w_down = inp.w_down.to(DEV)
        self.status = torch.zeros(1, dtype=torch.int32, device=DEV)

    def layer(self, **kw):
        out = dict(topk_idx=torch.empty((self.wl.T, self.wl.k), dtype=torch.int32, device=DEV),
                   topk_gate=torch.empty((self.wl.T, self.wl.k), dtype=torch.float32, device=DEV),
                   routed_counts=torch.empty(self.wl.E, dtype=torch.int32, device=DEV),
                   counts=torch.empty(self.wl.E, dtype=torch.int32, device=DEV))
        y = M.moe_layer_forward(self.cfg, self.h, self.w_router, self.bias, self.w13, self.w_down,
                                status=self.status, **out, **kw)
        out["y"] = y
        return out


def np_(t):
    return t.detach().cpu().numpy()


def np64(t):
    return t.detach().cpu().double().numpy()
