"""GPU parity of the layer backward against the oracle's gradients.

The oracle differentiates the forward definition in fp64 (pinned by central
differences in test_oracle_pins.py); here every gradient the library returns
is compared with it row by row on seeded inputs whose routing is away from
ties, with the same row-relative bound as the forward output."""
from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import combine_router_gemm_softmax_b200 as M
import oracle as O
import workloads as W
from oracle import cases
from oracle import check as C

from gpu_cases import DEV, DeviceCase, np64, parity_case

pytestmark = pytest.mark.gpu

# ragged rows and half-width column tiles (d = 384), skewed groups with empty
# experts, dropped slots under a capacity (compact and padded layouts), 128
# experts with k = 8, and a Mixtral-shaped layer at a quarter of its width
BWD_CASES = ["small_ragged", "small_skewed", "small_skewed_capacity", "small_skewed_padded", "small_many",
             "mixtral_scaled"]


@functools.lru_cache(maxsize=2)
def _dev(name):
    return DeviceCase(parity_case(name)[0])


def _unpack_w13(dw13, F):
    """Packed rows (block b: 128 gate rows, then the matching 128 up rows) ->
    (dW_gate, dW_up), each [E, F, d]."""
    E, _, d = dw13.shape
    blocks = dw13.reshape(E, F // 128, 2, 128, d)
    return blocks[:, :, 0].reshape(E, F, d), blocks[:, :, 1].reshape(E, F, d)


def _cfg(dc, preact):
    if preact == "recompute":
        return dc.cfg
    wl = dc.wl
    return M.config(wl.T, wl.d, wl.E, wl.k, wl.F, wl.dtype, wl.expert_kind, wl.capacity, wl.gemm_tiles, wl.layout,
                    preact=preact)


def _run(name, seed=0, preact="recompute"):
    dc = _dev(name)
    inp, _ = parity_case(name)
    wl = dc.wl
    cfg = _cfg(dc, preact)
    ws = M.workspace(cfg, M.MOE_OP_LAYER, DEV)
    M.moe_layer_forward(cfg, dc.h, dc.w_router, dc.bias, dc.w13, dc.w_down, ws=ws)
    w13_t, wd_t = M.moe_pack_weights_backward(cfg, dc.w13, dc.w_down)
    dy = W.draw_dy(wl, seed)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    g = M.moe_layer_backward(cfg, dc.h, dc.w_router, dc.w13, w13_t, wd_t, dy.to(DEV), ws,
                             with_bias=dc.bias is not None, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return dc, inp, dy, g


@pytest.mark.parametrize("name,preact", [(n, "recompute") for n in BWD_CASES] +
                         [(n, "save") for n in ("small_ragged", "small_skewed_capacity", "small_skewed_padded",
                                                "small_many")])
def test_layer_backward_matches_oracle(name, preact):
    """preact "save": the forward keeps the gate/up pre-activations (bf16) and
    the backward applies the SwiGLU backward in the dh_mid GEMM's epilogue
    instead of recomputing them; same bounds."""
    dc, inp, dy, g = _run(name, preact=preact)
    wl = dc.wl
    ref = O.layer_backward(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias), wl.k,
                           cases.weights_fn(inp), wl.capacity, cases.as64(dy))
    tol = C.tol_for(wl.dtype)
    # dh per token row, like the forward output; weight gradients per expert
    # matrix against its own largest element (oracle.check.matrix_rel_err)
    errs = {"dh": C.row_rel_err(np64(g["dh"]), ref["dh"]),
            "dw_router": C.matrix_rel_err(np64(g["dw_router"]), ref["dw_router"])}
    dwg, dwu = _unpack_w13(np64(g["dw13"]), wl.F)
    for key, got in (("dw_gate", dwg), ("dw_up", dwu), ("dw_down", np64(g["dw_down"]))):
        errs[key] = max(C.matrix_rel_err(got[e], ref[key][e]) for e in range(wl.E))
    if g["dbias"] is not None:
        errs["dbias"] = C.matrix_rel_err(np64(g["dbias"]), ref["dbias"])
    assert all(v <= tol for v in errs.values()), errs


def test_layer_backward_is_deterministic():
    _, _, _, g1 = _run("small_skewed", seed=1)
    g1 = {k: v.clone() for k, v in g1.items() if v is not None}
    _, _, _, g2 = _run("small_skewed", seed=1)
    for k, v in g1.items():
        assert torch.equal(v.view(torch.int16) if v.dtype == torch.bfloat16 else v.view(torch.int32),
                           g2[k].view(torch.int16) if g2[k].dtype == torch.bfloat16 else g2[k].view(torch.int32)), k


def test_pack_weights_backward_is_a_transpose():
    dc = _dev("small_ragged")
    w13_t, wd_t = M.moe_pack_weights_backward(dc.cfg, dc.w13, dc.w_down)
    torch.cuda.synchronize()
    assert torch.equal(w13_t, dc.w13.transpose(1, 2))
    assert torch.equal(wd_t, dc.w_down.transpose(1, 2))


def test_backward_rejects_unsupported_configs():
    dc = _dev("small_ragged")
    wl = dc.wl
    for kw in (dict(dispatch="gather"), dict(expert_kind="identity")):
        cfg = M.config(wl.T, wl.d, wl.E, wl.k, wl.F, wl.dtype, **kw)
        ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
        with pytest.raises(M.MoeError):
            M.moe_layer_backward(cfg, dc.h, dc.w_router, dc.w13, dc.w13.transpose(1, 2).contiguous(),
                                 dc.w_down.transpose(1, 2).contiguous(), dc.h, ws, ws=ws)


@pytest.mark.parametrize("name", ["mixtral_8x7b", "skewed_capacity", "many_small"])
def test_layer_backward_full_size_sampled(name):
    """Full-size layers, in the configuration bench.py --backward times: dh on
    sampled tokens (row-relative, like the forward), and whole rows of
    dW_gate and dW_up and whole columns of dW_down for two channels of each of
    four experts (the most and the least loaded expert with kept rows and two
    more), each compared against its own largest element at 2e-2 like a
    weight-gradient matrix. A zeroed, sign-flipped or term-missing row fails
    that bound (pinned on the CPU in test_oracle_pins.py)."""
    dc, inp, dy, g = _run(name)
    wl = dc.wl
    _, ref_route = parity_case(name)
    kept = np.asarray(ref_route["kept"])
    live = np.nonzero(kept > 0)[0]
    r = np.random.default_rng(11)
    experts = [int(live[kept[live].argmax()]), int(live[kept[live].argmin()])]
    experts += [int(e) for e in r.choice([e for e in live if e not in experts], size=2, replace=False)]
    chans = [(e, int(f)) for e in experts for f in r.choice(wl.F, size=2, replace=False)]
    tokens = np.sort(r.choice(wl.T, size=32, replace=False))
    probe = O.layer_backward_probe(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias), wl.k,
                                   cases.weights_fn(inp), wl.capacity, cases.as64(dy), tokens, [])
    tol = C.tol_for(wl.dtype)
    assert C.row_rel_err(np64(g["dh"][torch.from_numpy(tokens).to(DEV)]), probe["dh"]) <= tol
    ref = O.layer_backward_channels(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias), wl.k,
                                    cases.weights_fn(inp), wl.capacity, cases.as64(dy), chans)
    errs = {}
    for n, (e, f) in enumerate(chans):
        gate_row = (f // 128) * 256 + f % 128          # packed w13 row of gate channel f
        got = {"dw_gate_rows": np64(g["dw13"][e, gate_row]), "dw_up_rows": np64(g["dw13"][e, gate_row + 128]),
               "dw_down_cols": np64(g["dw_down"][e, :, f])}
        for key, v in got.items():
            assert np.abs(ref[key][n]).max() > 0, (key, e, f)           # a live expert has a non-zero row
            errs[(key, e, f)] = C.vector_rel_err(v, ref[key][n])
    assert max(errs.values()) <= tol, errs


def test_saving_preactivations_leaves_the_forward_unchanged():
    """The forward that keeps its pre-activations returns the same y, bit for
    bit, and the two backward forms agree to bf16 rounding."""
    dc = _dev("small_skewed")
    outs = {}
    for preact in ("recompute", "save"):
        cfg = _cfg(dc, preact)
        outs[preact] = M.moe_layer_forward(cfg, dc.h, dc.w_router, dc.bias, dc.w13, dc.w_down)
    torch.cuda.synchronize()
    assert torch.equal(outs["recompute"].view(torch.int16), outs["save"].view(torch.int16))
    _, _, _, g_r = _run("small_skewed", seed=2)
    g_r = {k: v.clone() for k, v in g_r.items() if v is not None}
    _, _, _, g_s = _run("small_skewed", seed=2, preact="save")
    for key in ("dh", "dw13", "dw_down", "dw_router"):
        a, b = np64(g_r[key]), np64(g_s[key])
        assert np.abs(a - b).max() <= 2e-2 * np.abs(a).max(), key


@pytest.mark.parametrize("name", ["mixtral_8x7b"])
def test_layer_backward_full_size_saved_preact(name):
    """The Mixtral 8x7B layer with saved pre-activations, in the configuration
    bench.py times: dh on sampled tokens and whole dW rows and columns, as
    test_layer_backward_full_size_sampled."""
    dc, inp, dy, g = _run(name, preact="save")
    wl = dc.wl
    r = np.random.default_rng(12)
    e0 = int(r.integers(wl.E))
    chans = [(e0, int(f)) for f in r.choice(wl.F, size=2, replace=False)]
    tokens = np.sort(r.choice(wl.T, size=16, replace=False))
    probe = O.layer_backward_probe(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias), wl.k,
                                   cases.weights_fn(inp), wl.capacity, cases.as64(dy), tokens, [])
    tol = C.tol_for(wl.dtype)
    assert C.row_rel_err(np64(g["dh"][torch.from_numpy(tokens).to(DEV)]), probe["dh"]) <= tol
    ref = O.layer_backward_channels(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias), wl.k,
                                    cases.weights_fn(inp), wl.capacity, cases.as64(dy), chans)
    for n, (e, f) in enumerate(chans):
        gate_row = (f // 128) * 256 + f % 128
        assert C.vector_rel_err(np64(g["dw13"][e, gate_row]), ref["dw_gate_rows"][n]) <= tol
        assert C.vector_rel_err(np64(g["dw13"][e, gate_row + 128]), ref["dw_up_rows"][n]) <= tol
        assert C.vector_rel_err(np64(g["dw_down"][e, :, f]), ref["dw_down_cols"][n]) <= tol
