"""Parity of the CUDA path with the CPU oracle, called through the C ABI.

Bars: routing indices, counts, offsets, drop decisions, dest_row/perm_src and
the permuted rows are bit-exact; layer outputs within the per-row relative
bound (2e-2 for bf16 storage, 1e-4 for fp32). Gates here are compared with
the oracle's gates computed from the oracle's own fp64 scores, so the bound
is derived from the score tolerance: |g - g_ref| <= g_ref (2 ds_max + 1e-5)
+ 1e-7 with ds_max = 1e-4 + 1e-4 |s| over the token's picks (about 1e-3
relative for scores near 3; oracle.check.gate_bound). The 1e-5 relative bar
on the kernel's gate arithmetic itself, given identical scores, is checked
at full size in test_gpu_dispatch_full.py.
"""
import numpy as np
import pytest
import torch

import combine_router_gemm_softmax_b200 as M
import oracle as O
import workloads as W
from oracle import cases
from oracle import check as C
from oracle import mxfp8 as X

from gpu_cases import DEV, DeviceCase, cfg_for, np64, np_, oracle_y, parity_case

pytestmark = pytest.mark.gpu

LAYER_CASES = ["tiny_f32", "tiny_f32_tagged", "small_ragged", "small_skewed", "small_skewed_capacity",
               "small_skewed_padded", "small_many", "small_pair", "small_pair_wide", "small_skewed_pair",
               "mixtral_scaled", "skewed", "skewed_capacity", "skewed_capacity_padded", "many_small",
               "many_small_identity", "mixtral_8x7b"]
FULL_ORACLE = {"tiny_f32", "tiny_f32_tagged", "small_ragged", "small_skewed", "small_skewed_capacity",
               "small_skewed_padded", "small_many", "small_pair", "small_pair_wide", "small_skewed_pair",
               "many_small_identity"}


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    torch.cuda.set_device(0)
    M.lib()


_dev_cache = {}


def dev_case(name):
    if name not in _dev_cache:
        _dev_cache.clear()
        torch.cuda.empty_cache()
        inp, _ = parity_case(name)
        _dev_cache[name] = DeviceCase(inp)
    return _dev_cache[name]


def gate_close(g, ref, logits_ref, idx_ref):
    return C.gates_match(g, ref, logits_ref, idx_ref)


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("name", ["tiny_f32", "small_ragged", "small_many", "mixtral_scaled", "skewed",
                                  "many_small", "mixtral_8x7b"])
def test_route_matches_oracle(name):
    dc = dev_case(name)
    _, ref = parity_case(name)
    wl = dc.wl
    logits = torch.empty((wl.T, wl.E), dtype=torch.float32, device=DEV)
    dc.status.zero_()
    idx, gate = M.moe_route(dc.cfg, dc.h, dc.w_router, dc.bias, logits_out=logits, status=dc.status)
    torch.cuda.synchronize()
    assert np.array_equal(np_(idx), ref["idx"])
    assert C.logits_match(np64(logits), ref["logits"])
    assert gate_close(np64(gate), ref["gate"], ref["logits"], ref["idx"])
    assert int(dc.status.item()) == 0


def _int_valued(T, d, E, seed, lo=-2, hi=3):
    r = np.random.default_rng(seed)
    return (r.integers(lo, hi, size=(T, d)).astype(np.float32), r.integers(lo, hi, size=(E, d)).astype(np.float32))


@pytest.mark.parametrize("dtype,T,d,E,k", [("bf16", 300, 128, 8, 2), ("bf16", 129, 256, 64, 6),
                                           ("bf16", 200, 128, 128, 8), ("bf16", 150, 128, 100, 4),
                                           ("bf16", 140, 128, 256, 8), ("f32", 77, 32, 6, 3)])
def test_route_exact_ties_go_to_lowest_index(dtype, T, d, E, k):
    """Small integers make every score exact in fp32 and fp64, so planted ties
    are real ties on both sides."""
    h, w = _int_valued(T, d, E, seed=T + E)
    w[E // 2] = w[0]                      # expert E/2 always ties expert 0
    w[E - 1] = w[1]
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    cfg = M.config(T, d, E, k, 128, dtype)
    ht, wt = torch.from_numpy(h).to(tdt), torch.from_numpy(w).to(tdt)
    idx, gate = M.moe_route(cfg, ht.to(DEV), wt.to(DEV))
    ref_idx, ref_gate, ref_s, _ = O.route(h.astype(np.float64), w.astype(np.float64), None, k)
    assert np.array_equal(np_(idx), ref_idx)
    assert gate_close(np64(gate), ref_gate, ref_s, ref_idx)


def test_route_nan_and_all_minus_inf():
    T, d, E, k = 130, 128, 16, 4
    h, w = _int_valued(T, d, E, seed=5)
    h[3, 7] = np.nan                      # NaN scores for every expert of token 3
    bias = np.zeros(E, np.float32)
    bias[E - 3:] = -np.inf
    hb = torch.from_numpy(h).to(torch.bfloat16)
    cfg = M.config(T, d, E, k, 128)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx, gate = M.moe_route(cfg, hb.to(DEV), torch.from_numpy(w).to(torch.bfloat16).to(DEV),
                            torch.from_numpy(bias).to(DEV), status=status)
    ref_idx, ref_gate, ref_s, nan_row = O.route(hb.double().numpy(), w.astype(np.float64), bias.astype(np.float64),
                                                k)
    assert nan_row[3]
    assert np.array_equal(np_(idx), ref_idx)
    assert np_(idx)[3].tolist() == [0, 1, 2, 3]
    assert np.all(np64(gate)[3] == 0)
    assert gate_close(np64(gate), ref_gate, ref_s, ref_idx)
    assert int(status.item()) & M.MOE_STATUS_NAN_LOGIT
    # all experts at -inf: picks 0..k-1, gate 0
    cfg2 = M.config(4, d, E, k, 128)
    idx2, gate2 = M.moe_route(cfg2, hb[:4].to(DEV), torch.from_numpy(w).to(torch.bfloat16).to(DEV),
                              torch.full((E,), -float("inf"), device=DEV))
    assert np_(idx2).tolist() == [[0, 1, 2, 3]] * 4
    assert np.all(np64(gate2) == 0)


def test_route_batch_invariance():
    """A token's scores do not depend on which other tokens share the batch."""
    dc = dev_case("small_ragged")
    wl = dc.wl
    full = torch.empty((wl.T, wl.E), dtype=torch.float32, device=DEV)
    M.moe_route(dc.cfg, dc.h, dc.w_router, dc.bias, logits_out=full)
    for lo, hi in ((0, 1), (5, 300), (517, 1000)):
        sub = cfg_for(wl.with_(T=hi - lo))
        part = torch.empty((hi - lo, wl.E), dtype=torch.float32, device=DEV)
        M.moe_route(sub, dc.h[lo:hi].contiguous(), dc.w_router, dc.bias, logits_out=part)
        assert torch.equal(part, full[lo:hi])
    perm = torch.randperm(wl.T, generator=torch.Generator().manual_seed(0)).to(DEV)
    shuffled = torch.empty_like(full)
    M.moe_route(dc.cfg, dc.h[perm].contiguous(), dc.w_router, dc.bias, logits_out=shuffled)
    assert torch.equal(shuffled, full[perm])


# ------------------------------------------------------------------ permute
def _permute_check(T, d, E, k, idx, cap=-1, dtype="bf16", seed=0):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    h = torch.from_numpy(np.random.default_rng(seed).standard_normal((T, d)).astype(np.float32)).to(tdt)
    cfg = M.config(T, d, E, k, 128, dtype, capacity=cap)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = M.moe_permute(cfg, h.to(DEV), torch.from_numpy(np.asarray(idx, np.int32)).to(DEV), status=status)
    torch.cuda.synchronize()
    ref = O.dispatch_meta(np.asarray(idx), E, cap)
    n = int(ref["offsets"][-1])
    assert np_(out["routed_counts"]).tolist() == ref["routed"].tolist()
    assert np_(out["counts"]).tolist() == ref["kept"].tolist()
    assert np_(out["offsets"]).tolist() == ref["offsets"].tolist()
    assert np.array_equal(np_(out["dest_row"]), ref["dest_row"])
    assert np.array_equal(np_(out["perm_src"])[:n], ref["perm_src"])
    xp = out["x_perm"][:n].cpu()
    want = h[torch.from_numpy(ref["perm_src"])]
    bits = torch.int16 if dtype == "bf16" else torch.int32
    assert torch.equal(xp.view(bits), want.view(bits))
    bad = bool(int(status.item()) & M.MOE_STATUS_BAD_ROUTE)
    assert bad == ref["bad_route"]
    return out, ref


@pytest.mark.parametrize("which", ["map1", "map2"])
def test_permute_worked_maps(golden_dir, which):
    """The two four-rank routing maps printed on the dispatch page, 2 KiB rows."""
    import json
    import os
    g = json.load(open(os.path.join(golden_dir, "dispatch_worked_maps.json")))
    m = g["maps"][which]
    idx = [[m["expert_of_token"][t]] for t in g["tokens"]]
    out, _ = _permute_check(8, g["row_bytes"] // 2, 4, 1, idx)
    assert np_(out["counts"]).tolist() == m["counts_printed"]
    toks = g["tokens"]
    off = np_(out["offsets"])
    ps = np_(out["perm_src"])
    assert [[toks[t] for t in ps[off[e]:off[e + 1]]] for e in range(4)] == m["expected_grouping_by_expert"]


def _routes(kind, T, E, k, seed=0):
    r = np.random.default_rng(seed)
    if kind == "random":
        return np.stack([r.permutation(E)[:k] for _ in range(T)])
    if kind == "all_to_one":                        # every token's first pick is expert 0
        rows = [np.concatenate([[0], r.permutation(np.arange(1, E))[:k - 1]]) for _ in range(T)]
        return np.stack(rows)
    if kind == "empty_experts":                     # only even experts are used
        return np.stack([r.permutation(np.arange(0, E, 2))[:k] for _ in range(T)])
    if kind == "bad":
        idx = np.stack([r.permutation(E)[:k] for _ in range(T)])
        idx[3, 1] = E + 5
        idx[10, 0] = -1
        idx[20, 1] = idx[20, 0]
        return idx
    raise ValueError(kind)


@pytest.mark.parametrize("kind,T,E,k,cap", [
    ("random", 1000, 8, 2, -1), ("random", 4097, 64, 6, -1), ("all_to_one", 700, 16, 3, -1),
    ("empty_experts", 513, 32, 4, -1), ("all_to_one", 700, 16, 3, 100), ("random", 999, 40, 4, 50),
    ("bad", 300, 8, 2, -1), ("random", 1, 8, 2, -1), ("random", 128, 256, 8, -1), ("random", 300, 4, 4, 0),
    # E * ceil(T/128) > 8192: chunk bases come from the separate scan kernel
    ("random", 8320, 256, 2, -1), ("all_to_one", 8320, 256, 3, 70)])
def test_permute_injected_routes(kind, T, E, k, cap):
    _permute_check(T, 256, E, k, _routes(kind, T, E, k), cap)


def _permute_check_padded(T, d, E, k, idx, cap, dtype="bf16", seed=0):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    h = torch.from_numpy(np.random.default_rng(seed).standard_normal((T, d)).astype(np.float32)).to(tdt)
    cfg = M.config(T, d, E, k, 128, dtype, capacity=cap, layout="padded")
    assert M.perm_rows(cfg) == E * cap
    # stale bytes in the output buffers must not survive: padding rows are written
    out = dict(routed_counts=torch.full((E,), -7, dtype=torch.int32, device=DEV),
               counts=torch.full((E,), -7, dtype=torch.int32, device=DEV),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=DEV),
               dest_row=torch.full((T, k), -7, dtype=torch.int32, device=DEV),
               perm_src=torch.full((max(E * cap, 1),), 12345, dtype=torch.int32, device=DEV),
               x_perm=torch.full((max(E * cap, 1), d), 3.0, dtype=tdt, device=DEV))
    M.moe_permute(cfg, h.to(DEV), torch.from_numpy(np.asarray(idx, np.int32)).to(DEV), out=out)
    torch.cuda.synchronize()
    ref = O.dispatch_meta_padded(np.asarray(idx), E, cap)
    assert np_(out["counts"]).tolist() == ref["kept"].tolist()
    assert np_(out["routed_counts"]).tolist() == ref["routed"].tolist()
    assert np_(out["offsets"]).tolist() == ref["offsets"].tolist()
    assert np.array_equal(np_(out["dest_row"]), ref["dest_row"])
    ps = np_(out["perm_src"])[:E * cap]
    assert np.array_equal(ps, ref["perm_src"])
    xp = out["x_perm"][:E * cap].cpu()
    bits = torch.int16 if dtype == "bf16" else torch.int32
    kept_rows = torch.from_numpy(np.nonzero(ref["perm_src"] >= 0)[0])
    pad_rows = torch.from_numpy(np.nonzero(ref["perm_src"] < 0)[0])
    assert torch.equal(xp[kept_rows].view(bits), h[torch.from_numpy(ref["perm_src"][ref["perm_src"] >= 0])].view(bits))
    assert bool((xp[pad_rows] == 0).all())


@pytest.mark.parametrize("kind,T,E,k,cap", [
    ("random", 999, 40, 4, 97), ("all_to_one", 700, 16, 3, 100), ("empty_experts", 513, 32, 4, 64),
    ("random", 300, 4, 4, 0), ("random", 8320, 256, 3, 70), ("random", 200, 8, 2, 400)])
def test_permute_padded_layout(kind, T, E, k, cap):
    """Padded capacity layout: offsets e*C, kept rows at e*C + rank, padding
    rows zero with perm_src -1 (checked against the oracle's padded layout)."""
    _permute_check_padded(T, 256, E, k, _routes(kind, T, E, k), cap)


def test_permute_padded_fp32_and_zero_tokens():
    _permute_check_padded(100, 36, 5, 2, _routes("random", 100, 5, 2), 30, dtype="f32")
    _permute_check_padded(0, 128, 4, 2, np.zeros((0, 2), np.int32), 8)


def test_layer_padded_equals_compact():
    """The padded arm computes the padding rows too but returns the same y,
    bit for bit, as the compact capacity layout."""
    a, b = dev_case("small_skewed_capacity"), dev_case("small_skewed_padded")
    assert (a.wl.T, a.wl.d, a.wl.E, a.wl.k, a.wl.F, a.wl.capacity) == (b.wl.T, b.wl.d, b.wl.E, b.wl.k, b.wl.F,
                                                                        b.wl.capacity)
    ya, yb = a.layer()["y"], b.layer()["y"]
    torch.cuda.synchronize()
    assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))


@pytest.mark.parametrize("name", ["small_ragged", "small_skewed", "small_many", "mixtral_scaled"])
def test_layer_gather_dispatch_equals_copy(name):
    """GEMM1 gathering its rows from h through the permutation gives the same
    y, bit for bit, as the row copy into x_perm followed by tiled loads."""
    dc = dev_case(name)
    wl = dc.wl
    base = dict(T=wl.T, d=wl.d, E=wl.E, k=wl.k, d_ff=wl.F, dtype=wl.dtype, expert_kind=wl.expert_kind,
                capacity=wl.capacity)
    ys = {}
    for mode in ("copy", "gather"):
        cfg = M.config(**base, dispatch=mode)
        ys[mode] = M.moe_layer_forward(cfg, dc.h, dc.w_router, dc.bias, dc.w13, dc.w_down)
    torch.cuda.synchronize()
    assert torch.equal(ys["copy"].view(torch.int16), ys["gather"].view(torch.int16))


@pytest.mark.parametrize("name", ["small_pair", "small_pair_wide", "small_skewed_pair"])
def test_layer_pair_tiles_equal_single(name):
    """256-row CTA-pair tiles accumulate every output over K in the same order
    as the single-CTA 128-row tiles, so y is the same bit for bit; the cases
    have ragged last pair tiles in which one CTA of the pair has no rows and
    32-row blocks cut by an expert's end."""
    dc = dev_case(name)
    wl = dc.wl
    base = dict(T=wl.T, d=wl.d, E=wl.E, k=wl.k, d_ff=wl.F, dtype=wl.dtype, expert_kind=wl.expert_kind,
                capacity=wl.capacity)
    ys = {}
    for tiles in ("single", "pair"):
        cfg = M.config(**base, gemm_tiles=tiles)
        ys[tiles] = M.moe_layer_forward(cfg, dc.h, dc.w_router, dc.bias, dc.w13, dc.w_down)
    torch.cuda.synchronize()
    assert torch.equal(ys["single"].view(torch.int16), ys["pair"].view(torch.int16))


def test_config_layout_checks():
    with pytest.raises(M.MoeError):
        M.moe_layer_forward(M.config(64, 128, 4, 2, 128, layout="padded"),  # padded needs a capacity
                            torch.zeros((64, 128), dtype=torch.bfloat16, device=DEV),
                            torch.zeros((4, 128), dtype=torch.bfloat16, device=DEV),
                            w13_packed=torch.zeros((4, 256, 128), dtype=torch.bfloat16, device=DEV),
                            w_down=torch.zeros((4, 128, 128), dtype=torch.bfloat16, device=DEV),
                            ws=torch.zeros(1 << 20, dtype=torch.uint8, device=DEV))


def test_permute_fp32_rows():
    _permute_check(100, 36, 5, 2, _routes("random", 100, 5, 2), dtype="f32")


@pytest.mark.parametrize("T,d,E,k,cap,dtype", [
    (301, 6144, 8, 2, -1, "bf16"),    # 12 KB rows: an 8 KB piece and a 4 KB piece
    (257, 8192, 16, 4, 40, "bf16"),   # 16 KB rows, two full pieces, with drops
    (129, 3000, 8, 3, -1, "f32"),     # 12000-byte rows: 8192 + 3808
])
def test_permute_multi_piece_rows(T, d, E, k, cap, dtype):
    """Rows longer than one bulk transfer move in pieces; every kept row still
    lands bit for bit, including the ragged last piece."""
    _permute_check(T, d, E, k, _routes("random", T, E, k, seed=d), cap, dtype=dtype)


def test_permute_zero_tokens():
    cfg = M.config(0, 128, 8, 2, 128)
    out = M.moe_permute(cfg, torch.empty((0, 128), dtype=torch.bfloat16, device=DEV),
                        torch.empty((0, 2), dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert np_(out["offsets"]).tolist() == [0] * 9
    assert np_(out["routed_counts"]).tolist() == [0] * 8


# ------------------------------------------------------------------ grouped FFN (fed by the oracle's dispatch)
@pytest.mark.parametrize("name", ["tiny_f32", "small_ragged", "small_skewed", "small_many", "small_pair",
                                  "small_pair_wide", "mixtral_scaled"])
def test_grouped_ffn_matches_oracle(name):
    dc = dev_case(name)
    inp, ref = parity_case(name)
    wl = dc.wl
    A = wl.T * wl.k
    x_perm = torch.zeros((A, wl.d), dtype=wl.torch_dtype)
    n = int(ref["offsets"][-1])
    x_perm[:n] = inp.h[ref["perm_src"]]
    offsets = torch.from_numpy(ref["offsets"].astype(np.int32))
    y_perm = M.moe_grouped_ffn(dc.cfg, x_perm.to(DEV), offsets.to(DEV), dc.w13, dc.w_down, status=dc.status)
    torch.cuda.synchronize()
    got = np64(y_perm[:n])
    rows = np.linspace(0, n - 1, min(n, 1536)).astype(np.int64)
    want = np.zeros((len(rows), wl.d))
    xs = cases.as64(x_perm)
    wf = cases.weights_fn(inp)
    for e in range(wl.E):
        sel = np.nonzero((rows >= ref["offsets"][e]) & (rows < ref["offsets"][e + 1]))[0]
        if sel.size:
            want[sel] = O.swiglu_expert(xs[rows[sel]], *wf(e))
    assert C.row_rel_err(got[rows], want) <= C.tol_for(wl.dtype)


@pytest.mark.parametrize("kind", ["identity", "scale"])
def test_combine_matches_oracle(kind):
    """Combine alone, fed y_perm = f_e(x_perm) for the identity and scale
    experts built on the CPU from the oracle's dispatch."""
    name = "small_skewed_capacity"
    inp, ref = parity_case(name)
    wl = inp.wl.with_(expert_kind=kind)
    A = wl.T * wl.k
    n = int(ref["offsets"][-1])
    h64 = cases.as64(inp.h)
    y_perm = np.zeros((A, wl.d))
    for e in range(wl.E):
        a, b = ref["offsets"][e], ref["offsets"][e + 1]
        y_perm[a:b] = O.expert_apply(kind, e, h64[ref["perm_src"][a:b]])
    cfg = cfg_for(wl)
    y = M.moe_unpermute_combine(cfg, torch.from_numpy(y_perm).to(torch.bfloat16).to(DEV),
                                torch.from_numpy(ref["dest_row"].astype(np.int32)).to(DEV),
                                torch.from_numpy(ref["gate"].astype(np.float32)).to(DEV))
    want = O.combine(h64, ref["idx"], ref["gate"], ref["dest_row"], kind)
    assert C.row_rel_err(np64(y), want) <= C.TOL_BF16
    assert n < A                                   # this case drops assignments


# ------------------------------------------------------------------ whole layer
@pytest.mark.parametrize("name", LAYER_CASES)
def test_layer_matches_oracle(name):
    dc = dev_case(name)
    inp, ref = parity_case(name)
    wl = dc.wl
    dc.status.zero_()
    out = dc.layer()
    torch.cuda.synchronize()
    assert np.array_equal(np_(out["topk_idx"]), ref["idx"])
    assert gate_close(np64(out["topk_gate"]), ref["gate"], ref["logits"], ref["idx"])
    assert np_(out["routed_counts"]).tolist() == ref["routed"].tolist()
    assert np_(out["counts"]).tolist() == ref["kept"].tolist()
    assert int(dc.status.item()) == 0
    if name in FULL_ORACLE:
        tokens = None
    else:
        tokens = cases.sample_tokens(ref["idx"], ref["dest_row"], 1024)
    want = oracle_y(name, tokens)
    got = np64(out["y"]) if tokens is None else np64(out["y"][torch.from_numpy(tokens).to(DEV)])
    err = C.row_rel_err(got, want)
    assert err <= C.tol_for(wl.dtype), err


def test_layer_identity_tagged_closed_form():
    """Identity-tagged tokens with scale experts: every output row is zero
    except position t mod d, which holds (t+1) * sum_j g_j (e_j + 1)."""
    dc = dev_case("tiny_f32_tagged")
    out = dc.layer()
    y = np64(out["y"])
    idx, g = np_(out["topk_idx"]), np64(out["topk_gate"])
    for t in range(dc.wl.T):
        c = t % dc.wl.d
        row = y[t].copy()
        assert row[c] == pytest.approx((t + 1) * float((g[t] * (idx[t] + 1)).sum()), rel=1e-5)
        row[c] = 0
        assert not row.any()


def test_layer_is_deterministic():
    dc = dev_case("small_skewed_capacity")
    a = dc.layer()["y"].clone()
    b = dc.layer()["y"]
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("T,E,k,cap", [(0, 8, 2, -1), (1, 8, 2, -1), (129, 1, 1, -1), (200, 8, 8, -1),
                                       (300, 8, 2, 0)])
def test_layer_edge_cases(T, E, k, cap):
    wl = W.Workload("edge", T=T, d=128, E=E, k=k, F=128, bias="none", capacity=cap)
    inp = W.draw(wl, 3)
    if T:
        inp = cases.enforce_margin(inp, 3)
    dc = DeviceCase(inp)
    out = dc.layer()
    torch.cuda.synchronize()
    if T == 0:
        assert out["y"].numel() == 0
        return
    ref = O.layer_forward(cases.as64(inp.h), cases.as64(inp.w_router), None, k, "swiglu", cases.weights_fn(inp),
                          cap)
    assert np.array_equal(np_(out["topk_idx"]), ref["idx"])
    assert C.row_rel_err(np64(out["y"]), ref["y"]) <= C.TOL_BF16
    if cap == 0:
        assert not out["y"].any()


def test_workspace_guard_bytes_untouched():
    """Bytes past the workspace the library asked for stay untouched."""
    dc = dev_case("small_ragged")
    need = M.moe_workspace_size(dc.cfg, M.MOE_OP_LAYER)
    ws = torch.full((need + 4096,), 0x5A, dtype=torch.uint8, device=DEV)
    dc.layer(ws=ws[:need])
    torch.cuda.synchronize()
    assert bool((ws[need:] == 0x5A).all())


def test_layer_replays_from_a_cuda_graph():
    """The whole layer is stream-ordered with no host synchronisation, so it
    captures into a CUDA graph; replays match eager runs bit for bit, also
    after new tokens are copied into the captured input buffer."""
    dc = dev_case("small_skewed_capacity")
    wl = dc.wl
    h_static = dc.h.clone()
    y_static = torch.empty((wl.T, wl.d), dtype=wl.torch_dtype, device=DEV)
    ws = M.workspace(dc.cfg, M.MOE_OP_LAYER, DEV)

    def run(h, y):
        return M.moe_layer_forward(dc.cfg, h, dc.w_router, dc.bias, dc.w13, dc.w_down, y=y, ws=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(h_static, y_static)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run(h_static, y_static)
    for h_new in (dc.h, dc.h.flip(0).contiguous()):
        h_static.copy_(h_new)
        graph.replay()
        eager = run(h_new.clone(), torch.empty_like(y_static))
        torch.cuda.synchronize()
        assert torch.equal(y_static.view(torch.int16), eager.view(torch.int16))


def test_layer_stage_events_time_the_same_layer():
    """moe_layer_forward_timed gives the same output bit for bit and records
    its 5 events in stage order on the launching stream."""
    dc = dev_case("small_skewed")
    wl = dc.wl
    ws = M.workspace(dc.cfg, M.MOE_OP_LAYER, DEV)
    y0 = M.moe_layer_forward(dc.cfg, dc.h, dc.w_router, dc.bias, dc.w13, dc.w_down, ws=ws)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    y1 = M.moe_layer_forward(dc.cfg, dc.h, dc.w_router, dc.bias, dc.w13, dc.w_down, ws=ws, stage_events=ev)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    parts = [ev[i].elapsed_time(ev[i + 1]) for i in range(4)]
    assert all(p >= 0 for p in parts)
    assert parts[2] > 0  # the expert stage did work between its two events
    assert abs(sum(parts) - ev[0].elapsed_time(ev[4])) < 1e-2
    # NULL entries are skipped
    y2 = M.moe_layer_forward(dc.cfg, dc.h, dc.w_router, dc.bias, dc.w13, dc.w_down, ws=ws,
                             stage_events=[None, ev[1], None, None, ev[4]])
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y2.view(torch.int16))
    with pytest.raises(ValueError):
        M.moe_layer_forward(dc.cfg, dc.h, dc.w_router, dc.bias, dc.w13, dc.w_down, ws=ws, stage_events=ev[:3])


@pytest.mark.parametrize("name,kw", [("small_ragged", {}), ("mixtral_scaled", {}),
                                     ("small_ragged", dict(capacity=150)), ("small_ragged", dict(k=1)),
                                     ("mixtral_8x7b", {})])
def test_layer_fused_combine_equals_separate(name, kw):
    """The combine done by the down projection's epilogue (k <= 2) gives y bit
    for bit equal to the separate combine kernel, with every slot kept, with
    capacity drops (tokens keeping one slot or none) and with k = 1; y_perm,
    which the backward reads, is written the same way."""
    dc = dev_case(name)
    wl = dc.wl.with_(**kw) if kw else dc.wl
    h = dc.h
    if "k" in kw:
        inp = W.draw(wl, 5)
        inp = cases.enforce_margin(inp, 5)
        dc = DeviceCase(inp)
        h = dc.h
    base = dict(T=wl.T, d=wl.d, E=wl.E, k=wl.k, d_ff=wl.F, dtype=wl.dtype, expert_kind=wl.expert_kind,
                capacity=wl.capacity)
    ys = {}
    for mode in ("separate", "fused"):
        cfg = M.config(**base, combine=mode)
        ws = M.workspace(cfg, M.MOE_OP_LAYER, DEV)
        y = torch.full((wl.T, wl.d), 7.0, dtype=torch.bfloat16, device=DEV)      # stale bytes must not survive
        ys[mode] = M.moe_layer_forward(cfg, h, dc.w_router, dc.bias, dc.w13, dc.w_down, y=y, ws=ws)
        torch.cuda.synchronize()
    assert torch.equal(ys["separate"].view(torch.int16), ys["fused"].view(torch.int16))
    if wl.capacity >= 0:
        cfg = M.config(**base)
        counts = torch.empty(wl.E, dtype=torch.int32, device=DEV)
        M.moe_layer_forward(cfg, h, dc.w_router, dc.bias, dc.w13, dc.w_down, counts=counts)
        assert int(counts.sum().item()) < wl.T * wl.k                            # drops happened


def test_fused_combine_rejected_where_it_does_not_apply():
    for kw in (dict(k=4, E=8), dict(gemm_tiles="pair"), dict(expert_kind="identity"), dict(precision="mxfp8")):
        base = dict(T=64, d=128, E=4, k=2, d_ff=128)
        base.update(kw)
        cfg = M.config(**base, combine="fused")
        assert M.moe_workspace_size(cfg, M.MOE_OP_LAYER) == 0, kw


@pytest.mark.parametrize("precision", ["bf16", "mxfp8"])
def test_grouped_ffn_expert_boundaries_inside_tiles(precision):
    """Experts whose row counts fall on and next to the 32-row blocks the
    epilogue stores whole (0, 1, 31, 32, 33, 64, 96, 128, 160, 255 rows):
    every row of every expert equals the oracle's expert output, and the rows
    past the last expert are left as they were."""
    counts = [32, 64, 96, 128, 31, 33, 0, 1, 160, 255]
    E, d, F, k = len(counts), 256, 256, 2
    n = sum(counts)
    T = n // k + 50                      # 100 rows past the last expert
    cfg = M.config(T, d, E, k, F, precision=precision)
    r = np.random.default_rng(11)
    x = r.standard_normal((T * k, d)).astype(np.float32)
    wg = (r.standard_normal((E, F, d)) / np.sqrt(d)).astype(np.float32)
    wu = (r.standard_normal((E, F, d)) / np.sqrt(d)).astype(np.float32)
    wd = (r.standard_normal((E, d, F)) / np.sqrt(F)).astype(np.float32)
    xb, wgb, wub, wdb = (torch.from_numpy(a).to(torch.bfloat16) for a in (x, wg, wu, wd))
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    w13 = M.moe_pack_weights(M.config(T, d, E, k, F), wgb.to(DEV), wub.to(DEV))
    wdd = wdb.to(DEV)
    if precision == "mxfp8":
        w13, wdd = M.moe_pack_weights_mxfp8(cfg, w13, wdd)
    y_perm = torch.full((T * k, d), 7.0, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    M.moe_grouped_ffn(cfg, xb.to(DEV), torch.from_numpy(offsets).to(DEV), w13, wdd, y_perm=y_perm, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & (M.MOE_STATUS_TIMEOUT | M.MOE_STATUS_BAD_ROUTE) == 0
    got = np64(y_perm)
    xs = cases.as64(xb)
    want = np.zeros((n, d))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            ws = (cases.as64(wgb[e]), cases.as64(wub[e]), cases.as64(wdb[e]))
            want[lo:hi] = X.mx_swiglu_expert(xs[lo:hi], *ws)[0] if precision == "mxfp8" else O.swiglu_expert(xs[lo:hi], *ws)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            assert C.row_rel_err(got[lo:hi], want[lo:hi]) <= C.TOL_BF16, f"expert {e} ({hi - lo} rows)"
    assert bool((got[n:] == 7.0).all())
