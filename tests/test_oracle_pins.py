"""Pins of the CPU oracle to facts fixed outside it (CPU only).

Each test checks the oracle against something it does not compute itself: the
numbers the dispatch page prints for its two worked routing maps, brute force
over all expert subsets, closed forms of identity-tagged tokens with
scale-by-constant experts, and torch library routines on special cases that
reduce to them (dense SwiGLU when E=k=1, a dense softmax mixture when k=E).
The last group plants known mistakes in a copy of the combine step and checks
that the comparison rules catch them.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from oracle import check as C
from oracle import cases
import workloads as W

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- worked maps
def _load_maps(golden_dir):
    with open(os.path.join(golden_dir, "dispatch_worked_maps.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("name", ["map1", "map2"])
def test_worked_routing_maps(golden_dir, name):
    g = _load_maps(golden_dir)
    toks = g["tokens"]
    m = g["maps"][name]
    idx = np.array([[m["expert_of_token"][t]] for t in toks], np.int32)
    meta = O.dispatch_meta(idx, E=4, cap=-1)
    assert meta["routed"].tolist() == m["counts_printed"]
    assert meta["kept"].tolist() == m["counts_printed"]
    assert meta["offsets"].tolist() == [0] + np.cumsum(m["counts_printed"]).tolist()
    grouped = [[toks[t] for t in meta["perm_src"][meta["offsets"][e]:meta["offsets"][e + 1]]]
               for e in range(4)]
    assert grouped == m["expected_grouping_by_expert"]
    remote = O.remote_assignments(idx[:, 0], tokens_per_rank=2, experts_per_rank=1)
    assert remote == m["remote_vectors_printed"]
    assert remote * g["row_bytes"] == m["remote_bytes_printed"]
    assert C.permutation_consistent(meta["dest_row"], meta["perm_src"], meta["offsets"], idx)


# ---------------------------------------------------------------- selection
def _brute_topk(row, k):
    """The k-subset whose every member beats every non-member under
    (higher score, then lower index); slots ordered the same way."""
    E = len(row)

    def beats(a, b):
        return row[a] > row[b] or (row[a] == row[b] and a < b)

    winners = [S for S in itertools.combinations(range(E), k)
               if all(beats(a, b) for a in S for b in range(E) if b not in S)]
    assert len(winners) == 1
    return sorted(winners[0], key=lambda e: (-row[e], e))


def _tie_rows(T, E):
    s = RNG.integers(-3, 4, size=(T, E)).astype(np.float32)   # many exact ties
    s[0] = 1.0                                                 # all tied
    s[1] = -np.inf                                             # all -inf
    s[2, : E // 2] = -np.inf
    return s


@pytest.mark.parametrize("E", [1, 2, 3, 4, 6])
def test_topk_against_brute_force(E):
    s = _tie_rows(16, E)
    for k in sorted({1, min(2, E), E}):
        idx = O.topk_select(s, k)
        for t in range(s.shape[0]):
            assert idx[t].tolist() == _brute_topk(s[t].tolist(), k)


def test_topk_against_library_sort():
    s = RNG.standard_normal((300, 64)).astype(np.float32)
    s[:, 5] = s[:, 9]                                          # planted ties
    for k in (1, 6, 64):
        idx = O.topk_select(s, k)
        order = np.lexsort((np.broadcast_to(np.arange(64), s.shape), -s), axis=1)[:, :k]
        assert np.array_equal(idx, order)


def test_topk_matches_torch_topk_without_ties():
    s = RNG.standard_normal((200, 16)).astype(np.float32)
    idx = O.topk_select(s, 4)
    ref = torch.topk(torch.from_numpy(s), 4, dim=1).indices.numpy()
    assert np.array_equal(idx, ref)


def test_nan_logits_count_as_minus_inf():
    s = np.array([[0.5, np.nan, 0.2, np.nan]], np.float64)
    s32, nan_row = O.decision_logits(s)
    assert nan_row.tolist() == [True]
    assert O.topk_select(s32, 3).tolist() == [[0, 2, 1]]


# ---------------------------------------------------------------- gates
def test_gates_are_softmax_over_picks():
    s = RNG.standard_normal((100, 8)) * 3
    idx = O.topk_select(s.astype(np.float32), 3)
    g = O.gates(s, idx)
    picked = torch.from_numpy(np.take_along_axis(s, idx.astype(np.int64), 1))
    ref = torch.softmax(picked, dim=1).numpy()                    # library softmax
    assert np.allclose(g, ref, rtol=1e-12, atol=1e-15)
    assert np.allclose(g.sum(1), 1.0)
    # equal to the full softmax renormalised (torch, different route)
    p = torch.softmax(torch.from_numpy(s), dim=1).numpy()
    pk = np.take_along_axis(p, idx.astype(np.int64), 1)
    assert np.allclose(g, pk / pk.sum(1, keepdims=True), rtol=1e-12)


def test_gates_degenerate_rows():
    s = np.array([[-np.inf, -np.inf, -np.inf], [0.0, -np.inf, -np.inf]])
    idx = O.topk_select(s.astype(np.float32), 2)
    assert idx.tolist() == [[0, 1], [0, 1]]
    g = O.gates(s, idx)
    assert g.tolist() == [[0.0, 0.0], [1.0, 0.0]]


def test_router_margin_closed_form():
    s = np.array([[3.0, 1.0, 2.5, 0.0], [1.0, 1.0, 1.0, 0.5]])
    assert O.router_margin(s, 1).tolist() == [0.5, 0.0]
    assert O.router_margin(s, 3).tolist() == [1.0, 0.5]
    assert O.min_adjacent_gap(s, 2).tolist() == [0.5, 0.0]


def test_router_logits_closed_form():
    h = np.array([[1.0, 2.0], [0.0, -1.0]])
    w = np.array([[1.0, 0.0], [0.5, 0.5], [0.0, 0.0]])
    b = np.array([0.0, 1.0, -np.inf])
    s = O.router_logits(h, w, b)
    assert s.tolist() == [[1.0, 2.5, -np.inf], [0.0, 0.5, -np.inf]]


# ---------------------------------------------------------------- dispatch / capacity
def _random_idx(T, E, k, seed):
    r = np.random.default_rng(seed)
    rows = [r.permutation(E)[:k] for _ in range(T)]
    return np.stack(rows).astype(np.int32) if rows else np.zeros((0, k), np.int32)


@pytest.mark.parametrize("T,E,k,cap", [(50, 5, 2, -1), (200, 8, 3, 40), (64, 4, 4, 10), (1, 3, 1, -1),
                                       (0, 3, 1, -1), (30, 6, 2, 0)])
def test_dispatch_invariants_and_capacity(T, E, k, cap):
    idx = _random_idx(T, E, k, T + E)
    meta = O.dispatch_meta(idx.reshape(T, k), E, cap)
    routed = np.bincount(idx.ravel(), minlength=E)
    assert meta["routed"].tolist() == routed.tolist()
    assert meta["routed"].sum() == T * k
    kept = routed if cap < 0 else np.minimum(routed, cap)
    assert meta["kept"].tolist() == kept.tolist()
    assert meta["offsets"][-1] == T * k - (0 if cap < 0 else np.maximum(routed - cap, 0).sum())
    assert C.permutation_consistent(meta["dest_row"], meta["perm_src"], meta["offsets"], idx.reshape(T, k))
    # the kept set of each expert is exactly its `cap` lowest token indices
    for e in range(E):
        users = sorted(t for t in range(T) if e in idx[t])
        want = users if cap < 0 else users[:cap]
        got = meta["perm_src"][meta["offsets"][e]:meta["offsets"][e + 1]].tolist()
        assert got == want


@pytest.mark.parametrize("T,E,k,cap", [(200, 8, 3, 40), (64, 4, 4, 10), (30, 6, 2, 0), (9, 3, 1, 5)])
def test_padded_layout_brute_force(T, E, k, cap):
    """Padded capacity layout, from its definition by brute force: expert e
    owns rows [e*cap, (e+1)*cap); the first min(routed_e, cap) hold the tokens
    that picked e, in ascending order; the rest are padding (-1)."""
    idx = _random_idx(T, E, k, 7 * T + E).reshape(T, k)
    pm = O.dispatch_meta_padded(idx, E, cap)
    assert pm["offsets"].tolist() == [e * cap for e in range(E + 1)]
    assert len(pm["perm_src"]) == E * cap
    for e in range(E):
        users = [t for t in range(T) if e in idx[t]]
        kept = users[:cap]
        seg = pm["perm_src"][e * cap:(e + 1) * cap].tolist()
        assert seg == kept + [-1] * (cap - len(kept))
        for r, t in enumerate(kept):
            j = list(idx[t]).index(e)
            assert pm["dest_row"][t, j] == e * cap + r
        for t in users[cap:]:
            assert pm["dest_row"][t, list(idx[t]).index(e)] == -1
    # the same assignments are kept as in the compact capacity layout
    cm = O.dispatch_meta(idx, E, cap)
    assert ((pm["dest_row"] >= 0) == (cm["dest_row"] >= 0)).all()
    assert pm["kept"].tolist() == cm["kept"].tolist()
    with pytest.raises(ValueError):
        O.dispatch_meta_padded(idx, E, -1)


def test_invalid_routes_are_dropped_and_flagged():
    idx = np.array([[0, 0], [1, 5], [-1, 2], [2, 1]], np.int32)
    meta = O.dispatch_meta(idx, E=3, cap=-1)
    assert meta["bad_route"]
    assert (meta["dest_row"][0] >= 0).tolist() == [True, False]
    assert (meta["dest_row"][1] >= 0).tolist() == [True, False]
    assert (meta["dest_row"][2] >= 0).tolist() == [False, True]
    assert meta["routed"].tolist() == [1, 2, 2]


def test_capacity_formula_values():
    assert O.capacity(16384, 6, 64) == 1920
    assert O.capacity(64, 2, 4) == 40
    assert O.capacity(8, 1, 4) == 2
    assert W.capacity_factor_cap(16384, 6, 64) == 1920


# ---------------------------------------------------------------- closed forms of the layer
def test_identity_tagged_scale_experts_closed_form():
    inp = cases.parity_inputs("tiny_f32_tagged")
    wl = inp.wl
    h = cases.as64(inp.h)
    out = O.layer_forward(h, cases.as64(inp.w_router), None, wl.k, "scale")
    idx, g, y = out["idx"], out["gate"], out["y"]
    for t in range(wl.T):
        c = t % wl.d
        expect = (t + 1) * sum(g[t, j] * (idx[t, j] + 1) for j in range(wl.k))
        row = y[t].copy()
        assert row[c] == pytest.approx(expect, rel=1e-13)
        row[c] = 0.0
        assert not row.any()


def test_identity_experts_return_input():
    inp = cases.parity_inputs("tiny_f32")
    wl = inp.wl
    h = cases.as64(inp.h)
    out = O.layer_forward(h, cases.as64(inp.w_router), None, wl.k, "identity")
    assert np.allclose(out["y"], h, rtol=1e-14, atol=1e-14)


def test_identity_experts_with_drops_scale_by_kept_gates():
    h = RNG.standard_normal((40, 8))
    w = RNG.standard_normal((4, 8))
    out = O.layer_forward(h, w, None, 2, "identity", cap=10)
    kept_gate = np.where(out["dest_row"] >= 0, out["gate"], 0.0).sum(1)
    assert np.allclose(out["y"], h * kept_gate[:, None], rtol=1e-14, atol=1e-14)
    assert (kept_gate < 1).any()                                # something was dropped


def test_single_expert_is_dense_swiglu():
    T, d, F = 20, 16, 24
    h = RNG.standard_normal((T, d))
    wg, wu, wd = RNG.standard_normal((1, F, d)), RNG.standard_normal((1, F, d)), RNG.standard_normal((1, d, F))
    out = O.layer_forward(h, RNG.standard_normal((1, d)), None, 1, "swiglu",
                          weights=lambda e: (wg[e], wu[e], wd[e]))
    ht = torch.from_numpy(h)
    ref = (torch.nn.functional.silu(ht @ torch.from_numpy(wg[0]).T) * (ht @ torch.from_numpy(wu[0]).T)) \
        @ torch.from_numpy(wd[0]).T
    assert np.allclose(out["y"], ref.numpy(), rtol=1e-12, atol=1e-12)
    assert (out["gate"] == 1.0).all()


def test_all_experts_is_dense_softmax_mixture():
    T, d, F, E = 12, 8, 10, 4
    h = RNG.standard_normal((T, d))
    wr = RNG.standard_normal((E, d))
    b = RNG.standard_normal(E)
    wg, wu, wd = RNG.standard_normal((E, F, d)), RNG.standard_normal((E, F, d)), RNG.standard_normal((E, d, F))
    out = O.layer_forward(h, wr, b, E, "swiglu", weights=lambda e: (wg[e], wu[e], wd[e]))
    ht = torch.from_numpy(h)
    p = torch.softmax(ht @ torch.from_numpy(wr).T + torch.from_numpy(b), dim=1)
    ref = torch.zeros(T, d, dtype=torch.float64)
    for e in range(E):
        fe = (torch.nn.functional.silu(ht @ torch.from_numpy(wg[e]).T) * (ht @ torch.from_numpy(wu[e]).T)) \
            @ torch.from_numpy(wd[e]).T
        ref += p[:, e:e + 1] * fe
    assert np.allclose(out["y"], ref.numpy(), rtol=1e-12, atol=1e-12)
    assert (out["routed"] == T).all()


def test_silu_against_library():
    z = np.linspace(-30, 30, 1001)
    assert np.allclose(O.silu(z), torch.nn.functional.silu(torch.from_numpy(z)).numpy(), rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------- planted mistakes
def _permuted_pipeline(h, idx, gate, meta, kind, wrong_index=False, swap_gates=False):
    """CPU emulation of the grouped path: gather rows by expert, apply experts
    per segment, scatter back. wrong_index plants the bug of scattering with the
    pre-permutation index; swap_gates pairs each output with the other slot's
    gate."""
    x_perm = h[meta["perm_src"]]
    y_perm = np.zeros_like(x_perm)
    off = meta["offsets"]
    for e in range(len(off) - 1):
        y_perm[off[e]:off[e + 1]] = O.expert_apply(kind, e, x_perm[off[e]:off[e + 1]])
    y = np.zeros_like(h)
    T, k = idx.shape
    for t in range(T):
        for j in range(k):
            r = meta["dest_row"][t, j]
            if r < 0:
                continue
            src = y_perm[r] if not wrong_index else y_perm[min(t * k + j, len(y_perm) - 1)]
            gj = gate[t, (j + 1) % k] if swap_gates else gate[t, j]
            y[t] += gj * src
    return y


@pytest.mark.parametrize("kind", ["scale", "identity"])
def test_checker_catches_planted_mistakes(kind):
    inp = cases.parity_inputs("tiny_f32_tagged")
    h = cases.as64(inp.h)
    out = O.layer_forward(h, cases.as64(inp.w_router), None, inp.wl.k, kind)
    meta = {k_: out[k_] for k_ in ("perm_src", "offsets", "dest_row")}
    good = _permuted_pipeline(h, out["idx"], out["gate"], meta, kind)
    assert C.row_rel_err(good, out["y"]) < 1e-12
    bad_index = _permuted_pipeline(h, out["idx"], out["gate"], meta, kind, wrong_index=True)
    assert not C.outputs_match(bad_index, out["y"], "f32")
    if kind == "scale":   # identity experts sum to h whatever gate goes with which slot
        bad_gate = _permuted_pipeline(h, out["idx"], out["gate"], meta, kind, swap_gates=True)
        assert not C.outputs_match(bad_gate, out["y"], "f32")


def test_permutation_check_catches_swapped_rows():
    idx = _random_idx(40, 5, 2, 7)
    meta = O.dispatch_meta(idx, 5)
    assert C.permutation_consistent(meta["dest_row"], meta["perm_src"], meta["offsets"], idx)
    dr = meta["dest_row"].copy()
    a, b = np.argwhere(dr >= 0)[[0, 7]]
    dr[tuple(a)], dr[tuple(b)] = dr[tuple(b)], dr[tuple(a)]
    assert not C.permutation_consistent(dr, meta["perm_src"], meta["offsets"], idx)


# ---------------------------------------------------------------- generator + margin pass
def test_generator_is_deterministic_and_streams_differ():
    wl = W.get("mixtral_scaled").with_(T=64)
    a, b = W.draw_h(wl, 0), W.draw_h(wl, 0)
    assert torch.equal(a, b)
    assert not torch.equal(a, W.draw_h(wl, 1))
    g0 = W.draw_w_gate(wl.with_(F=128, d=128, E=3), 0)
    g1 = W.draw_w_gate(wl.with_(F=128, d=128, E=3), 0, experts=[1])
    assert torch.equal(g0[1], g1[0])


def test_margin_pass_reaches_min_gap():
    inp = cases.parity_inputs("mixtral_scaled", weights=False)
    s = O.router_logits(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias))
    assert O.min_adjacent_gap(s, inp.wl.k).min() >= cases.MIN_GAP


def test_many_small_hot_bias_gives_half_the_assignments():
    wl = W.get("many_small")
    inp = cases.parity_inputs(wl, weights=False)
    out = O.route(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias), wl.k)
    share = (out[0] < W.HOT_EXPERTS).mean()
    assert abs(share - 0.5) <= 0.01
    assert not (out[0] >= W.EMPTY_FROM).any()


def test_skewed_bias_gives_hot_experts_and_empties():
    wl = W.get("skewed")
    inp = cases.parity_inputs(wl, weights=False)
    idx = O.route(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias), wl.k)[0]
    counts = np.bincount(idx.ravel(), minlength=wl.E)
    assert counts[list(W.SKEWED_EMPTY)].sum() == 0
    assert counts.max() >= 5 * counts.mean()
    assert O.dispatch_meta(idx, wl.E, O.capacity(wl.T, wl.k, wl.E))["kept"].max() == 1920


# ---------------------------------------------------------------- backward: finite differences
def _bwd_problem(seed, T=6, d=8, E=4, k=2, F=5):
    r = np.random.default_rng(seed)
    h = r.standard_normal((T, d))
    w_r = r.standard_normal((E, d))
    bias = r.standard_normal(E) * 0.3
    wg = r.standard_normal((E, F, d)) / np.sqrt(d)
    wu = r.standard_normal((E, F, d)) / np.sqrt(d)
    wd = r.standard_normal((E, d, F)) / np.sqrt(F)
    dy = r.standard_normal((T, d))
    return h, w_r, bias, wg, wu, wd, dy


@pytest.mark.parametrize("seed,cap", [(1, -1), (2, -1), (3, 2)])
def test_backward_matches_central_differences(seed, cap):
    """Every gradient of L = <dy, y> against central differences of the
    forward definition (eps 1e-6, fp64); the routing decision is checked to
    be unchanged by each perturbation, and cap=2 drops slots."""
    h, w_r, bias, wg, wu, wd, dy = _bwd_problem(seed)
    k, E = 2, w_r.shape[0]
    s = O.router_logits(h, w_r, bias)
    assert O.min_adjacent_gap(s, k).min() > 1e-3             # decisions far from any tie

    def loss(h_, w_r_, b_, wg_, wu_, wd_):
        out = O.layer_forward(h_, w_r_, b_, k, "swiglu", lambda e: (wg_[e], wu_[e], wd_[e]), cap)
        return float(np.sum(dy * out["y"])), out["idx"], out["dest_row"]

    g = O.layer_backward(h, w_r, bias, k, lambda e: (wg[e], wu[e], wd[e]), cap, dy)
    base = [h, w_r, bias, wg, wu, wd]
    names = ["dh", "dw_router", "dbias", "dw_gate", "dw_up", "dw_down"]
    _, idx0, dest0 = loss(*base)
    if cap >= 0:
        assert (dest0 < 0).any()                                  # some slot is dropped
    eps = 1e-6
    r = np.random.default_rng(seed + 100)
    for pi, name in enumerate(names):
        p = base[pi]
        flat = p.reshape(-1)
        picks = r.choice(flat.size, size=min(flat.size, 12), replace=False)
        for i in picks:
            args_p = [a.copy() for a in base]
            args_m = [a.copy() for a in base]
            args_p[pi].reshape(-1)[i] += eps
            args_m[pi].reshape(-1)[i] -= eps
            lp, ip, dp = loss(*args_p)
            lm, im, dm = loss(*args_m)
            assert np.array_equal(ip, idx0) and np.array_equal(im, idx0)
            assert np.array_equal(dp, dest0) and np.array_equal(dm, dest0)
            fd = (lp - lm) / (2 * eps)
            an = g[name].reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, an)


def test_backward_gate_gradient_sums_to_zero():
    """Softmax over the picks: for every token, sum_j ds_j = 0 (the gates sum
    to one whatever the scores), so db sums to zero and each token's router
    gradient lies in the span of the picked rows."""
    h, w_r, bias, wg, wu, wd, dy = _bwd_problem(5, T=20)
    g = O.layer_backward(h, w_r, bias, 2, lambda e: (wg[e], wu[e], wd[e]), -1, dy)
    assert np.allclose(g["ds"].sum(axis=1), 0.0, atol=1e-12)
    assert abs(g["dbias"].sum()) < 1e-10


def test_matrix_rel_err_measure():
    r = np.random.default_rng(0)
    w = r.standard_normal((5, 7))
    assert C.matrix_rel_err(w, w) == 0.0
    bad = w.copy()
    bad[2, 3] += 0.03 * np.abs(w).max()
    assert C.matrix_rel_err(bad, w) == pytest.approx(0.03)
    assert C.matrix_rel_err(np.zeros((3, 3)), np.zeros((3, 3))) == 0.0


@pytest.mark.parametrize("cap", [-1, 2])
def test_backward_probe_equals_full_backward(cap):
    """The one-by-one entries used at full size agree with the full
    (finite-difference-pinned) backward."""
    h, w_r, bias, wg, wu, wd, dy = _bwd_problem(9, T=12)
    wf = lambda e: (wg[e], wu[e], wd[e])
    full = O.layer_backward(h, w_r, bias, 2, wf, cap, dy)
    tokens = np.array([0, 3, 7, 11])
    elems = [(0, 1, 2, 3), (1, 4, 0, 7), (3, 2, 5, 1), (2, 0, 7, 6)]
    pr = O.layer_backward_probe(h, w_r, bias, 2, wf, cap, dy, tokens, elems)
    assert np.allclose(pr["dh"], full["dh"][tokens], rtol=1e-12, atol=1e-12)
    for n, (e, f, i, j) in enumerate(elems):
        assert pr["dw_down"][n] == pytest.approx(full["dw_down"][e][i, f], rel=1e-10, abs=1e-12)
        assert pr["dw_gate"][n] == pytest.approx(full["dw_gate"][e][f, j], rel=1e-10, abs=1e-12)
        assert pr["dw_up"][n] == pytest.approx(full["dw_up"][e][f, j], rel=1e-10, abs=1e-12)


@pytest.mark.parametrize("cap", [-1, 2])
def test_backward_channels_equal_full_backward(cap):
    """The whole rows and columns used at full size agree with the full
    (finite-difference-pinned) backward; an expert with no kept rows gives
    zero rows."""
    h, w_r, bias, wg, wu, wd, dy = _bwd_problem(9, T=12)
    wf = lambda e: (wg[e], wu[e], wd[e])
    full = O.layer_backward(h, w_r, bias, 2, wf, cap, dy)
    chans = [(0, 1), (1, 4), (3, 2), (2, 0), (0, 3)]
    ch = O.layer_backward_channels(h, w_r, bias, 2, wf, cap, dy, chans)
    for n, (e, f) in enumerate(chans):
        assert np.allclose(ch["dw_gate_rows"][n], full["dw_gate"][e][f, :], rtol=1e-10, atol=1e-12)
        assert np.allclose(ch["dw_up_rows"][n], full["dw_up"][e][f, :], rtol=1e-10, atol=1e-12)
        assert np.allclose(ch["dw_down_cols"][n], full["dw_down"][e][:, f], rtol=1e-10, atol=1e-12)


def test_gradient_row_check_rejects_zero_and_sign_flip():
    """The full-size weight-gradient check compares whole rows against their
    own largest element at 2e-2; a zeroed row, a sign-flipped row and a row
    missing one expert row's term all fail it, while bf16-sized rounding of
    every term passes."""
    r = np.random.default_rng(4)
    n, d = 4000, 256
    terms_a = r.standard_normal((n, 1)) * r.standard_normal((n, d))   # random-sign terms of a sum over rows
    row = terms_a.sum(axis=0)
    assert C.vector_rel_err(np.zeros(d), row) > C.TOL_BF16
    assert C.vector_rel_err(-row, row) > C.TOL_BF16
    assert C.vector_rel_err(row - terms_a[np.abs(terms_a).sum(axis=1).argmax()], row) > C.TOL_BF16
    rounded = terms_a * (1.0 + r.uniform(-2.0 ** -8, 2.0 ** -8, size=terms_a.shape))
    assert C.vector_rel_err(rounded.sum(axis=0), row) < 0.1 * C.TOL_BF16
