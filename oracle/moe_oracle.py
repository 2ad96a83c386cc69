"""CPU oracle of the token-choice MoE layer forward (test infrastructure only).

Only tests, the smoke check and the benchmark's CPU-baseline leg may import
this module; the product path never does. It shares no code with the CUDA
library: it takes plain arrays, computes in fp64 (the pages fix no precision),
and uses numpy's matmul as its one library primitive.

Sources (page title -- section):
  [REPEAT]   "How Does Mixture-of-Experts Routing Affect LLM Repeatability?" --
             the simplified token-choice layer (s_t = h_t W_r, E_t = TopK(s_t, k),
             y_t = sum_{e in E_t} g_{t,e} f_e(h_t)); "Boundary Matters" (router
             margin m_t = s_(k) - s_(k+1)); deterministic tie handling and
             capacity resolved in request order.
  [DISPATCH] "MoE Token Dispatch: Why an All-Reduce Result Does Not Describe the
             Exchange" -- "Follow one documented dispatch and return path"
             (per-expert counts from the routing map, rearrange tokens and
             probabilities, restore order and shape); the two worked routing maps.
  [UNPERM]   archcrux "moe-unpermute-wrong-token" -- outputs restored to the
             original positions, top-2 weights tied to the same token.
  [DROPLESS] "Dropless MoE Is a Runtime Problem as Much as a Model Design" --
             variable-length expert groups, grouped computation.
  [CAPACITY] "How does dropless MoE dispatch differ from capacity factor token
             dropping?" -- buffer cap = factor x tokens / experts; an overflowed
             token skips the FFN and keeps its residual.

Readings where the pages are silent or garbled (each also listed in the
design notes):
  * gate g_{t,e}: the definition list under the layer formulas was lost in
    extraction; g = softmax(s_t) over all E experts, renormalised over the k
    picks.
  * top-k is decided on the fp32 logits (the kernel's precision), ties to the
    lowest expert index; slot j of token t holds its (j+1)-th best expert.
  * NaN logits count as -inf; a token whose logits are all -inf picks experts
    0..k-1 with gate 0.
  * capacity counts assignments: C = floor(1.25 * T * k / E); within an expert
    lower token index wins; dropped assignments contribute 0 and the kept gates
    are not renormalised.
  * the expert FFN is SwiGLU: f_e(x) = W_down,e (silu(W_gate,e x) * (W_up,e x)),
    silu(z) = z / (1 + exp(-z)); test experts: identity f_e(x) = x and scale
    f_e(x) = (e + 1) x.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def router_logits(h, w_r, bias=None):
    """s_t = h_t W_r^T (+ b), fp64. [REPEAT] layer formulas; W_r stored [E, d]."""
    s = np.asarray(h, F64) @ np.asarray(w_r, F64).T
    if bias is not None:
        s = s + np.asarray(bias, F64)[None, :]
    return s


def decision_logits(s):
    """Round logits to fp32 (the precision the selection is decided in).

    NaN becomes -inf. Returns (s32, nan_row) where nan_row flags tokens that
    had a NaN logit.
    """
    s32 = np.asarray(s, F64).astype(np.float32)
    nan = np.isnan(s32)
    return np.where(nan, np.float32(-np.inf), s32), nan.any(axis=1)


def topk_select(s, k, chunk=512):
    """E_t = TopK(s_t, k) with deterministic ties. [REPEAT] layer formulas and
    "stable score ordering, deterministic tie handling".

    rank(e) = #{e' : s_e' > s_e  or  (s_e' == s_e and e' < e)}; expert e is
    picked iff rank(e) < k and goes to slot rank(e). Returns idx [T, k] int32.
    """
    s = np.asarray(s)
    T, E = s.shape
    if not 0 < k <= E:
        raise ValueError("need 0 < k <= E")
    idx = np.empty((T, k), np.int32)
    e_col = np.arange(E)[None, :, None]   # the expert being ranked
    e_row = np.arange(E)[None, None, :]   # the experts it is compared with
    for c0 in range(0, T, chunk):
        sc = s[c0:c0 + chunk]
        mine = sc[:, :, None]
        other = sc[:, None, :]
        beats = (other > mine) | ((other == mine) & (e_row < e_col))
        rank = beats.sum(axis=2)
        tt, ee = np.nonzero(rank < k)
        idx[c0 + tt, rank[tt, ee]] = ee
    return idx


def softmax(s):
    """p = softmax(s) over the experts, fp64, max-subtracted. A row of all -inf
    gives all zeros (degenerate case, no expert has a finite score)."""
    s = np.asarray(s, F64)
    s = np.where(np.isnan(s), -np.inf, s)
    m = s.max(axis=1, keepdims=True)
    finite = np.isfinite(m)
    ex = np.exp(s - np.where(finite, m, 0.0))
    den = ex.sum(axis=1, keepdims=True)
    return np.where(den > 0, ex / np.where(den > 0, den, 1.0), 0.0)


def gates(s, idx):
    """g_{t,j} = p_t[e_j] / sum_j' p_t[e_j'] with p_t = softmax(s_t).
    [REPEAT] layer formulas (gate weight g_{t,e}); renormalised over the picks."""
    p = softmax(s)
    picked = np.take_along_axis(p, np.asarray(idx, np.int64), axis=1)
    den = picked.sum(axis=1, keepdims=True)
    return np.where(den > 0, picked / np.where(den > 0, den, 1.0), 0.0)


def route(h, w_r, bias, k):
    """Router scores -> (idx [T,k] int32, gate [T,k] fp64, logits fp64, nan_row)."""
    s = router_logits(h, w_r, bias)
    s32, nan_row = decision_logits(s)
    idx = topk_select(s32, k)
    return idx, gates(s, idx), s, nan_row


def router_margin(s, k):
    """m_t = s_t,(k) - s_t,(k+1), the gap between the k-th and (k+1)-th largest
    scores. [REPEAT] "Boundary Matters". Needs k < E."""
    srt = -np.sort(-np.asarray(s, F64), axis=1)
    return srt[:, k - 1] - srt[:, k]


def min_adjacent_gap(s, k):
    """Smallest gap between consecutive scores among the k+1 largest (so that
    both the picked set and the slot order are away from a boundary)."""
    srt = -np.sort(-np.asarray(s, F64), axis=1)
    top = srt[:, :min(k + 1, srt.shape[1])]
    if top.shape[1] < 2:
        return np.full(top.shape[0], np.inf)
    with np.errstate(invalid="ignore"):
        gaps = top[:, :-1] - top[:, 1:]
    gaps = np.where(np.isnan(gaps), np.inf, gaps)   # -inf - -inf: both out of reach
    return gaps.min(axis=1)


def capacity(T, k, E, factor_num=5, factor_den=4):
    """Per-expert cap in assignments, floor(factor * T * k / E), factor 1.25.
    [CAPACITY] capacity is a factor times the tokens per expert; counted here in
    assignments (T*k), the configuration text's reading."""
    return (factor_num * T * k) // (factor_den * E)


def valid_slots(idx, E):
    """A slot is valid iff its expert is in [0, E) and no earlier slot of the same
    token names the same expert. Invalid slots are dropped and flagged."""
    idx = np.asarray(idx)
    T, k = idx.shape
    ok = (idx >= 0) & (idx < E)
    for j in range(1, k):
        for jj in range(j):
            ok[:, j] &= idx[:, j] != idx[:, jj]
    return ok


def dispatch_meta(idx, E, cap=-1):
    """Per-expert counts, offsets, drop decisions and the permutation.
    [DISPATCH] counts per expert are derived from the routing map and tokens
    grouped by expert; [REPEAT] capacity resolved in order; [CAPACITY] overflow.

    Walks the assignments in token order. rank = number of earlier tokens that
    picked the same expert; the assignment is kept iff dropless (cap < 0) or
    rank < cap. Kept rows of expert e occupy [offsets[e], offsets[e+1]) in
    ascending token order.

    Returns dict: routed [E], kept [E], offsets [E+1], dest_row [T,k] (-1 =
    dropped or invalid), perm_src [n_kept], rank [T,k], bad_route (bool).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    ok = valid_slots(idx, E)
    seen = [0] * E
    rank = np.full((T, k), -1, np.int64)
    for t in range(T):
        for j in range(k):
            if ok[t, j]:
                e = int(idx[t, j])
                rank[t, j] = seen[e]
                seen[e] += 1
    routed = np.array(seen, np.int64)
    kept = routed if cap < 0 else np.minimum(routed, cap)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(kept)
    dest_row = np.full((T, k), -1, np.int64)
    keep = ok & ((cap < 0) | (rank < cap))
    tt, jj = np.nonzero(keep)
    dest_row[tt, jj] = offsets[idx[tt, jj]] + rank[tt, jj]
    perm_src = np.full(int(offsets[-1]), -1, np.int64)
    perm_src[dest_row[tt, jj]] = tt
    return dict(routed=routed, kept=kept, offsets=offsets, dest_row=dest_row,
                perm_src=perm_src, rank=rank, bad_route=bool((~ok).any()))


def dispatch_meta_padded(idx, E, cap):
    """The padded layout with a fixed per-expert capacity: the comparison arm
    of the evaluation in "Dropless MoE Is a Runtime Problem as Much as a Model
    Design" (its grouped-GEMM paragraph contrasts one grouped computation with
    padding every expert up to one shared capacity; its evaluation paragraph
    lists that padded capacity arm beside the dropless one). Every expert owns
    a buffer of exactly cap rows: expert e's rows are [e*cap, (e+1)*cap). The
    kept assignments and their ranks are those of the capacity mode
    (dispatch_meta with the same cap); a kept assignment of rank r goes to row
    e*cap + r, and the rows past an expert's kept count are padding
    (perm_src = -1, a zero row in x_perm).

    Returns dispatch_meta's dict with offsets [E+1] = e*cap, dest_row [T,k] and
    perm_src [E*cap] in this layout.
    """
    if cap < 0:
        raise ValueError("the padded layout needs a capacity")
    m = dispatch_meta(idx, E, cap)
    idx = np.asarray(idx)
    offsets = np.arange(E + 1, dtype=np.int64) * cap
    dest_row = np.full(idx.shape, -1, np.int64)
    keep = m["dest_row"] >= 0
    tt, jj = np.nonzero(keep)
    dest_row[tt, jj] = offsets[idx[tt, jj]] + m["rank"][tt, jj]
    perm_src = np.full(E * cap, -1, np.int64)
    perm_src[dest_row[tt, jj]] = tt
    return dict(m, offsets=offsets, dest_row=dest_row, perm_src=perm_src)


def silu(z):
    """silu(z) = z / (1 + exp(-z))."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_expert(x, w_gate, w_up, w_down):
    """f_e(x) = W_down (silu(W_gate x) * (W_up x)) for each row of x, fp64, no
    intermediate rounding. Rows are independent, so applying it to a stack of
    tokens is f_e applied to each token."""
    x = np.asarray(x, F64)
    g = x @ np.asarray(w_gate, F64).T
    u = x @ np.asarray(w_up, F64).T
    return (silu(g) * u) @ np.asarray(w_down, F64).T


def expert_apply(kind, e, x, weights=None):
    """f_e on rows x for one expert e. weights(e) -> (w_gate, w_up, w_down)."""
    if kind == "identity":
        return np.asarray(x, F64)
    if kind == "scale":
        return (e + 1.0) * np.asarray(x, F64)
    if kind == "swiglu":
        return swiglu_expert(x, *weights(e))
    raise ValueError(kind)


def combine(h, idx, gate, dest_row, kind, weights=None, tokens=None):
    """y_t = sum over kept slots j of g_{t,j} f_{e_j}(h_t).
    [REPEAT] layer formulas; [UNPERM] output returned to token t itself;
    [CAPACITY] a dropped assignment adds nothing (the residual is outside).

    No permutation is used: each token is evaluated at its own position. Each
    expert is evaluated once on the tokens that kept it (a token names an
    expert at most once, so each token appears once per expert).
    tokens: optional subset of token indices; y has one row per listed token.
    """
    h = np.asarray(h, F64)
    T, d = h.shape
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    idx = np.asarray(idx)[tok]
    gate = np.asarray(gate, F64)[tok]
    kept = np.asarray(dest_row)[tok] >= 0
    y = np.zeros((len(tok), d), F64)
    for e in (np.unique(idx[kept]) if kept.any() else []):
        rows, js = np.nonzero(kept & (idx == e))
        out = expert_apply(kind, int(e), h[tok[rows]], weights)
        y[rows] += gate[rows, js, None] * out
    return y


def layer_forward(h, w_r, bias, k, kind, weights=None, cap=-1, tokens=None):
    """Whole layer: route, dispatch metadata, experts, combine. Returns dict."""
    idx, g, s, nan_row = route(h, w_r, bias, k)
    meta = dispatch_meta(idx, w_r.shape[0], cap)
    y = combine(h, idx, g, meta["dest_row"], kind, weights, tokens)
    return dict(idx=idx, gate=g, logits=s, nan_row=nan_row, y=y, **meta)


def remote_assignments(expert_of_token, tokens_per_rank, experts_per_rank):
    """Count assignments whose expert lives on another rank than the token's
    origin, and their bytes at a given row size. [DISPATCH] worked example of the
    routing maps (an uneven map sends most of eight assignments to one rank;
    origin rank r owns tokens r*tokens_per_rank ...). Host-side diagnostic only."""
    e = np.asarray(expert_of_token)
    origin = np.arange(e.shape[0]) // tokens_per_rank
    dest = e // experts_per_rank
    return int((origin != dest).sum())


# ---------------------------------------------------------------- backward
def layer_backward(h, w_r, bias, k, weights, cap, dy):
    """Gradients of the scalar L = sum_t <dy_t, y_t> for the SwiGLU layer.

    The pages define the forward pass only ([REPEAT] layer formulas) and treat
    dropless MoE as a training workload ([DROPLESS]); the backward pass is the
    chain rule through that definition, with the routing decision (which
    experts, which slots are kept) held fixed, as it is piecewise constant:

      y_t = sum over kept j of g_{t,j} o_{t,j},   o = W_d (silu(a) * u),
      a = W_g h_t, u = W_u h_t,                  g_j = exp(s_j) / sum_i exp(s_i)
                                                 over the picked slots i of t
      dgate_{t,j} = <dy_t, o_{t,j}> (0 for a dropped slot)
      ds_{t,j}    = g_j (dgate_j - sum_i g_i dgate_i)     (softmax over the picks)
      do = g_j dy_t;  dW_d += do m^T with m = silu(a) * u;  dm = W_d^T do
      da = dm * u * silu'(a),  silu'(a) = sig(a) (1 + a (1 - sig(a)));  du = dm * silu(a)
      dW_g += da h_t^T;  dW_u += du h_t^T;  dh_t += W_g^T da + W_u^T du
      router: dh_t += sum_j ds_j W_r[e_j];  dW_r[e_j] += ds_j h_t;  db[e_j] += ds_j

    weights(e) -> (w_gate [F,d], w_up [F,d], w_down [d,F]). Returns dict with
    dh [T,d], dw_router [E,d], dbias [E], dw_gate, dw_up [E,F,d], dw_down
    [E,d,F], dgate and ds [T,k], all fp64.
    """
    h = np.asarray(h, F64)
    w_r = np.asarray(w_r, F64)
    dy = np.asarray(dy, F64)
    T, d = h.shape
    E = w_r.shape[0]
    idx, g, _, _ = route(h, w_r, bias, k)
    meta = dispatch_meta(idx, E, cap)
    kept = meta["dest_row"] >= 0
    F = np.asarray(weights(0)[0]).shape[0]
    dh = np.zeros((T, d))
    dwg = np.zeros((E, F, d))
    dwu = np.zeros((E, F, d))
    dwd = np.zeros((E, d, F))
    dgate = np.zeros((T, k))
    for e in range(E):
        rows, js = np.nonzero(kept & (idx == e))
        if rows.size == 0:
            continue
        wg, wu, wd = (np.asarray(w, F64) for w in weights(e))
        x = h[rows]
        a = x @ wg.T
        u = x @ wu.T
        with np.errstate(over="ignore"):
            sg = 1.0 / (1.0 + np.exp(-a))
        m = a * sg * u
        o = m @ wd.T
        dgate[rows, js] = np.sum(dy[rows] * o, axis=1)
        do = g[rows, js, None] * dy[rows]
        dwd[e] = do.T @ m
        dm = do @ wd
        da = dm * u * (sg * (1.0 + a * (1.0 - sg)))
        du = dm * a * sg
        dwg[e] = da.T @ x
        dwu[e] = du.T @ x
        dh[rows] += da @ wg + du @ wu          # a token names expert e at most once
    ds = g * (dgate - np.sum(g * dgate, axis=1, keepdims=True))
    dwr = np.zeros((E, d))
    db = np.zeros(E)
    for j in range(k):
        e = np.asarray(idx[:, j], np.int64)
        np.add.at(dwr, e, ds[:, j, None] * h)
        np.add.at(db, e, ds[:, j])
        dh += ds[:, j, None] * w_r[e]
    return dict(dh=dh, dw_router=dwr, dbias=db, dw_gate=dwg, dw_up=dwu, dw_down=dwd, dgate=dgate, ds=ds,
                idx=idx, gate=g, **{kk: meta[kk] for kk in ("dest_row", "offsets", "kept", "routed")})


def layer_backward_probe(h, w_r, bias, k, weights, cap, dy, tokens, elems):
    """Selected entries of layer_backward's gradients, computed one by one so
    that a full-size layer stays within reach (same definitions, same fixed
    routing decision):
      dh rows for the listed tokens;
      for each (e, f, i, j) in elems: dW_down[e][i, f], dW_gate[e][f, j] and
      dW_up[e][f, j], each a sum over the rows routed to and kept by expert e
      of one gate/up channel f (the channel's pre-activations a[:, f], u[:, f]
      and its output gradient dm[:, f] = do . W_down[e][:, f]).
    Each expert's weights are fetched once. Returns dict dh [len(tokens), d]
    and dw_down, dw_gate, dw_up [len(elems)], plus dw_down_l1, dw_gate_l1,
    dw_up_l1: the sum of the absolute values of each element's terms, the
    natural scale of the rounding error of a sum."""
    h = np.asarray(h, F64)
    w_r = np.asarray(w_r, F64)
    dy = np.asarray(dy, F64)
    E = w_r.shape[0]
    idx, g, _, _ = route(h, w_r, bias, k)
    kept = dispatch_meta(idx, E, cap)["dest_row"] >= 0
    tokens = np.asarray(tokens)
    dh = np.zeros((len(tokens), h.shape[1]))
    dgate = np.zeros((len(tokens), k))
    keys = ("dw_down", "dw_gate", "dw_up")
    out = {key: np.zeros(len(elems)) for key in keys}
    out.update({key + "_l1": np.zeros(len(elems)) for key in keys})
    for e in range(E):
        pairs = [(n, j) for n, t in enumerate(tokens) for j in range(k) if kept[t, j] and idx[t, j] == e]
        mine = [(m, el) for m, el in enumerate(elems) if el[0] == e]
        if not pairs and not mine:
            continue
        wg, wu, wd = (np.asarray(w, F64) for w in weights(e))
        for n, j in pairs:
            t = tokens[n]
            a = wg @ h[t]
            u = wu @ h[t]
            with np.errstate(over="ignore"):
                sg = 1.0 / (1.0 + np.exp(-a))
            dgate[n, j] = dy[t] @ (wd @ (a * sg * u))
            dm = wd.T @ (g[t, j] * dy[t])
            dh[n] += wg.T @ (dm * u * sg * (1.0 + a * (1.0 - sg))) + wu.T @ (dm * a * sg)
        if mine:
            rows, js = np.nonzero(kept & (idx == e))
            x = h[rows]
            do = g[rows, js, None] * dy[rows]
            for m, (_, f, i, j) in mine:
                a = x @ wg[f]
                u = x @ wu[f]
                with np.errstate(over="ignore"):
                    sg = 1.0 / (1.0 + np.exp(-a))
                dm = do @ wd[:, f]
                terms = {"dw_down": do[:, i] * (a * sg * u),
                         "dw_gate": (dm * u * sg * (1.0 + a * (1.0 - sg))) * x[:, j],
                         "dw_up": (dm * a * sg) * x[:, j]}
                for key, tv in terms.items():
                    out[key][m] = tv.sum()
                    out[key + "_l1"][m] = np.abs(tv).sum()
    for n, t in enumerate(tokens):
        ds = g[t] * (dgate[n] - np.sum(g[t] * dgate[n]))
        dh[n] += ds @ w_r[np.asarray(idx[t], np.int64)]
    out["dh"] = dh
    return out


def layer_backward_channels(h, w_r, bias, k, weights, cap, dy, chans):
    """Whole gradient rows and columns of layer_backward for chosen (expert,
    channel) pairs, at O(n_e * d) cost each, so that a full-size layer stays
    within reach (same definitions, same fixed routing decision).

    For each (e, f) in chans, over the rows routed to and kept by expert e:
      dw_gate[e][f, :] = sum_r da[r, f] h_r      (row of d entries)
      dw_up[e][f, :]   = sum_r du[r, f] h_r      (row of d entries)
      dw_down[e][:, f] = sum_r do_r m[r, f]      (column of d entries)
    with a = W_gate[e] h, u = W_up[e] h, m = silu(a) * u, do = g * dy and
    dm[r, f] = do_r . W_down[e][:, f], as in layer_backward. Returns dict
    dw_gate_rows, dw_up_rows, dw_down_cols, each [len(chans), d]."""
    h = np.asarray(h, F64)
    w_r = np.asarray(w_r, F64)
    dy = np.asarray(dy, F64)
    E = w_r.shape[0]
    d = h.shape[1]
    idx, g, _, _ = route(h, w_r, bias, k)
    kept = dispatch_meta(idx, E, cap)["dest_row"] >= 0
    out = {key: np.zeros((len(chans), d)) for key in ("dw_gate_rows", "dw_up_rows", "dw_down_cols")}
    for e in sorted(set(int(c[0]) for c in chans)):
        rows, js = np.nonzero(kept & (idx == e))
        if rows.size == 0:
            continue
        wg, wu, wd = (np.asarray(w, F64) for w in weights(e))
        x = h[rows]
        do = g[rows, js, None] * dy[rows]
        for n, (ce, f) in enumerate(chans):
            if int(ce) != e:
                continue
            a = x @ wg[f]
            u = x @ wu[f]
            with np.errstate(over="ignore"):
                sg = 1.0 / (1.0 + np.exp(-a))
            dm = do @ wd[:, f]
            out["dw_gate_rows"][n] = (dm * u * sg * (1.0 + a * (1.0 - sg))) @ x
            out["dw_up_rows"][n] = (dm * a * sg) @ x
            out["dw_down_cols"][n] = do.T @ (a * sg * u)
    return out
