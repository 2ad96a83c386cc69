"""Full-size dispatch parity on every workload's own routes (GPU).

For each workload, at its full size and in the configuration bench.py times:

  1. moe_route (through the C ABI) must pick exactly the oracle's experts, slot
     by slot, and its gates must equal the oracle's gate formula evaluated on
     the kernel's own fp32 scores within TOL_GATE = 1e-5 relative. With the
     same scores on both sides, this pins the kernel's softmax over the picks
     (its exp, sum and division) rather than the router GEMM's rounding.
  2. moe_permute (through the C ABI) on the router's own topk_idx must give
     the oracle's routed counts, kept counts, offsets, every dest_row entry
     (so every capacity drop decision) and perm_src, bit for bit, and every
     kept x_perm row must be the token row h[perm_src[r]] bitwise. In the
     padded layout the padding rows must be zero.

Sources: the inverse-permutation and counts checks follow archcrux
"moe-unpermute-wrong-token" (its test plan) and "MoE Token Dispatch: Why an
All-Reduce Result Does Not Describe the Exchange" ("Follow one documented
dispatch and return path"); capacity resolved in token order follows "How
Does Mixture-of-Experts Routing Affect LLM Repeatability?".
"""
import numpy as np
import pytest
import torch

import combine_router_gemm_softmax_b200 as M
import oracle as O
import workloads as W
from oracle import cases
from oracle import check as C

from gpu_cases import DEV, cfg_for, np64, np_

pytestmark = pytest.mark.gpu

FULL = ["mixtral_scaled", "skewed", "skewed_capacity", "skewed_capacity_padded", "mixtral_8x7b", "many_small",
        "many_small_identity"]


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    torch.cuda.set_device(0)
    M.lib()


def _gates_from_scores(logits_gpu, idx):
    """The oracle's gate formula (softmax over all E, renormalised over the
    picks) evaluated on the kernel's own fp32 scores."""
    return O.gates(np.asarray(logits_gpu, np.float64), idx)


@pytest.mark.parametrize("name", FULL)
def test_full_size_route_and_dispatch_bit_exact(name):
    wl = W.get(name)
    inp = cases.parity_inputs(wl, 0, weights=False)
    h64 = cases.as64(inp.h)
    ref_idx, _, ref_s, _ = O.route(h64, cases.as64(inp.w_router), cases.as64(inp.bias), wl.k)
    cfg = cfg_for(wl)
    h = inp.h.to(DEV)
    wr = inp.w_router.to(DEV)
    bias = None if inp.bias is None else inp.bias.to(DEV)
    logits = torch.empty((wl.T, wl.E), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx, gate = M.moe_route(cfg, h, wr, bias, logits_out=logits, status=status)
    torch.cuda.synchronize()

    # 1. routes identical first, so everything below compares identical routes
    idx_np = np_(idx)
    assert np.array_equal(idx_np, ref_idx)
    s_gpu = np64(logits)
    assert C.logits_match(s_gpu, ref_s)
    g_ref = _gates_from_scores(s_gpu, idx_np)
    g = np64(gate)
    assert np.all(np.abs(g - g_ref) <= C.TOL_GATE * g_ref + 1e-12), float(np.abs(g - g_ref).max())

    # 2. the dispatch of those routes
    padded = wl.layout == "padded"
    meta = O.dispatch_meta_padded(idx_np, wl.E, wl.capacity) if padded else O.dispatch_meta(idx_np, wl.E,
                                                                                              wl.capacity)
    out = M.moe_permute(cfg, h, idx, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np_(out["routed_counts"]).tolist() == meta["routed"].tolist()
    assert np_(out["counts"]).tolist() == meta["kept"].tolist()
    assert np_(out["offsets"]).tolist() == meta["offsets"].tolist()
    assert np.array_equal(np_(out["dest_row"]), meta["dest_row"])           # every drop decision
    n_rows = wl.E * wl.capacity if padded else int(meta["offsets"][-1])
    ps = np_(out["perm_src"])[:n_rows]
    assert np.array_equal(ps, meta["perm_src"])
    if wl.capacity >= 0:
        assert int(meta["kept"].sum()) < wl.T * wl.k                         # this workload drops
    kept_rows = np.nonzero(meta["perm_src"] >= 0)[0]
    xp = out["x_perm"][:n_rows]
    src = torch.from_numpy(meta["perm_src"][kept_rows]).to(DEV)
    rows = torch.from_numpy(kept_rows).to(DEV)
    for c0 in range(0, len(kept_rows), 16384):                              # bounded temporaries
        sl = slice(c0, c0 + 16384)
        assert torch.equal(xp[rows[sl]].view(torch.int16), h[src[sl]].view(torch.int16))
    if padded:
        pad = torch.from_numpy(np.nonzero(meta["perm_src"] < 0)[0]).to(DEV)
        assert bool((xp[pad] == 0).all())
