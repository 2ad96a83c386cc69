"""moe_permute_static_scratch, the permute entry point for callers that
cannot allocate device memory, against moe_permute (GPU).

Such callers (code whose host framework or memory pool owns all device
memory, or a path that must not allocate) cannot pass a workspace; the
library then keeps the permute scratch in its own fixed 1 MiB device array.
Its results must be bit-identical to moe_permute's, also on a second call
that finds the previous call's leftovers in that array.
"""
import numpy as np
import pytest
import torch

import combine_router_gemm_softmax_b200 as M

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _case(T, d, E, k, cap, seed):
    r = np.random.default_rng(seed)
    h = torch.from_numpy(r.standard_normal((T, d)).astype(np.float32)).to(torch.bfloat16).to(DEV)
    rows = []
    for t in range(T):
        if t % 3 == 0:                                     # expert 0 is hot: every third token picks it first
            rows.append(np.concatenate([[0], r.permutation(np.arange(1, E))[:k - 1]]))
        else:
            rows.append(r.permutation(E)[:k])
    idx = np.stack(rows).astype(np.int32)
    return M.config(T, d, E, k, 128, capacity=cap), h, torch.from_numpy(idx).to(DEV)


def _same(a, b, n):
    for key in ("routed_counts", "counts", "offsets", "dest_row"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["perm_src"][:n], b["perm_src"][:n])
    assert torch.equal(a["x_perm"][:n].view(torch.int16), b["x_perm"][:n].view(torch.int16))


def test_static_scratch_matches_workspace_permute_on_consecutive_calls():
    torch.cuda.set_device(0)
    # the second call is smaller and uses other experts, so it runs on top of
    # the first call's leftovers in the shared array
    for T, d, E, k, cap, seed in ((4097, 256, 64, 6, -1, 1), (1000, 128, 8, 2, 200, 2)):
        cfg, h, idx = _case(T, d, E, k, cap, seed)
        st_a = torch.zeros(1, dtype=torch.int32, device=DEV)
        st_b = torch.zeros(1, dtype=torch.int32, device=DEV)
        ref = M.moe_permute(cfg, h, idx, status=st_a)
        got = M.moe_permute_static_scratch(cfg, h, idx, status=st_b)
        torch.cuda.synchronize()
        _same(ref, got, int(ref["offsets"][-1].item()))
        assert int(st_a.item()) == int(st_b.item()) == 0


def test_static_scratch_rejects_problems_beyond_its_array():
    cfg = M.config(65537, 128, 256, 2, 128)               # E * ceil(T/128) = 256 * 513 > 131072
    rc = M.lib().moe_permute_static_scratch(__import__("ctypes").byref(cfg), None, None, None, None, None, None,
                                            None, None, None, None)
    assert rc == M.MOE_ERR_WORKSPACE
    ok = M.config(65536, 128, 256, 2, 128)
    assert M.moe_workspace_size(ok, M.MOE_OP_PERMUTE) <= 1 << 20
