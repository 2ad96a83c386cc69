"""Derive the stored workload constants with the oracle (test infrastructure).

many_small: the router bias of the 16 hot experts (beta) is set by bisection
so that they receive 50% of all T*k assignments on the seeded draws (experts
120..127 carry -inf and receive none). The result is written to
workloads/derived.json; both the tests and the benchmark read the stored
number.

Run:  python -m oracle.derive_workloads
"""
from __future__ import annotations

import json

import numpy as np

import workloads as W
from . import moe_oracle as O
from .cases import as64


def hot_share(s_nobias, beta, k):
    E = s_nobias.shape[1]
    b = np.zeros(E)
    b[:W.HOT_EXPERTS] = np.float32(beta)
    b[W.EMPTY_FROM:] = -np.inf
    s32, _ = O.decision_logits(s_nobias + b[None, :])
    idx = O.topk_select(s32, k)
    return float((idx < W.HOT_EXPERTS).mean())


def derive_many_small_beta(seed=0, target=0.5):
    wl = W.get("many_small")
    s = O.router_logits(as64(W.draw_h(wl, seed)), as64(W.draw_w_router(wl, seed)), None)
    lo, hi = 0.0, 8.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if hot_share(s, mid, wl.k) < target:
            lo = mid
        else:
            hi = mid
    beta = float(np.float32(hi))
    return beta, hot_share(s, beta, wl.k)


def main():
    beta, share = derive_many_small_beta()
    out = {"many_small_hot_bias": beta, "many_small_hot_share": share,
           "written_by": "python -m oracle.derive_workloads"}
    with open(W.DERIVED_PATH, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(json.dumps(out))


if __name__ == "__main__":
    main()
