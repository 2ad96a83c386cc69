"""CPU oracle for the token-choice MoE layer forward.

TEST INFRASTRUCTURE ONLY. Only tests/, the smoke check in __graft_entry__ and
the CPU-baseline leg of bench.py may import or run anything in this package.
The product path (the CUDA library and its binding) never does, and this
package never imports the product.

Every function is pinned by CPU tests against facts fixed outside the oracle
itself (worked examples printed on the pages, closed forms, brute force,
library routines on reducible special cases). None is unpinned.
"""
from .moe_oracle import *  # noqa: F401,F403
