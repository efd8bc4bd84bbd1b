"""fp64 CPU oracle for kernelized linear attention.

TEST INFRASTRUCTURE: only tests/, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of bench.py may import it. The CUDA path never does,
and the two share no code. Every function is pinned by tests that run without
a GPU (tests/test_oracle_pins.py); no function here is "parity unpinned".
"""

from .linear_attention import *  # noqa: F401,F403
from .metrics import max_row_grad_err, max_row_rel_err  # noqa: F401
from .backward import backward_batched, backward_dense, phi_grad  # noqa: F401
