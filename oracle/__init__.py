"""CPU oracle for the SVDQuant W4A4 (NVFP4) linear layer and the AWQ W4A16
weight-only layer used beside it.

TEST INFRASTRUCTURE ONLY. A plain, slow, float64 restatement of what the
layer computes, used to check the CUDA library. Only the test suite, the
smoke check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py``
may import it; the library itself never imports, links or calls anything
here, and nothing here imports the library.

Parity pins (tests/test_oracle_*.py) tie each function to something other
than itself: the OCP FP8 anchor values and torch's float8_e4m3fn conversion,
the E2M1 grid, brute-force nearest-value searches, the Eckart-Young theorem,
the r = 0 and r = full special cases, and a pure-Python 16x16 triple loop.
"""
from . import awq, nvfp4, svdq  # noqa: F401
