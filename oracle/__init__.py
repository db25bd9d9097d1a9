"""CPU oracle for the ternary group-scaled products (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference legs import this
package. The product path (gemm_tern_gemv_b200) never does.
"""
from .tern_oracle import *  # noqa: F401,F403
from .rotate_oracle import BLOCK as ROTATE_BLOCK, hadamard, rotate, rotate_tolerance, sign_diagonal  # noqa: F401
