"""fp64 CPU oracle for the Mamba-3 selective scan.

TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports this package.
"""
from .oracle import (  # noqa: F401
    build_oracle, discretize, rope_bc, siso_loop, mimo_loop, siso_chunked,
    step_decode, mimo_step_decode, step_decode_factored, loop_bwd, GRAD_NAMES, oracle_lib_path,
    oracle_source_path, compile_source, use_library,
)
from .chunked_bwd import chunked_bwd  # noqa: F401
