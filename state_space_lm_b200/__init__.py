"""B200-native (sm_100a) Mamba-3 selective scan.

The compute lives in the CUDA library built from ``csrc/`` (see ``build.py``);
``m3`` is its thin ctypes binding, ``autograd`` wraps the forward and the
backward as one differentiable call, and ``inputs`` holds the seeded
synthetic input generators.  Importing the package does not load the library; the first call
does, and fails loudly if it has not been built.
"""
from . import m3  # noqa: F401
from .m3 import (  # noqa: F401
    M3Error, discretize, rope_bc, siso_chunked_fwd, mimo_chunked_fwd, step_decode,
    workspace_bytes, launch_count, limits, chunked_bwd,
)
from .autograd import mamba3_scan  # noqa: F401
