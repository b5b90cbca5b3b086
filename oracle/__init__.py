"""fp64 CPU oracle for the Mamba-2 SSD layer -- test infrastructure only.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg may import
this package.  The CUDA library never imports, links or calls it.
"""
from .oracle import (  # noqa: F401
    recurrence,
    quadratic,
    chunked,
    default_threads,
)
from .frontend import frontend, causal_conv, softplus, silu  # noqa: F401,E402
