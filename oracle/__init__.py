"""CPU oracle for the FLUX.3 Image Klein denoiser hot path.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, float64 NumPy
restatement of what the pages describe. Only the test suite, the package
smoke check and the benchmark's CPU-baseline leg may import it; the product
path (the CUDA library and its Python binding) never does and shares no code
with it.

Parity status of each function is stated in its docstring; the one part that
cannot be pinned to anything outside this package is the match to the real
trained model (no weights or printed intermediate values exist), so that
comparison is "parity unpinned".
"""
from .klein import *  # noqa: F401,F403
