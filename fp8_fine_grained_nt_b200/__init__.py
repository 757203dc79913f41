"""FP8 (E4M3) NT GEMM with fine-grained scaling and BF16 output, for B200 (sm_100a).

The compute lives in a C-ABI shared library (``libfp8nt.so``, declared in
``include/fp8_nt.h``); ``binding`` marshals torch tensors into its calls.  The
library is loaded on first use and a missing or unloadable library raises: there
is no CPU fallback.
"""

from .binding import *  # noqa: F401,F403
from .binding import __all__  # noqa: F401
