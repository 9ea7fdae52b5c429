"""Sol-Attn on B200: query-adaptive block-sparse attention (sm_100a CUDA).

The compute path is the C-ABI library ``libsolattn.so`` built from ``csrc/``;
``abi`` is its thin ctypes binding.  Importing this package does not load the
library, so the input generator (``synthetic``) is usable on machines without
a GPU.
"""

__version__ = "0.1.0"

BLOCK = 64
