"""B200 (sm_100a) multi-token-prediction draft-head library.

The hot path -- the embed+hidden combiner, the draft lm_head sweep fused with a
(masked) argmax over BF16 / FP8 per-row / NVFP4 tables, the two weight quantizers
and the drafter-context prefill -- runs in hand-written CUDA kernels behind the C ABI
of ``include/mtp.h`` (``libmtp.so``). ``_lib`` is the ctypes binding with the same
entry-point names; ``api`` allocates buffers with torch and calls it.
"""
from . import _lib  # noqa: F401
from ._lib import MtpError, load  # noqa: F401
