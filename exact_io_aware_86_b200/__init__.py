"""Exact IO-aware attention on B200 (sm_100a).

Entry points, all running entirely in this package's CUDA library
(``libfa.so``, C ABI declared in ``include/fa.h``):

* ``prefill`` / ``fa_prefill``: causal or full attention over packed
  variable-length sequences with grouped kv heads, computed tile by tile with
  an online softmax on the tcgen05 tensor cores.
* ``decode_paged`` / ``fa_decode_paged``: one query token per request against
  a paged KV cache, split along the context and merged by log-sum-exp.
* ``prefill_fp8`` / ``fa_prefill_fp8``: the prefill on e4m3 inputs with
  descale factors, both products in FP8 on the tensor cores.
* ``decode_paged_append`` / ``fa_decode_paged_append``: the same after
  appending the new token's key and value to the cache, with optional RoPE.

The Python layer only marshals arguments.  Importing the package loads
nothing; the first call loads ``libfa.so`` and raises if it is missing.
"""
from .api import (  # noqa: F401
    FAError,
    decode_append_workspace_size,
    decode_auto_splits,
    decode_paged,
    decode_paged_append,
    decode_paged_f32,
    decode_workspace_size,
    device_error,
    error_string,
    fa_decode_paged,
    fa_decode_paged_append,
    fa_prefill,
    fa_prefill_fp8,
    load_library,
    prefill,
    prefill_f32,
    prefill_fp8,
)
