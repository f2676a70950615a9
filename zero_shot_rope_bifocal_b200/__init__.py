"""B200 (sm_100a) library for Jet-Long's bifocal-RoPE attention.

The compute lives in ``libjetlong.so`` (C ABI in ``include/jetlong.h``); the
``jetlong`` module is its Python binding.  Importing the package loads
nothing: the library is opened on the first call, which raises if it has not
been built (``python -m zero_shot_rope_bifocal_b200.build``).
"""
from .jetlong import (  # noqa: F401
    JL_BF16,
    JL_F32,
    JetLongError,
    jetlong_decode,
    jetlong_decode_interp,
    jetlong_decode_two_form,
    jetlong_decode_workspace_size,
    jetlong_device_status,
    jetlong_group_size,
    jetlong_prefill,
    jetlong_prefill_attend,
    jetlong_prefill_interp,
    jetlong_prefill_chunk,
    jetlong_prefill_chunk_interp,
    jetlong_prefill_chunk_workspace_size,
    jetlong_prefill_rotate,
    jetlong_prefill_three_pass,
    jetlong_prefill_three_pass_workspace_size,
    jetlong_prefill_workspace_size,
    jetlong_remote_cache,
    jetlong_rope_cache,
)

__version__ = "0.1.0"
