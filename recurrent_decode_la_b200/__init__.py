"""Causal linear attention over a recurrent state, B200-native (sm_100a).

Chunkwise-parallel prefill and one-token decode, as in the slides
"Chunking, causality, and parallel prefill": per chunk of C tokens
O = tril(Q K^T) V + Q S_in and S_out = S_in + K^T V; decode is the same
mechanism for one token, S <- S + k v^T, o = q^T S.

Every step runs in the CUDA library ``liblinattn.so`` (C ABI declared in
``include/linattn.h``).  This package is a thin ctypes binding with the same
entry-point names; importing it does not load the library, the first call
does, and fails loudly when the library is missing.
"""
from .binding import (  # noqa: F401
    LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA, LA_ERR_TIMEOUT,
    LA_F32, LA_BF16, LinAttnError, lib_path, load_library,
    la_state_init, la_prefill, la_prefill_workspace_size, la_decode_step,
    la_device_status, la_status_string, la_prefill_path, la_prefill_kernel, la_resolve_chunk,
    la_selftest_wait_timeout,
)
