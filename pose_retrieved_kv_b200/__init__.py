"""B200 (sm_100a) library for LiveAnimate's PR-Sink per-block step.

The compute path is ``libprsink.so`` (hand-written CUDA, C ABI in ``include/prsink.h``);
this package is its thin Python binding (``_lib``) plus the host-side bookkeeping of a stream
(``stream.PRSinkStream``).  PyTorch only supplies device memory and streams.
"""
from ._lib import (  # noqa: F401
    FP_DIM, MAX_BANK, MAX_RING, PRSINK_ERR_ALIGN, PRSINK_ERR_ARG, PRSINK_ERR_LAUNCH,
    PRSINK_ERR_TIMEOUT, PRSINK_ERR_UNSUPPORTED, PRSINK_OK, SLOT_DYNAMIC, SLOT_REF, SLOT_RING0,
    SLOT_STATIC, LIB_PATH, Layout, PRSinkError, exported_symbols, make_layout,
    prsink_attention, prsink_bank_update, prsink_debug_wait_timeout, prsink_fingerprint,
    prsink_kv_append, prsink_last_error, prsink_launch_count, prsink_layout_tokens,
    prsink_retrieve, prsink_sync_status, prsink_version, BANK_DECAY, BANK_FROZEN, BANK_GATED,
    BANK_MODE_BLEND, BANK_MODE_NONE, BANK_MODE_STORE, BankPolicy, make_policy,
    prsink_bank_update_policy, prsink_retrieve_fallback, prsink_attention_fused,
    prsink_rotate_sinks, prsink_debug_attention_stall, prsink_attention_split,
    prsink_attention_scratch_bytes, prsink_attention_split_noalloc, prsink_attention_fused_split)
from .stream import PRSinkStream, stream_valid_mask  # noqa: F401
