"""The allocation-free split attention (``prsink_attention_split_noalloc``), called through the
C ABI: for callers that cannot allocate device memory (under a runtime that owns the device's
memory pool, or in a real-time loop that may not call the allocator), its scratch is a static
array inside the library.  Its output must match the entry point that takes caller scratch
(``prsink_attention_split``), within the attention tolerance, on two calls in a row (the
array keeps the previous call's contents, so the second call checks that nothing stale is
used).  Collected last on purpose; it passes alone in a fresh process and after the others."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import pose_retrieved_kv_b200 as P
import synth
from tests._gpu import ATTN_MAX_ABS, ATTN_MEAN_ABS, attention_inputs, f64, need_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,heads", [("384x672", 40), ("480x480", 5), ("tiny", 1)])
def test_noalloc_split_matches_the_scratch_entry_point(name, heads):
    need_gpu()
    cfg = synth.preset(name, block_index=1000, valid_mask=0xFF, n_heads=heads)
    lay = P.make_layout(**cfg)
    n = P.prsink_attention_scratch_bytes(lay)
    assert 0 < n <= 20 << 20, "a split is planned and fits the static array"
    s = oracle.layout_sizes(cfg)
    q, k, v = (t.cuda() for t in attention_inputs(cfg, seed=71))
    lib = P._lib._lib
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        if call == 1:              # different inputs for the second call
            q = q.flip(0).contiguous()
        ref = torch.empty((s["L_blk"], heads, cfg["head_dim"]), dtype=torch.bfloat16,
                          device="cuda")
        P.prsink_attention_split(lay, q, k, v, ref,
                                 torch.empty(n, dtype=torch.uint8, device="cuda"))
        out = torch.full_like(ref, float("nan"))
        rc = lib.prsink_attention_split_noalloc(ctypes.byref(lay), q.data_ptr(), k.data_ptr(),
                                                v.data_ptr(), out.data_ptr(), None, None, stream)
        assert rc == P.PRSINK_OK, P.prsink_last_error()
        assert P.prsink_sync_status() == P.PRSINK_OK
        err = np.abs(f64(out) - f64(ref))
        assert np.all(np.isfinite(f64(out)))
        assert err.max() <= ATTN_MAX_ABS and err.mean() <= ATTN_MEAN_ABS, (call, err.max())
