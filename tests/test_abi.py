"""The C ABI library loads, exports every symbol ``include/prsink.h`` declares, and rejects
invalid arguments on the host before launching anything (CPU only: no compute call)."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import pose_retrieved_kv_b200 as P
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "prsink.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(prsink_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("prsink_attention", "prsink_kv_append", "prsink_retrieve", "prsink_bank_update",
              "prsink_fingerprint", "prsink_sync_status"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(P.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", P.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (prsink_\w+)", out))
    assert set(_declared()) <= exported
    assert set(P.exported_symbols()) <= exported


def test_build_targets_sm100a():
    from pose_retrieved_kv_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_layout_tokens_match_slot_arithmetic():
    for name, T in [("tiny", 256), ("480x480", 14400), ("384x672", 16128), ("384x672_r4", 19152)]:
        lay = P.make_layout(**synth.preset(name))
        L_f, L_blk, L_ref, TT = P.prsink_layout_tokens(lay)
        assert TT == T and L_blk == 3 * L_f and L_ref == L_f


@pytest.mark.parametrize("bad", [dict(n_heads=0), dict(ring_slots=0), dict(ring_slots=9),
                                 dict(rope_split=(44, 42, 40)), dict(rope_split=(43, 43, 42)),
                                 dict(rope_mode=2), dict(block_index=-1), dict(rope_base=0.0)])
def test_invalid_layout_rejected(bad):
    lay = P.make_layout(**{**synth.preset("480x480"), **bad})
    with pytest.raises(P.PRSinkError) as e:
        P.prsink_layout_tokens(lay)
    assert e.value.code == P.PRSINK_ERR_ARG


def _lib():
    return P._lib._lib


def test_null_and_range_errors_do_not_launch():
    lib = _lib()
    lay = P.make_layout(**synth.preset("tiny"))
    before = P.prsink_launch_count()
    assert lib.prsink_attention(ctypes.byref(lay), None, None, None, None, None, None,
                                None) == P.PRSINK_ERR_ARG
    assert lib.prsink_kv_append(ctypes.byref(lay), 16, 16, 16, 16, 99, None) == P.PRSINK_ERR_ARG
    assert lib.prsink_kv_append(ctypes.byref(lay), 16, 16, 16, 16, -1, None) == P.PRSINK_ERR_ARG
    assert lib.prsink_kv_append(ctypes.byref(lay), 17, 16, 16, 16, 3, None) == P.PRSINK_ERR_ALIGN
    assert lib.prsink_attention(ctypes.byref(lay), 16, 16, 16, 24, None, None,
                                None) == P.PRSINK_ERR_ALIGN
    lay96 = P.make_layout(**{**synth.preset("tiny"), "head_dim": 96, "rope_split": (96, 0, 0)})
    assert lib.prsink_attention(ctypes.byref(lay96), 16, 16, 16, 16, None, None,
                                None) == P.PRSINK_ERR_UNSUPPORTED
    assert lib.prsink_retrieve(None, 16, 16, 16, 16, 0, 0, 16, 16, 16, 16, None, None, 0,
                               None) == P.PRSINK_ERR_ARG          # M = 0
    assert lib.prsink_retrieve(None, 16, 16, 16, 16, 33, 0, 16, 16, 16, 16, None, None, 0,
                               None) == P.PRSINK_ERR_ARG          # M > 32
    assert lib.prsink_retrieve(None, 16, 16, 16, 16, 5, 0, 16, 16, 16, 16, 16, None, 1,
                               None) == P.PRSINK_ERR_ARG          # copy without a layout
    assert lib.prsink_bank_update(ctypes.byref(lay), 16, 16, 16, 5, 16, -1, 20, 16, None,
                                  None, 0, None) == P.PRSINK_ERR_ARG   # b < 0
    assert lib.prsink_fingerprint(None, 16, 16, None) == P.PRSINK_ERR_ARG
    assert P.prsink_launch_count() == before
    assert "null" in P.prsink_last_error() or P.prsink_last_error()


def test_rope_table_limit_reported():
    # 1-D RoPE over a large frame needs a table that does not fit in shared memory
    lay = P.make_layout(**{**synth.preset("480x480"), "rope_mode": 1, "rope_split": (128, 0, 0)})
    assert _lib().prsink_attention(ctypes.byref(lay), 16, 16, 16, 16, None, None,
                                   None) == P.PRSINK_ERR_UNSUPPORTED


def test_build_module_loads_without_the_package():
    """build() must work on a fresh checkout, where the library does not exist yet: loading
    the build script may not import the package (whose import loads the library)."""
    code = ("import sys, __graft_entry__ as g; m = g._build_module(); "
            "assert callable(m.build) and m.ARCH; "
            "assert 'pose_retrieved_kv_b200' not in sys.modules, 'package imported'")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_copy_buffers_sized_for_the_layout_or_rejected_before_launch():
    """The dynamic fill and the bank store address bank_kv and cache_kv from the layout, M and
    n_layers alone: the binding checks both sizes on the host before anything is launched."""
    import torch
    cfg = synth.preset("tiny")
    lay = P.make_layout(**cfg)
    _, lblk, _, T = P.prsink_layout_tokens(lay)
    M, n_layers = 5, 2
    f32 = lambda n: torch.zeros(n, dtype=torch.float32)       # noqa: E731
    i32 = lambda n: torch.zeros(n, dtype=torch.int32)         # noqa: E731
    i64 = lambda n: torch.zeros(n, dtype=torch.int64)         # noqa: E731
    bf = lambda n: torch.zeros(n, dtype=torch.bfloat16)       # noqa: E731
    good_bank, good_cache = n_layers * M * 2 * lblk * 64, n_layers * 2 * T * 64
    before = P.prsink_launch_count()
    for bank_n, cache_n, what in [(good_bank - 64, good_cache, "bank_kv"),
                                  (good_bank, good_cache + 64, "cache_kv"),
                                  (n_layers * 4 * 2 * lblk * 64, good_cache, "bank_kv")]:
        with pytest.raises(ValueError, match=what):
            P.prsink_retrieve(lay, f32(558), f32(M * 558), i64(M), i32(1), M, 0, i32(1),
                              None, i32(1), i64(1), bf(bank_n), bf(cache_n), n_layers)
        with pytest.raises(ValueError, match=what):
            P.prsink_bank_update(lay, f32(M * 558), i64(M), i32(1), M, f32(558), 0, 20,
                                 i32(1), bf(cache_n), bf(bank_n), n_layers)
    # a wrong n_layers for the given buffers
    with pytest.raises(ValueError, match="bank_kv"):
        P.prsink_retrieve(lay, f32(558), f32(M * 558), i64(M), i32(1), M, 0, i32(1), None,
                          i32(1), i64(1), bf(good_bank), bf(good_cache), n_layers + 1)
    # right sizes on host tensors: rejected for the device, not for the size
    with pytest.raises(ValueError, match="CUDA"):
        P.prsink_retrieve(lay, f32(558), f32(M * 558), i64(M), i32(1), M, 0, i32(1), None,
                          i32(1), i64(1), bf(good_bank), bf(good_cache), n_layers)
    assert P.prsink_launch_count() == before


def test_split_scratch_plan_sizes():
    """The split of the last wave, as planned for a 148-SM device (the count a B200 reports;
    without a GPU the planner assumes it): 384x672 leaves 36 units in its last wave -> 4 shares
    each; 480x480 fills its last wave (144 of 148) -> no split."""
    def size(name, **kw):
        return P.prsink_attention_scratch_bytes(P.make_layout(**synth.preset(name, **kw)))
    r, S, rows, d = 36, 4, 256, 128
    want = r * S * rows * d * 4 + r * S * rows * 8 + 256
    assert size("384x672") == want
    assert size("480x480") == 0
    assert size("480x480", n_heads=5) > 0             # 55 units < 148: every unit split
