"""ctypes binding of ``libprsink.so`` (the C ABI declared in ``include/prsink.h``).

Argument marshalling only: every function checks the torch tensors it is given (device, dtype,
contiguity, size), passes their data pointers and the current CUDA stream to the C entry point
of the same name, and raises :class:`PRSinkError` on a non-zero status.  All computation happens
in the library's CUDA kernels; there is no fallback of any kind.  If the library has not been
built (``python pose_retrieved_kv_b200/build.py``) importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libprsink.so")

PRSINK_OK = 0
PRSINK_ERR_ARG = -1
PRSINK_ERR_ALIGN = -2
PRSINK_ERR_LAUNCH = -3
PRSINK_ERR_TIMEOUT = -4
PRSINK_ERR_UNSUPPORTED = -5

SLOT_REF, SLOT_STATIC, SLOT_DYNAMIC, SLOT_RING0 = 0, 1, 2, 3
FP_DIM = 558
MAX_BANK = 32
MAX_RING = 8

_NAMES = {PRSINK_ERR_ARG: "PRSINK_ERR_ARG", PRSINK_ERR_ALIGN: "PRSINK_ERR_ALIGN",
          PRSINK_ERR_LAUNCH: "PRSINK_ERR_LAUNCH", PRSINK_ERR_TIMEOUT: "PRSINK_ERR_TIMEOUT",
          PRSINK_ERR_UNSUPPORTED: "PRSINK_ERR_UNSUPPORTED"}


class PRSinkError(RuntimeError):
    def __init__(self, code: int, fn: str, msg: str):
        super().__init__(f"{fn}: {_NAMES.get(code, code)}: {msg}")
        self.code = code


class Layout(ctypes.Structure):
    """Mirror of ``prsink_layout``."""
    _fields_ = [("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
                ("frames_per_block", ctypes.c_int), ("ref_frames", ctypes.c_int),
                ("ring_slots", ctypes.c_int), ("rope_mode", ctypes.c_int),
                ("rope_split", ctypes.c_int * 3), ("rope_base", ctypes.c_float),
                ("block_index", ctypes.c_longlong), ("valid_mask", ctypes.c_uint)]


BANK_FROZEN, BANK_DECAY, BANK_GATED = 0, 1, 2
BANK_MODE_NONE, BANK_MODE_STORE, BANK_MODE_BLEND = 0, 1, 2
_KINDS = {"frozen": BANK_FROZEN, "decay": BANK_DECAY, "gated": BANK_GATED}


class BankPolicy(ctypes.Structure):
    """Mirror of ``prsink_bank_policy``."""
    _fields_ = [("kind", ctypes.c_int), ("write_blocks", ctypes.c_int),
                ("alpha", ctypes.c_float), ("gate", ctypes.c_float)]


def make_policy(kind="frozen", write_blocks: int = 20, alpha: float = 0.0,
                gate: float = 0.0) -> BankPolicy:
    pol = BankPolicy()
    pol.kind = _KINDS[kind] if isinstance(kind, str) else int(kind)
    pol.write_blocks, pol.alpha, pol.gate = int(write_blocks), float(alpha), float(gate)
    return pol


def make_layout(n_heads, head_dim, grid_h, grid_w, frames_per_block=3, ref_frames=1,
                ring_slots=3, rope_mode=3, rope_split=(44, 42, 42), rope_base=10000.0,
                block_index=0, valid_mask=0xFFFFFFFF, **_ignored) -> Layout:
    lay = Layout()
    lay.n_heads, lay.head_dim = int(n_heads), int(head_dim)
    lay.grid_h, lay.grid_w = int(grid_h), int(grid_w)
    lay.frames_per_block, lay.ref_frames = int(frames_per_block), int(ref_frames)
    lay.ring_slots, lay.rope_mode = int(ring_slots), int(rope_mode)
    for i in range(3):
        lay.rope_split[i] = int(rope_split[i])
    lay.rope_base = float(rope_base)
    lay.block_index = int(block_index)
    lay.valid_mask = int(valid_mask) & 0xFFFFFFFF
    return lay


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python pose_retrieved_kv_b200/build.py` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, ll, i, f = ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int, ctypes.c_float
    lp = ctypes.POINTER(Layout)
    sig = {
        "prsink_version": ([], i),
        "prsink_last_error": ([], ctypes.c_char_p),
        "prsink_launch_count": ([], ll),
        "prsink_layout_tokens": ([lp, vp, vp, vp, vp], i),
        "prsink_attention": ([lp, vp, vp, vp, vp, vp, vp, vp], i),
        "prsink_kv_append": ([lp, vp, vp, vp, vp, i, vp], i),
        "prsink_fingerprint": ([vp, vp, vp, vp], i),
        "prsink_retrieve": ([lp, vp, vp, vp, vp, i, ll, vp, vp, vp, vp, vp, vp, i, vp], i),
        "prsink_bank_update": ([lp, vp, vp, vp, i, vp, ll, i, vp, vp, vp, i, vp], i),
        "prsink_attention_fused": ([lp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp], i),
        "prsink_attention_split": ([lp, vp, vp, vp, vp, vp, vp, vp, ll, vp], i),
        "prsink_attention_fused_split": ([lp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ll, vp], i),
        "prsink_attention_scratch_bytes": ([lp], ll),
        "prsink_attention_split_noalloc": ([lp, vp, vp, vp, vp, vp, vp, vp], i),
        "prsink_rotate_sinks": ([lp, vp, vp, ctypes.c_uint, vp, vp, vp], i),
        "prsink_retrieve_fallback": ([lp, vp, vp, i, vp, vp, vp, i, ll, vp, vp, vp, vp, vp, vp,
                                      i, vp], i),
        "prsink_bank_update_policy": ([lp, ctypes.POINTER(BankPolicy), vp, vp, vp, i, vp, ll,
                                       vp, vp, vp, vp, i, vp], i),
        "prsink_sync_status": ([vp], i),
        "prsink_debug_wait_timeout": ([ll, vp], i),
        "prsink_debug_attention_stall": ([ll], i),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def exported_symbols() -> list:
    return ["prsink_version", "prsink_last_error", "prsink_launch_count", "prsink_layout_tokens",
            "prsink_attention", "prsink_kv_append", "prsink_fingerprint", "prsink_retrieve",
            "prsink_bank_update", "prsink_sync_status", "prsink_debug_wait_timeout",
            "prsink_retrieve_fallback", "prsink_bank_update_policy", "prsink_attention_fused",
            "prsink_rotate_sinks", "prsink_debug_attention_stall", "prsink_attention_split",
            "prsink_attention_scratch_bytes", "prsink_attention_split_noalloc",
            "prsink_attention_fused_split"]


def _check(rc: int, fn: str):
    if rc != PRSINK_OK:
        raise PRSinkError(rc, fn, _lib.prsink_last_error().decode(errors="replace"))


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, numel=None, device=True) -> int:
    if t is None:
        return 0
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must hold {numel} elements, got {t.numel()}")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t.data_ptr()


def _kv_sizes(layout: Optional[Layout], M: int, n_layers: int, bank_kv, cache_kv):
    """Element counts the copy kernels address: bank_kv [n_layers][M][2][H][L_blk][d] and
    cache_kv [n_layers][2][H][T][d] (None, None when no copy is requested)."""
    if bank_kv is None and cache_kv is None and not n_layers:
        return None, None
    if layout is None:
        raise ValueError("the K/V copy needs a layout")
    _, lblk, _, T = prsink_layout_tokens(layout)
    H, d = layout.n_heads, layout.head_dim
    n_bank, n_cache = n_layers * M * 2 * H * lblk * d, n_layers * 2 * H * T * d
    # checked before any other argument: a wrong size here would make a copy kernel run past
    # the end of a buffer
    for t, name, n in ((bank_kv, "bank_kv", n_bank), (cache_kv, "cache_kv", n_cache)):
        if isinstance(t, torch.Tensor) and t.numel() != n:
            raise ValueError(f"{name} must hold {n} elements for this layout, M = {M} and "
                             f"n_layers = {n_layers}, got {t.numel()}")
    return n_bank, n_cache


def prsink_version() -> int:
    return _lib.prsink_version()


def prsink_last_error() -> str:
    return _lib.prsink_last_error().decode(errors="replace")


def prsink_launch_count() -> int:
    return _lib.prsink_launch_count()


def prsink_layout_tokens(layout: Layout):
    vals = [ctypes.c_longlong() for _ in range(4)]
    _check(_lib.prsink_layout_tokens(ctypes.byref(layout), *[ctypes.byref(v) for v in vals]),
           "prsink_layout_tokens")
    return tuple(v.value for v in vals)


def prsink_attention(layout: Layout, q, k_cache, v_cache, out, lse=None, dyn_src=None,
                     stream=None):
    _, lblk, _, T = prsink_layout_tokens(layout)
    H, d = layout.n_heads, layout.head_dim
    rc = _lib.prsink_attention(
        ctypes.byref(layout), _ptr(q, "q", torch.bfloat16, lblk * H * d),
        _ptr(k_cache, "k_cache", torch.bfloat16, H * T * d),
        _ptr(v_cache, "v_cache", torch.bfloat16, H * T * d),
        _ptr(out, "out", torch.bfloat16, lblk * H * d),
        _ptr(lse, "lse", torch.float32, H * lblk), _ptr(dyn_src, "dyn_src", torch.int64, 1),
        _stream(stream))
    _check(rc, "prsink_attention")


def prsink_attention_scratch_bytes(layout: Layout) -> int:
    n = _lib.prsink_attention_scratch_bytes(ctypes.byref(layout))
    if n < 0:
        raise PRSinkError(PRSINK_ERR_ARG, "prsink_attention_scratch_bytes", prsink_last_error())
    return n


def prsink_attention_split(layout: Layout, q, k_cache, v_cache, out, scratch, lse=None,
                           dyn_src=None, stream=None):
    """``scratch``: a uint8 CUDA tensor of at least prsink_attention_scratch_bytes bytes (None
    when that is 0)."""
    _, lblk, _, T = prsink_layout_tokens(layout)
    H, d = layout.n_heads, layout.head_dim
    rc = _lib.prsink_attention_split(
        ctypes.byref(layout), _ptr(q, "q", torch.bfloat16, lblk * H * d),
        _ptr(k_cache, "k_cache", torch.bfloat16, H * T * d),
        _ptr(v_cache, "v_cache", torch.bfloat16, H * T * d),
        _ptr(out, "out", torch.bfloat16, lblk * H * d),
        _ptr(lse, "lse", torch.float32, H * lblk), _ptr(dyn_src, "dyn_src", torch.int64, 1),
        _ptr(scratch, "scratch", torch.uint8),
        0 if scratch is None else int(scratch.numel()), _stream(stream))
    _check(rc, "prsink_attention_split")


def prsink_attention_split_noalloc(layout: Layout, q, k_cache, v_cache, out, lse=None,
                                   dyn_src=None, stream=None):
    """prsink_attention_split with the library's static scratch array (no allocation)."""
    _, lblk, _, T = prsink_layout_tokens(layout)
    H, d = layout.n_heads, layout.head_dim
    rc = _lib.prsink_attention_split_noalloc(
        ctypes.byref(layout), _ptr(q, "q", torch.bfloat16, lblk * H * d),
        _ptr(k_cache, "k_cache", torch.bfloat16, H * T * d),
        _ptr(v_cache, "v_cache", torch.bfloat16, H * T * d),
        _ptr(out, "out", torch.bfloat16, lblk * H * d),
        _ptr(lse, "lse", torch.float32, H * lblk), _ptr(dyn_src, "dyn_src", torch.int64, 1),
        _stream(stream))
    _check(rc, "prsink_attention_split_noalloc")


def prsink_attention_fused(layout: Layout, q, k_new, v_new, k_rot, k_cache, v_cache, out,
                           lse=None, dyn_src=None, stream=None, scratch=None):
    """With ``scratch`` (a uint8 CUDA tensor of prsink_attention_scratch_bytes bytes) the last
    wave is split over the key range (prsink_attention_fused_split)."""
    _, lblk, _, T = prsink_layout_tokens(layout)
    H, d = layout.n_heads, layout.head_dim
    if scratch is not None:
        rc = _lib.prsink_attention_fused_split(
            ctypes.byref(layout), _ptr(q, "q", torch.bfloat16, lblk * H * d),
            _ptr(k_new, "k_new", torch.bfloat16, lblk * H * d),
            _ptr(v_new, "v_new", torch.bfloat16, lblk * H * d),
            _ptr(k_rot, "k_rot", torch.bfloat16, H * T * d),
            _ptr(k_cache, "k_cache", torch.bfloat16, H * T * d),
            _ptr(v_cache, "v_cache", torch.bfloat16, H * T * d),
            _ptr(out, "out", torch.bfloat16, lblk * H * d),
            _ptr(lse, "lse", torch.float32, H * lblk), _ptr(dyn_src, "dyn_src", torch.int64, 1),
            _ptr(scratch, "scratch", torch.uint8), int(scratch.numel()), _stream(stream))
        _check(rc, "prsink_attention_fused_split")
        return
    rc = _lib.prsink_attention_fused(
        ctypes.byref(layout), _ptr(q, "q", torch.bfloat16, lblk * H * d),
        _ptr(k_new, "k_new", torch.bfloat16, lblk * H * d),
        _ptr(v_new, "v_new", torch.bfloat16, lblk * H * d),
        _ptr(k_rot, "k_rot", torch.bfloat16, H * T * d),
        _ptr(k_cache, "k_cache", torch.bfloat16, H * T * d),
        _ptr(v_cache, "v_cache", torch.bfloat16, H * T * d),
        _ptr(out, "out", torch.bfloat16, lblk * H * d),
        _ptr(lse, "lse", torch.float32, H * lblk), _ptr(dyn_src, "dyn_src", torch.int64, 1),
        _stream(stream))
    _check(rc, "prsink_attention_fused")


def prsink_rotate_sinks(layout: Layout, k_cache, k_rot, slot_mask: int, dyn_flag=None,
                        dyn_src=None, stream=None):
    _, _, _, T = prsink_layout_tokens(layout)
    H, d = layout.n_heads, layout.head_dim
    rc = _lib.prsink_rotate_sinks(
        ctypes.byref(layout), _ptr(k_cache, "k_cache", torch.bfloat16, H * T * d),
        _ptr(k_rot, "k_rot", torch.bfloat16, H * T * d), int(slot_mask) & 0xFFFFFFFF,
        _ptr(dyn_flag, "dyn_flag", torch.int32, 1), _ptr(dyn_src, "dyn_src", torch.int64, 1),
        _stream(stream))
    _check(rc, "prsink_rotate_sinks")


def prsink_kv_append(layout: Layout, k_new, v_new, k_cache, v_cache, dest_slot: int,
                     stream=None):
    _, lblk, lref, T = prsink_layout_tokens(layout)
    H, d = layout.n_heads, layout.head_dim
    n = lref if dest_slot == SLOT_REF else lblk
    rc = _lib.prsink_kv_append(
        ctypes.byref(layout), _ptr(k_new, "k_new", torch.bfloat16, n * H * d),
        _ptr(v_new, "v_new", torch.bfloat16, n * H * d),
        _ptr(k_cache, "k_cache", torch.bfloat16, H * T * d),
        _ptr(v_cache, "v_cache", torch.bfloat16, H * T * d), int(dest_slot), _stream(stream))
    _check(rc, "prsink_kv_append")


def prsink_fingerprint(kp, frame_ok, phi, stream=None):
    rc = _lib.prsink_fingerprint(_ptr(kp, "kp", torch.float32, FP_DIM),
                                 _ptr(frame_ok, "frame_ok", torch.uint8, 3),
                                 _ptr(phi, "phi", torch.float32, FP_DIM), _stream(stream))
    _check(rc, "prsink_fingerprint")


def prsink_retrieve(layout: Optional[Layout], phi_b, bank_phi, bank_src, bank_count, M: int,
                    exclude_block: int, r_out, score_out, copy_out, dyn_src, bank_kv=None,
                    cache_kv=None, n_layers: int = 0, stream=None):
    n_bank, n_cache = _kv_sizes(layout, M, n_layers, bank_kv, cache_kv)
    rc = _lib.prsink_retrieve(
        ctypes.byref(layout) if layout is not None else None,
        _ptr(phi_b, "phi_b", torch.float32, FP_DIM),
        _ptr(bank_phi, "bank_phi", torch.float32, M * FP_DIM),
        _ptr(bank_src, "bank_src", torch.int64, M), _ptr(bank_count, "bank_count", torch.int32, 1),
        int(M), int(exclude_block), _ptr(r_out, "r_out", torch.int32, 1),
        _ptr(score_out, "score_out", torch.float32, 1),
        _ptr(copy_out, "copy_out", torch.int32, 1), _ptr(dyn_src, "dyn_src", torch.int64, 1),
        _ptr(bank_kv, "bank_kv", torch.bfloat16, n_bank),
        _ptr(cache_kv, "cache_kv", torch.bfloat16, n_cache), int(n_layers), _stream(stream))
    _check(rc, "prsink_retrieve")


def prsink_bank_update(layout: Optional[Layout], bank_phi, bank_src, bank_count, M: int, phi_b,
                       b: int, write_blocks: int, action_out, cache_kv=None, bank_kv=None,
                       n_layers: int = 0, stream=None):
    n_bank, n_cache = _kv_sizes(layout, M, n_layers, bank_kv, cache_kv)
    rc = _lib.prsink_bank_update(
        ctypes.byref(layout) if layout is not None else None,
        _ptr(bank_phi, "bank_phi", torch.float32, M * FP_DIM),
        _ptr(bank_src, "bank_src", torch.int64, M), _ptr(bank_count, "bank_count", torch.int32, 1),
        int(M), _ptr(phi_b, "phi_b", torch.float32, FP_DIM), int(b), int(write_blocks),
        _ptr(action_out, "action_out", torch.int32, 1),
        _ptr(cache_kv, "cache_kv", torch.bfloat16, n_cache),
        _ptr(bank_kv, "bank_kv", torch.bfloat16, n_bank), int(n_layers), _stream(stream))
    _check(rc, "prsink_bank_update")


def prsink_retrieve_fallback(layout: Optional[Layout], phi_b, frame_ok, min_detected: int,
                             bank_phi, bank_src, bank_count, M: int, exclude_block: int, r_out,
                             score_out, copy_out, dyn_src, bank_kv=None, cache_kv=None,
                             n_layers: int = 0, stream=None):
    n_bank, n_cache = _kv_sizes(layout, M, n_layers, bank_kv, cache_kv)
    rc = _lib.prsink_retrieve_fallback(
        ctypes.byref(layout) if layout is not None else None,
        _ptr(phi_b, "phi_b", torch.float32, FP_DIM), _ptr(frame_ok, "frame_ok", torch.uint8, 3),
        int(min_detected), _ptr(bank_phi, "bank_phi", torch.float32, M * FP_DIM),
        _ptr(bank_src, "bank_src", torch.int64, M), _ptr(bank_count, "bank_count", torch.int32, 1),
        int(M), int(exclude_block), _ptr(r_out, "r_out", torch.int32, 1),
        _ptr(score_out, "score_out", torch.float32, 1),
        _ptr(copy_out, "copy_out", torch.int32, 1), _ptr(dyn_src, "dyn_src", torch.int64, 1),
        _ptr(bank_kv, "bank_kv", torch.bfloat16, n_bank),
        _ptr(cache_kv, "cache_kv", torch.bfloat16, n_cache), int(n_layers), _stream(stream))
    _check(rc, "prsink_retrieve_fallback")


def prsink_bank_update_policy(layout: Optional[Layout], policy: BankPolicy, bank_phi, bank_src,
                              bank_count, M: int, phi_b, b: int, action_out, mode_out,
                              cache_kv=None, bank_kv=None, n_layers: int = 0, stream=None):
    n_bank, n_cache = _kv_sizes(layout, M, n_layers, bank_kv, cache_kv)
    rc = _lib.prsink_bank_update_policy(
        ctypes.byref(layout) if layout is not None else None, ctypes.byref(policy),
        _ptr(bank_phi, "bank_phi", torch.float32, M * FP_DIM),
        _ptr(bank_src, "bank_src", torch.int64, M), _ptr(bank_count, "bank_count", torch.int32, 1),
        int(M), _ptr(phi_b, "phi_b", torch.float32, FP_DIM), int(b),
        _ptr(action_out, "action_out", torch.int32, 1), _ptr(mode_out, "mode_out", torch.int32, 1),
        _ptr(cache_kv, "cache_kv", torch.bfloat16, n_cache),
        _ptr(bank_kv, "bank_kv", torch.bfloat16, n_bank), int(n_layers), _stream(stream))
    _check(rc, "prsink_bank_update_policy")


def prsink_sync_status(stream=None) -> int:
    """Synchronise and return the status code (0 or PRSINK_ERR_TIMEOUT); does not raise."""
    return _lib.prsink_sync_status(_stream(stream))


def prsink_debug_wait_timeout(timeout_ns: int, stream=None):
    _check(_lib.prsink_debug_wait_timeout(int(timeout_ns), _stream(stream)),
           "prsink_debug_wait_timeout")


def prsink_debug_attention_stall(timeout_ns: int):
    _check(_lib.prsink_debug_attention_stall(int(timeout_ns)), "prsink_debug_attention_stall")


def prsink_attention_fused_split(layout: Layout, q, k_new, v_new, k_rot, k_cache, v_cache, out,
                                 scratch, lse=None, dyn_src=None, stream=None):
    """prsink_attention_fused with the last wave split over the key range; ``scratch`` a uint8
    CUDA tensor of prsink_attention_scratch_bytes(layout) bytes."""
    if scratch is None:
        raise ValueError("prsink_attention_fused_split needs scratch")
    prsink_attention_fused(layout, q, k_new, v_new, k_rot, k_cache, v_cache, out, lse, dyn_src,
                           stream, scratch=scratch)
