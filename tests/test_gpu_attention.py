"""GPU parity of ``prsink_attention`` against the float64 oracle (through the C ABI).

Tiny layouts are compared element by element over every query; the full workload sizes
(480x480, 384x672 with 3 and 4 ring slots, 672x384) run in the same launch configuration as the
benchmark and are compared on sampled query rows of every head, including the ragged last tile.
"""
import numpy as np
import pytest
import torch

import oracle
import pose_retrieved_kv_b200 as P
import synth
from tests._gpu import (LSE_MAX_ABS, attention_inputs, check_attention, f64, need_gpu)

pytestmark = pytest.mark.gpu


def _run(cfg, q, k, v, dyn_src=None):
    lay = P.make_layout(**cfg)
    s = oracle.layout_sizes(cfg)
    out = torch.full((s["L_blk"], cfg["n_heads"], cfg["head_dim"]), float("nan"),
                     dtype=torch.bfloat16, device="cuda")
    lse = torch.full((cfg["n_heads"], s["L_blk"]), float("nan"), dtype=torch.float32,
                     device="cuda")
    P.prsink_attention(lay, q.cuda(), k.cuda(), v.cuda(), out, lse,
                       None if dyn_src is None else torch.tensor([dyn_src], device="cuda"))
    assert P.prsink_sync_status() == P.PRSINK_OK
    return f64(out), f64(lse)


@pytest.mark.parametrize("b,mask", [(7, 0b111111), (0, 0b001001), (1, 0b011011),
                                    (2, 0b111111), (5, 0b101011), (9, 0b110101)])
def test_tiny_1d_every_element(b, mask):
    need_gpu()
    cfg = synth.preset("tiny", block_index=b, valid_mask=mask)
    q, k, v = attention_inputs(cfg, seed=1 + b)
    got, lse = _run(cfg, q, k, v)
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v))
    check_attention(got, ref, f"tiny b={b} mask={mask:#x}")
    assert np.abs(lse - ref_lse).max() <= LSE_MAX_ABS


SMALL_3D = [
    # several key tiles, slot boundaries inside tiles, ragged query and key tails
    dict(n_heads=3, head_dim=128, grid_h=5, grid_w=7, frames_per_block=3, ref_frames=1,
         ring_slots=3, rope_mode=3, rope_split=(44, 42, 42), rope_base=10000.0),
    dict(n_heads=2, head_dim=64, grid_h=6, grid_w=9, frames_per_block=3, ref_frames=2,
         ring_slots=4, rope_mode=3, rope_split=(24, 20, 20), rope_base=10000.0),
    dict(n_heads=2, head_dim=128, grid_h=9, grid_w=5, frames_per_block=2, ref_frames=1,
         ring_slots=2, rope_mode=3, rope_split=(40, 44, 44), rope_base=500.0),
]


@pytest.mark.parametrize("ci", range(len(SMALL_3D)))
@pytest.mark.parametrize("b,mask", [(11, 0xFF), (1, 0b0011011), (6, 0b1010111)])
def test_small_3d_every_element(ci, b, mask):
    need_gpu()
    cfg = dict(SMALL_3D[ci], block_index=b, valid_mask=mask)
    q, k, v = attention_inputs(cfg, seed=10 + ci)
    got, lse = _run(cfg, q, k, v)
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v))
    check_attention(got, ref, f"3d cfg{ci} b={b}")
    assert np.abs(lse - ref_lse).max() <= LSE_MAX_ABS


def test_no_valid_key_gives_zeros():
    need_gpu()
    cfg = synth.preset("tiny", block_index=4, valid_mask=0)
    q, k, v = attention_inputs(cfg, seed=3)
    got, lse = _run(cfg, q, k, v)
    assert np.all(got == 0) and np.all(np.isneginf(lse))


def test_device_dynamic_source_overrides_mask():
    """dyn_src < 0 on the device empties the dynamic slot whatever valid_mask says."""
    need_gpu()
    cfg = synth.preset("tiny", block_index=8, valid_mask=0b111111)
    q, k, v = attention_inputs(cfg, seed=4)
    got, _ = _run(cfg, q, k, v, dyn_src=-1)
    ref, _ = oracle.attention(dict(cfg, valid_mask=0b111011), f64(q), f64(k), f64(v))
    check_attention(got, ref, "dyn_src=-1")
    got2, _ = _run(cfg, q, k, v, dyn_src=17)
    ref2, _ = oracle.attention(cfg, f64(q), f64(k), f64(v))
    check_attention(got2, ref2, "dyn_src=17")


def test_empty_slots_holding_nan_are_ignored():
    """Bytes of empty slots never reach the output, even NaN patterns."""
    need_gpu()
    cfg = synth.preset("tiny", block_index=1, valid_mask=0b011011)
    q, k, v = attention_inputs(cfg, seed=5)
    a, e = oracle.slot_ranges(cfg)[oracle.SLOT_DYNAMIC]
    k2, v2 = k.clone(), v.clone()
    k2[:, a:e] = float("nan")
    v2[:, a:e] = float("nan")
    got, _ = _run(cfg, q, k2, v2)
    ref, _ = oracle.attention(cfg, f64(q), f64(k), f64(v))
    check_attention(got, ref, "nan in empty slot")


def _sample_rows(lblk, seed):
    g = np.random.default_rng(seed)
    edge = [0, 1, 127, 128, lblk - 13, lblk - 12, lblk - 1]
    return np.unique(np.concatenate([edge, g.choice(lblk, 40, replace=False)]))


@pytest.mark.parametrize("name", ["480x480", "384x672", "384x672_r4", "672x384"])
def test_full_size_sampled_rows(name):
    need_gpu()
    cfg = synth.preset(name, block_index=1000, valid_mask=0xFF)
    q, k, v = attention_inputs(cfg, seed=2)
    got, lse = _run(cfg, q, k, v)
    s = oracle.layout_sizes(cfg)
    rows = _sample_rows(s["L_blk"], 7)
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v), rows=rows)
    check_attention(got[rows], ref, name)
    assert np.abs(lse[:, rows] - ref_lse).max() <= LSE_MAX_ABS
    assert np.all(np.isfinite(got))


def test_full_size_early_block():
    """Block 1 at 480x480: the dynamic slot and one ring slot are empty."""
    need_gpu()
    cfg = synth.preset("480x480", block_index=1, valid_mask=0b0011011)
    q, k, v = attention_inputs(cfg, seed=6)
    got, _ = _run(cfg, q, k, v)
    rows = _sample_rows(2700, 8)
    ref, _ = oracle.attention(cfg, f64(q), f64(k), f64(v), rows=rows, heads=[0, 17, 39])
    check_attention(got[rows][:, [0, 17, 39]], ref, "480x480 b=1")
