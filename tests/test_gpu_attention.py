"""GPU parity of ``prsink_attention`` against the float64 oracle (through the C ABI).

Tiny layouts are compared element by element over every query; the full workload sizes
(480x480, 384x672 with 3 and 4 ring slots, 672x384) run in the same launch configuration as the
benchmark and are compared on sampled query rows of every head, including the ragged last tile,
and on every row of a few heads.
"""
import numpy as np
import pytest
import torch

import oracle
import pose_retrieved_kv_b200 as P
import synth
from tests._gpu import (ATTN_MAX_ABS, ATTN_MEAN_ABS, LSE_MAX_ABS, attention_inputs,
                        check_attention, f64, need_gpu)
from tests._cases import (GAIN_CASES, RESCALE_CASES, gain_case, rescale_case,
                          sample_rows)
from tests._probe import probe_inputs
from tests._rounding import model_errors, rescaled_rows

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


# Inputs whose logits reach far beyond those of N(0,1) draws exceed the stated tolerance
# through the bf16 rounding of the rotated q and k alone (tests/_rounding.py; pinned on the CPU
# in tests/test_rounding_model.py): there the bound is 1.25 x the rounding model's error on the
# same inputs, and the stated tolerance where that is larger.
MODEL_FACTOR = 1.25


def _model_bounds(cfg, q, k, v, rows, ref, ref_lse):
    emax, emean, else_ = model_errors(cfg, f64(q), f64(k), f64(v), rows, ref, ref_lse)
    return (max(ATTN_MAX_ABS, MODEL_FACTOR * emax), max(ATTN_MEAN_ABS, MODEL_FACTOR * emean),
            max(LSE_MAX_ABS, MODEL_FACTOR * else_))


@pytest.mark.parametrize("S,sign", [(5.0, -1.0), (60.0, -1.0), (900.0, -1.0), (60.0, 1.0),
                                    (900.0, 1.0)])
def test_scores_far_from_zero(S, sign):
    """Every score about sign * S (tests/_probe.py): the running max must follow rows whose
    scores are all large negative or large positive (a max stuck at 0 underflows every weight
    and returns LSE = -inf, O = 0)."""
    need_gpu()
    cfg = synth.preset("tiny", block_index=7, valid_mask=0xFF)
    q, k, v = probe_inputs(cfg, S, seed=3, sign=sign)
    got, lse = _run(cfg, q, k, v)
    rows = np.arange(48)
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v))
    bmax, bmean, blse = _model_bounds(cfg, q, k, v, rows, ref, ref_lse)
    assert np.all(np.isfinite(lse))
    assert np.abs(lse - ref_lse).max() <= blse
    err = np.abs(got - ref)
    assert err.max() <= bmax and err.mean() <= bmean, (err.max(), err.mean(), bmax, bmean)
    assert np.abs(got).max() > 0.1 * np.abs(ref).max()        # not an all-zero output


@pytest.mark.parametrize("name,slot,gain", GAIN_CASES)
def test_max_growing_or_shrinking_across_tiles(name, slot, gain):
    """Keys of one slot scaled by `gain` (logits up to ~24): when it is the last slot the row
    max grows by far more than 2^8 between key tiles, so the output accumulator is rescaled
    mid-row; when it is the ref slot (first tiles) later tiles sit far below the max."""
    need_gpu()
    cfg, q, k, v, rows = gain_case(name, slot, gain)
    got, lse = _run(cfg, q, k, v)
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v), rows=rows)
    bmax, bmean, blse = _model_bounds(cfg, q, k, v, rows, ref, ref_lse)
    err = np.abs(got[rows] - ref)
    assert np.all(np.isfinite(got))
    assert err.max() <= bmax and err.mean() <= bmean, (err.max(), err.mean(), bmax, bmean)
    assert np.abs(lse[:, rows] - ref_lse).max() <= blse


@pytest.mark.parametrize("name,gain", RESCALE_CASES)
def test_rescale_path_at_stated_tolerance(name, gain):
    """Logits below ~10 whose row max still jumps by more than 2^8 between key tiles on a good
    share of rows (counted on the CPU from the oracle's scores in the kernel's tile order): the
    accumulator rescale is exercised under the stated tolerance itself."""
    need_gpu()
    cfg, q, k, v, rows = rescale_case(name, gain)
    assert np.mean(np.concatenate([rescaled_rows(cfg, f64(q), f64(k), rows, h)
                                   for h in range(cfg["n_heads"])])) >= 0.15
    got, lse = _run(cfg, q, k, v)
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v), rows=rows)
    check_attention(got[rows], ref, f"rescale {name}")
    assert np.abs(lse[:, rows] - ref_lse).max() <= LSE_MAX_ABS


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


@pytest.mark.parametrize("name", ["480x480", "384x672", "384x672_r4", "672x384"])
def test_full_size_sampled_rows(name):
    need_gpu()
    cfg = synth.preset(name, block_index=1000, valid_mask=0xFF)
    q, k, v = attention_inputs(cfg, seed=2)
    got, lse = _run(cfg, q, k, v)
    s = oracle.layout_sizes(cfg)
    rows = sample_rows(s["L_blk"], 7)
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v), rows=rows)
    check_attention(got[rows], ref, name)
    assert np.abs(lse[:, rows] - ref_lse).max() <= LSE_MAX_ABS
    assert np.all(np.isfinite(got))


@pytest.mark.parametrize("name,heads", [("480x480", [0, 13, 26, 39]),
                                        ("384x672_r4", [0, 39])])
def test_full_size_every_row_of_some_heads(name, heads):
    """Every query row (every query tile, the ragged last one included) of a few heads at the
    full workload size, in the launch configuration the benchmark times (all 40 heads)."""
    need_gpu()
    cfg = synth.preset(name, block_index=1000, valid_mask=0xFF)
    q, k, v = attention_inputs(cfg, seed=2)
    got, lse = _run(cfg, q, k, v)
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v), heads=heads)
    check_attention(got[:, heads], ref, f"{name} all rows")
    assert np.abs(lse[heads] - ref_lse).max() <= LSE_MAX_ABS


def test_full_size_early_block():
    """Block 1 at 480x480: the dynamic slot and one ring slot are empty."""
    need_gpu()
    cfg = synth.preset("480x480", block_index=1, valid_mask=0b0011011)
    q, k, v = attention_inputs(cfg, seed=6)
    got, _ = _run(cfg, q, k, v)
    rows = sample_rows(2700, 8)
    ref, _ = oracle.attention(cfg, f64(q), f64(k), f64(v), rows=rows, heads=[0, 17, 39])
    check_attention(got[rows][:, [0, 17, 39]], ref, "480x480 b=1")


# Position probe (tests/_probe.py): correctly rotated keys all score -S; a key rotated at a
# wrong position takes over the output (a one-column shift of one key moves the output by
# 0.36 at the tiny layout and 2.9 at 480x480).  Legitimate rounding (bf16 rotated q and k, bf16
# P) stays below 0.015 and 0.006 on these inputs, so the bounds below separate the two.
PROBES = [
    ("tiny", 300.0, 1, 7, 0xFF, 0.05),
    ("tiny", 300.0, 1, 1, 0b011011, 0.05),
    ("480x480", 1000.0, 2, 1000, 0xFF, 0.03),
    ("480x480", 1000.0, 2, 4, 0b0111011, 0.03),
    ("384x672_r4", 1000.0, 2, 1001, 0xFF, 0.03),
    ("672x384", 1000.0, 2, 999, 0xFF, 0.03),
]


@pytest.mark.parametrize("name,S,H,b,mask,bound", PROBES)
def test_every_key_rotated_at_its_position(name, S, H, b, mask, bound):
    need_gpu()
    cfg = synth.preset(name, block_index=b, valid_mask=mask, n_heads=H)
    q, k, v = probe_inputs(cfg, S)
    got, lse = _run(cfg, q, k, v)
    s = oracle.layout_sizes(cfg)
    rows = np.unique(np.concatenate([np.arange(0, s["L_blk"], 37), [s["L_blk"] - 1]]))
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v), rows=rows)
    err = np.abs(got[rows] - ref)
    assert err.max() <= bound, f"{name} b={b}: max {err.max():.3e}"
    # every score is about -S here: the running max must follow negative scores (an output of
    # zeros would also be within `bound` at large T; the LSE is not)
    assert np.all(np.isfinite(lse[:, rows]))
    assert np.abs(lse[:, rows] - ref_lse).max() <= 1e-3 * S, f"{name}: LSE"
