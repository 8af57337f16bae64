"""GPU parity of ``prsink_attention_split`` (the last wave's units split over the key range,
partials combined by the last CTA of each unit) against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import pose_retrieved_kv_b200 as P
import synth
from tests._cases import sample_rows
from tests._gpu import LSE_MAX_ABS, attention_inputs, check_attention, f64, need_gpu

pytestmark = pytest.mark.gpu

SMALL3D = dict(n_heads=3, head_dim=128, grid_h=5, grid_w=7, frames_per_block=3, ref_frames=1,
               ring_slots=3, rope_mode=3, rope_split=(44, 42, 42), rope_base=10000.0)


def _split(cfg, q, k, v, scratch=None, reps=2):
    lay = P.make_layout(**cfg)
    s = oracle.layout_sizes(cfg)
    H, d = cfg["n_heads"], cfg["head_dim"]
    n = P.prsink_attention_scratch_bytes(lay)
    if scratch is None and n:
        scratch = torch.empty(n, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(reps):                       # twice: the arrival counters must start over
        out = torch.full((s["L_blk"], H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((H, s["L_blk"]), float("nan"), dtype=torch.float32, device="cuda")
        P.prsink_attention_split(lay, q.cuda(), k.cuda(), v.cuda(), out, scratch, lse)
        assert P.prsink_sync_status() == P.PRSINK_OK
        outs.append((f64(out), f64(lse)))
    assert np.array_equal(outs[0][0], outs[1][0])
    return outs[0][0], outs[0][1], n


@pytest.mark.parametrize("name,heads,b,mask", [("384x672", 40, 1000, 0xFF),
                                               ("384x672_r4", 40, 1001, 0xFF),
                                               ("672x384", 40, 999, 0xFF),
                                               ("480x480", 5, 1000, 0xFF),
                                               ("480x480", 5, 1, 0b0011011)])
def test_split_full_size(name, heads, b, mask):
    need_gpu()
    cfg = synth.preset(name, block_index=b, valid_mask=mask, n_heads=heads)
    q, k, v = attention_inputs(cfg, seed=41)
    got, lse, n = _split(cfg, q, k, v)
    assert n > 0, "a split is planned for this layout"
    s = oracle.layout_sizes(cfg)
    rows = sample_rows(s["L_blk"], 12)
    hs = sorted({0, heads - 3, heads - 2, heads - 1})   # the last heads hold the split units
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v), rows=rows, heads=hs)
    check_attention(got[rows][:, hs], ref, f"split {name}")
    assert np.abs(lse[hs][:, rows] - ref_lse).max() <= LSE_MAX_ABS
    assert np.all(np.isfinite(got))


@pytest.mark.parametrize("cfg,b,mask", [(dict(synth.PRESETS["tiny"]), 7, 0xFF),
                                        (dict(synth.PRESETS["tiny"]), 1, 0b011011),
                                        (SMALL3D, 11, 0xFF), (SMALL3D, 6, 0b1010111)])
def test_split_small_every_element(cfg, b, mask):
    need_gpu()
    cfg = dict(cfg, block_index=b, valid_mask=mask)
    q, k, v = attention_inputs(cfg, seed=42)
    got, lse, n = _split(cfg, q, k, v)
    assert n > 0
    ref, ref_lse = oracle.attention(cfg, f64(q), f64(k), f64(v))
    check_attention(got, ref, "split small")
    assert np.abs(lse - ref_lse).max() <= LSE_MAX_ABS


def test_split_without_a_planned_split_is_plain_attention():
    """480x480 with 40 heads fills its last wave (440 units): no scratch, the plain kernel."""
    need_gpu()
    cfg = synth.preset("480x480", block_index=1000, valid_mask=0xFF)
    assert P.prsink_attention_scratch_bytes(P.make_layout(**cfg)) == 0
    q, k, v = attention_inputs(cfg, seed=43)
    got, _, _ = _split(cfg, q, k, v, reps=2)
    out = torch.empty((2700, 40, 128), dtype=torch.bfloat16, device="cuda")
    P.prsink_attention(P.make_layout(**cfg), q.cuda(), k.cuda(), v.cuda(), out)
    assert np.array_equal(got, f64(out))


def test_split_rejects_small_scratch():
    need_gpu()
    cfg = synth.preset("384x672", block_index=1000, valid_mask=0xFF)
    lay = P.make_layout(**cfg)
    n = P.prsink_attention_scratch_bytes(lay)
    q = torch.zeros((3024, 40, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((40, 16128, 128), dtype=torch.bfloat16, device="cuda")
    small = torch.empty(n - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(P.PRSinkError):
        P.prsink_attention_split(lay, q, kv, kv, q.clone(), small)


@pytest.mark.parametrize("name,heads,b,mask", [("480x480", 5, 1000, 0xFF),
                                               ("480x480", 5, 1, 0b0011011),
                                               ("384x672", 40, 1002, 0xFF)])
def test_fused_split_is_append_then_attention(name, heads, b, mask):
    """The fused call with the last wave split: outputs as the oracle's append + attention,
    the block's raw K/V in its ring slot exactly once (cache bytes bit for bit)."""
    need_gpu()
    cfg = synth.preset(name, block_index=b, valid_mask=mask, n_heads=heads)
    s = oracle.layout_sizes(cfg)
    H, d = heads, 128
    q, k, v = attention_inputs(cfg, seed=44)
    kn = synth.normal_bf16((s["L_blk"], H, d), 44, 7)
    vn = synth.normal_bf16((s["L_blk"], H, d), 44, 8)
    lay = P.make_layout(**cfg)
    kd, vd = k.cuda(), v.cuda()
    k_rot = torch.empty_like(kd)
    P.prsink_rotate_sinks(lay, kd, k_rot, 0xFFFF)
    n = P.prsink_attention_scratch_bytes(lay)
    assert n > 0
    scratch = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.full((s["L_blk"], H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, s["L_blk"]), float("nan"), dtype=torch.float32, device="cuda")
    P.prsink_attention_fused_split(lay, q.cuda(), kn.cuda(), vn.cuda(), k_rot, kd, vd, out,
                                   scratch, lse)
    assert P.prsink_sync_status() == P.PRSINK_OK
    ring = oracle.SLOT_RING0 + b % cfg["ring_slots"]
    k2, v2 = oracle.kv_append(cfg, f64(kn), f64(vn), f64(k), f64(v), ring)
    assert np.array_equal(f64(kd), k2) and np.array_equal(f64(vd), v2)
    rows = sample_rows(s["L_blk"], 13)
    hs = sorted({0, heads - 2, heads - 1})
    ref, ref_lse = oracle.attention(dict(cfg, valid_mask=mask | (1 << ring)), f64(q), k2, v2,
                                    rows=rows, heads=hs)
    check_attention(f64(out)[rows][:, hs], ref, f"fused split {name}")
    assert np.abs(f64(lse)[hs][:, rows] - ref_lse).max() <= LSE_MAX_ABS
