"""GPU parity of the sink pre-rotation (``prsink_rotate_sinks``) and of the attention with the
append folded in (``prsink_attention_fused``) against the oracle, through the C ABI.

The fused call must equal the oracle's kv_append of the block into its ring slot followed by
the oracle's attention: cache bytes bit for bit (the raw block lands in its ring slot, no other
byte changes), outputs within the attention tolerance.  The rotated copy must hold each key
rotated at its current position, within one bf16 rounding of the oracle's rotation."""
import numpy as np
import pytest
import torch

import oracle
import pose_retrieved_kv_b200 as P
import synth
from tests._cases import sample_rows
from tests._gpu import LSE_MAX_ABS, attention_inputs, check_attention, f64, need_gpu
from tests._rounding import bf16

pytestmark = pytest.mark.gpu

ALL = 0xFFFF


def _rotate(cfg, k, mask=ALL, dyn_flag=None, dyn_src=None, k_rot=None):
    kd = k.cuda()
    kr = torch.full_like(kd, float("nan")) if k_rot is None else k_rot
    P.prsink_rotate_sinks(P.make_layout(**cfg), kd, kr, mask, dyn_flag, dyn_src)
    assert P.prsink_sync_status() == P.PRSINK_OK
    return kr


def _check_rotated(got, ref, what):
    """The kernel rotates in float32 (cos / sin tables rounded from float64) and rounds once to
    bf16: it equals the oracle's rotation rounded to bf16 except where the float32 error crosses
    a rounding boundary, and then by one bf16 unit (or a tiny absolute amount near zero)."""
    ref16 = bf16(ref)
    d = np.abs(got - ref16)
    assert np.mean(d == 0) > 0.99, (what, np.mean(d == 0))
    assert np.all(d <= 2.0 ** -7 * np.abs(ref16) + 1e-6), (what, d.max())


def _rotated_ref(cfg, k):
    kpos, _ = oracle.key_positions(cfg)
    return np.stack([oracle.rope_rotate(cfg, f64(k)[h], kpos) for h in range(cfg["n_heads"])])


@pytest.mark.parametrize("name,b,mask", [("tiny", 7, 0xFF), ("tiny", 1, 0b011011),
                                         ("480x480", 1000, 0xFF), ("384x672_r4", 1001, 0xFF)])
def test_rotated_copy_holds_keys_at_their_positions(name, b, mask):
    need_gpu()
    cfg = synth.preset(name, block_index=b, valid_mask=mask)
    if name != "tiny":
        cfg = dict(cfg, n_heads=3)
    q, k, v = attention_inputs(cfg, seed=21)
    kr = f64(_rotate(cfg, k))
    ref = _rotated_ref(cfg, k)
    cur = oracle.SLOT_RING0 + b % cfg["ring_slots"]
    for slot, (a, e) in enumerate(oracle.slot_ranges(cfg)):
        if slot == cur or not (mask >> slot) & 1:
            continue
        _check_rotated(kr[:, a:e], ref[:, a:e], f"slot {slot}")


def test_rotation_mask_and_dynamic_predicates():
    """Only the requested slots are written: the dynamic slot is skipped when the refill flag is
    0 or the slot is empty; the current block's ring slot is never written."""
    need_gpu()
    cfg = synth.preset("tiny", block_index=7, valid_mask=0xFF)
    q, k, v = attention_inputs(cfg, seed=22)
    ranges = oracle.slot_ranges(cfg)
    cur = oracle.SLOT_RING0 + 7 % 3
    ref = _rotated_ref(cfg, k)
    zero = torch.zeros(1, dtype=torch.int32, device="cuda")
    one = torch.ones(1, dtype=torch.int32, device="cuda")
    empty = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    full = torch.full((1,), 5, dtype=torch.int64, device="cuda")
    for flag, src, dyn_written in [(zero, full, False), (one, full, True), (one, empty, False),
                                   (None, None, True)]:
        # slots 1 and 2 (static, dynamic) share tiles with nothing else requested at tiny size
        kr = f64(_rotate(cfg, k, mask=(1 << oracle.SLOT_DYNAMIC), dyn_flag=flag, dyn_src=src))
        a, e = ranges[oracle.SLOT_DYNAMIC]
        assert np.all(np.isnan(kr[:, a:e])) != dyn_written
        if dyn_written:
            _check_rotated(kr[:, a:e], ref[:, a:e], "dynamic")
    kr = f64(_rotate(cfg, k, mask=ALL))
    a, e = ranges[cur]
    # the current slot's rows are only written where they share a tile with rotated slots
    tile_rows = set()
    for slot, (sa, se) in enumerate(ranges):
        if slot != cur:
            tile_rows |= {t for t in range(sa // 128, (se - 1) // 128 + 1)}
    untouched = [r for r in range(a, e) if r // 128 not in tile_rows]
    assert all(np.all(np.isnan(kr[:, r])) for r in untouched)


FUSED_CASES = [("tiny", 7, 0xFF), ("tiny", 1, 0b011011), ("tiny", 2, 0b101111),
               ("small3d", 11, 0xFF), ("small3d", 4, 0b1010111), ("two_tiles", 5, 0xFF),
               ("two_tiles", 9, 0b1011111), ("480x480", 1000, 0xFF),
               ("480x480", 1, 0b0011011), ("384x672_r4", 1002, 0xFF), ("672x384", 999, 0xFF)]
SMALL3D = dict(n_heads=3, head_dim=128, grid_h=5, grid_w=7, frames_per_block=3, ref_frames=1,
               ring_slots=3, rope_mode=3, rope_split=(44, 42, 42), rope_base=10000.0)
# 192 queries: one CTA per head stores both of the block's key tiles (consecutive stores)
TWO_TILES = dict(SMALL3D, n_heads=2, grid_h=8, grid_w=8)


@pytest.mark.parametrize("name,b,mask", FUSED_CASES)
def test_fused_attention_is_append_then_attention(name, b, mask):
    need_gpu()
    if name in ("small3d", "two_tiles"):
        cfg = dict(SMALL3D if name == "small3d" else TWO_TILES, block_index=b, valid_mask=mask)
    else:
        cfg = synth.preset(name, block_index=b, valid_mask=mask)
    if name in ("480x480", "384x672_r4", "672x384"):
        cfg = dict(cfg, n_heads=4)
    s = oracle.layout_sizes(cfg)
    H, d = cfg["n_heads"], cfg["head_dim"]
    q, k, v = attention_inputs(cfg, seed=23)
    kn = synth.normal_bf16((s["L_blk"], H, d), 23, 7)
    vn = synth.normal_bf16((s["L_blk"], H, d), 23, 8)
    ring = oracle.SLOT_RING0 + b % cfg["ring_slots"]
    kd, vd = k.cuda(), v.cuda()
    k_rot = _rotate(cfg, k)
    k_rot0 = k_rot.clone()
    lay = P.make_layout(**cfg)
    out = torch.full((s["L_blk"], H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, s["L_blk"]), float("nan"), dtype=torch.float32, device="cuda")
    P.prsink_attention_fused(lay, q.cuda(), kn.cuda(), vn.cuda(), k_rot, kd, vd, out, lse)
    assert P.prsink_sync_status() == P.PRSINK_OK
    k2, v2 = oracle.kv_append(cfg, f64(kn), f64(vn), f64(k), f64(v), ring)
    assert np.array_equal(f64(kd), k2) and np.array_equal(f64(vd), v2)
    assert torch.equal(k_rot.view(torch.int16), k_rot0.view(torch.int16))   # read only
    rows = np.arange(s["L_blk"]) if s["L_blk"] <= 300 else sample_rows(s["L_blk"], 4)
    cfg_v = dict(cfg, valid_mask=mask | (1 << ring))
    ref, ref_lse = oracle.attention(cfg_v, f64(q), k2, v2, rows=rows)
    check_attention(f64(out)[rows], ref, f"fused {name} b={b}")
    assert np.abs(f64(lse)[:, rows] - ref_lse).max() <= LSE_MAX_ABS


def test_fused_with_nan_in_unread_rows():
    """Bytes the fused call must not use: NaN in k_rot's current-slot and empty-slot rows, in
    v_cache's current-slot rows (overwritten) and empty-slot rows."""
    need_gpu()
    cfg = dict(SMALL3D, block_index=4, valid_mask=0b1011011)   # dynamic empty, ring 1 empty
    s = oracle.layout_sizes(cfg)
    H, d = cfg["n_heads"], cfg["head_dim"]
    q, k, v = attention_inputs(cfg, seed=24)
    kn = synth.normal_bf16((s["L_blk"], H, d), 24, 7)
    vn = synth.normal_bf16((s["L_blk"], H, d), 24, 8)
    ring = oracle.SLOT_RING0 + 4 % 3
    k_rot = _rotate(cfg, k)
    v_nan = v.clone()
    for slot in (oracle.SLOT_DYNAMIC, oracle.SLOT_RING0 + 1, ring):
        a, e = oracle.slot_ranges(cfg)[slot]
        k_rot[:, a:e] = float("nan")
        v_nan[:, a:e] = float("nan")
    kd, vd = k.cuda(), v_nan.cuda()
    out = torch.empty((s["L_blk"], H, d), dtype=torch.bfloat16, device="cuda")
    P.prsink_attention_fused(P.make_layout(**cfg), q.cuda(), kn.cuda(), vn.cuda(), k_rot, kd, vd,
                             out)
    assert P.prsink_sync_status() == P.PRSINK_OK
    k2, v2 = oracle.kv_append(cfg, f64(kn), f64(vn), f64(k), f64(v), ring)
    ref, _ = oracle.attention(dict(cfg, valid_mask=cfg["valid_mask"] | (1 << ring)), f64(q), k2,
                              v2)
    check_attention(f64(out), ref, "fused nan")


def test_fused_stream_matches_the_unfused_stream():
    """A whole stream through PRSinkStream(fused=True) against the same stream unfused: identical
    decisions and cache / bank bytes at every block, attention outputs within twice the
    tolerance of each other (each is within the tolerance of the oracle)."""
    need_gpu()
    cfg = dict(SMALL3D, n_heads=2)
    n_layers, n_blocks = 2, 26
    a = P.PRSinkStream(cfg, n_layers=n_layers, M=5, write_blocks=20)
    f = P.PRSinkStream(cfg, n_layers=n_layers, M=5, write_blocks=20, fused=True)
    s = oracle.layout_sizes(cfg)
    for layer in range(n_layers):
        kr = synth.normal_bf16((s["L_ref"], 2, 128), 60 + layer, 1).cuda()
        a.set_ref(layer, kr, kr)
        f.set_ref(layer, kr, kr)
    kp, ok, _ = synth.pose_stream(13, n_blocks)
    oa = torch.empty((s["L_blk"], 2, 128), dtype=torch.bfloat16, device="cuda")
    of = torch.empty_like(oa)
    worst = 0.0
    for b in range(n_blocks):
        kpd = torch.from_numpy(np.ascontiguousarray(kp[b][:, :62])).cuda()
        okd = torch.from_numpy(ok[b]).cuda()
        a.begin_block(kpd, okd)
        f.begin_block(kpd, okd)
        for layer in range(n_layers):
            for p in range(4):
                q, kn, vn = (synth.normal_bf16((s["L_blk"], 2, 128), 3000 + 10 * b + p, j).cuda()
                             for j in range(3))
                a.layer_pass(layer, q, kn, vn, oa, clean=p == 3)
                f.layer_pass(layer, q, kn, vn, of, clean=p == 3)
                worst = max(worst, float((oa.float() - of.float()).abs().max()))
        a.end_block()
        f.end_block()
        da = (int(a.r.item()), int(a.copied.item()), int(a.action.item()))
        df = (int(f.r.item()), int(f.copied.item()), int(f.action.item()))
        assert da == df, b
        assert torch.equal(a.cache_kv, f.cache_kv), b
    assert P.prsink_sync_status() == P.PRSINK_OK
    assert torch.equal(a.bank_kv, f.bank_kv)
    assert worst <= 2 * 2e-2, worst
