"""Pins of the oracle's slot layout, ring order, positions and RoPE (CPU only).

Each check ties the oracle to something other than itself: constants the pages print, closed
forms of a plane rotation, invariants (rotations keep norms, relative positions decide scores,
every logical position is used once) and independent re-derivations on tiny inputs.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from tests._pages import pages_constants


def test_pages_constants_match_oracle():
    c = pages_constants()
    assert int(c["fingerprint_dim"]) == oracle.FP_DIM
    assert (int(c["fingerprint_frames"]) * int(c["fingerprint_keypoints"])
            * int(c["fingerprint_channels"])) == int(c["fingerprint_dim"])
    assert int(c["ring_slots"]) == synth.PRESETS["480x480"]["ring_slots"]
    assert int(c["latent_frames_per_block"]) == synth.PRESETS["480x480"]["frames_per_block"]


@pytest.mark.parametrize("name,T,lblk", [
    ("tiny", 256, 48), ("480x480", 14400, 2700), ("384x672", 16128, 3024),
    ("672x384", 16128, 3024), ("384x672_r4", 19152, 3024)])
def test_layout_sizes(name, T, lblk):
    # key counts of the workload list: ref 1 frame + static + dynamic + R ring blocks
    s = oracle.layout_sizes(synth.preset(name))
    assert s["T"] == T and s["L_blk"] == lblk
    rng = oracle.slot_ranges(synth.preset(name))
    assert rng[0][0] == 0 and rng[-1][1] == T
    assert all(a[1] == b[0] for a, b in zip(rng, rng[1:]))


@pytest.mark.parametrize("R", [1, 2, 3, 4, 5])
def test_ring_rank_is_age_order(R):
    for b in range(0, 3 * R + 2):
        ranks = [oracle.ring_rank(s, b, R) for s in range(R)]
        assert sorted(ranks) == list(range(R))            # a permutation
        assert oracle.ring_rank(b % R, b, R) == R - 1     # current block is the newest
        for s in range(R):                                # slot s holds block b-R+1+rank
            held = b - R + 1 + ranks[s]
            assert held % R == s
        if b > 0:                                         # one block later every slot ages by 1
            prev = [oracle.ring_rank(s, b - 1, R) for s in range(R)]
            for s in range(R):
                if s != b % R:
                    assert ranks[s] == prev[s] - 1


@pytest.mark.parametrize("name", ["tiny", "480x480", "384x672", "672x384", "384x672_r4"])
@pytest.mark.parametrize("b", [0, 1, 2, 7, 1000])
def test_positions_tile_the_logical_layout(name, b):
    """Every logical (frame, token) is held by exactly one physical row, and the queries sit on
    the newest ring slot."""
    cfg = synth.preset(name, block_index=b, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    pos, valid = oracle.key_positions(cfg)
    qpos = oracle.query_positions(cfg)
    if cfg["rope_mode"] == 1:
        assert sorted(pos.tolist()) == list(range(s["T"]))
        lin = pos
        qlin = qpos
    else:
        gh, gw = cfg["grid_h"], cfg["grid_w"]
        assert pos[:, 1].min() == 0 and pos[:, 1].max() == gh - 1
        assert pos[:, 2].min() == 0 and pos[:, 2].max() == gw - 1
        lin = pos[:, 0] * s["L_f"] + pos[:, 1] * gw + pos[:, 2]
        qlin = qpos[:, 0] * s["L_f"] + qpos[:, 1] * gw + qpos[:, 2]
        assert sorted(lin.tolist()) == list(range(s["T"]))
    # queries = the rows held by the current block's ring slot, in the same order
    a, e = oracle.slot_ranges(cfg)[oracle.SLOT_RING0 + b % cfg["ring_slots"]]
    assert np.array_equal(qlin, lin[a:e])
    assert qlin.min() == s["T"] - s["L_blk"]


def test_rope_closed_forms():
    """Rotation of basis vectors gives (cos a, sin a) and (-sin a, cos a); frequencies are
    base^(-2j/d) per axis."""
    cfg = dict(head_dim=4, rope_mode=1, rope_base=10000.0, rope_split=(4, 0, 0))
    for pos in (0, 1, 3, 17):
        e0 = oracle.rope_rotate(cfg, np.array([1.0, 0.0, 0.0, 1.0]), np.array(pos))
        a0, a1 = pos * 1.0, pos * 0.01      # theta_0 = 1, theta_1 = 10000^(-1/2)
        assert e0 == pytest.approx([math.cos(a0), math.sin(a0), -math.sin(a1), math.cos(a1)],
                                   abs=1e-15)
    cfg3 = dict(head_dim=8, rope_mode=3, rope_base=100.0, rope_split=(4, 2, 2))
    x = np.zeros(8)
    x[4] = 1.0                               # first pair of the h axis (d_a = 2, theta = 1)
    y = oracle.rope_rotate(cfg3, x, np.array([5, 2, 9]))
    assert y[4:6] == pytest.approx([math.cos(2.0), math.sin(2.0)], abs=1e-15)
    assert np.all(y[[0, 1, 2, 3, 6, 7]] == 0)
    x = np.zeros(8)
    x[2] = 1.0                               # second pair of the t axis: theta = 100^(-2/4)
    y = oracle.rope_rotate(cfg3, x, np.array([5, 2, 9]))
    assert y[2:4] == pytest.approx([math.cos(0.5), math.sin(0.5)], abs=1e-15)


def test_rope_position_zero_is_identity_and_norm_kept():
    cfg = synth.preset("480x480")
    x = np.random.default_rng(0).standard_normal((64, 128))
    assert np.array_equal(oracle.rope_rotate(cfg, x, np.zeros((64, 3), dtype=np.int64)), x)
    pos = np.random.default_rng(1).integers(0, 40, size=(64, 3))
    y = oracle.rope_rotate(cfg, x, pos)
    assert np.linalg.norm(y, axis=1) == pytest.approx(np.linalg.norm(x, axis=1), rel=1e-14)
    # pairwise: each interleaved pair keeps its own norm
    assert (y[:, 0::2] ** 2 + y[:, 1::2] ** 2) == pytest.approx(x[:, 0::2] ** 2 + x[:, 1::2] ** 2,
                                                                rel=1e-13)


@pytest.mark.parametrize("name", ["tiny", "480x480"])
def test_rope_relative_invariance(name):
    """q~ . k~ depends only on the position difference: shifting every position of one axis by
    the same constant leaves all scores unchanged."""
    cfg = synth.preset(name)
    d = cfg["head_dim"]
    g = np.random.default_rng(2)
    q = g.standard_normal((16, d))
    k = g.standard_normal((24, d))
    if cfg["rope_mode"] == 1:
        qp, kp = g.integers(0, 300, 16), g.integers(0, 300, 24)
        shifts = [np.int64(37)]
    else:
        qp, kp = g.integers(0, 30, (16, 3)), g.integers(0, 30, (24, 3))
        shifts = [np.array([5, 0, 0]), np.array([0, 11, 0]), np.array([0, 0, 3]),
                  np.array([2, 7, 13])]
    s0 = oracle.rope_rotate(cfg, q, qp) @ oracle.rope_rotate(cfg, k, kp).T
    for sh in shifts:
        s1 = oracle.rope_rotate(cfg, q, qp + sh) @ oracle.rope_rotate(cfg, k, kp + sh).T
        assert np.max(np.abs(s1 - s0)) <= 1e-10


def test_valid_mask_early_blocks():
    cfg = synth.preset("480x480")
    # block 0: ref + its own ring slot; block 1: + static + ring slot 1; steady state: all
    assert oracle.valid_mask(cfg, 0, False) == 0b0001001
    assert oracle.valid_mask(cfg, 1, False) == 0b0011011
    assert oracle.valid_mask(cfg, 2, True) == 0b0111111
    assert oracle.valid_mask(cfg, 1000, True) == 0b0111111
    cfg4 = synth.preset("384x672_r4")
    assert oracle.valid_mask(cfg4, 2, True) == 0b0111111
    assert oracle.valid_mask(cfg4, 3, True) == 0b1111111
