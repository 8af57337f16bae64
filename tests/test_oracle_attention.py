"""Pins of the oracle's PR-Sink attention (CPU only).

* an independent pure-Python re-derivation on tiny layouts: the logical sequence is gathered
  block by block (ref, static, dynamic, ring blocks b-R+1..b in age order), positions are the
  logical token indices, rotation is complex multiplication, softmax is the textbook one;
* softmax rows sum to one and vanish on invalid slots;
* special cases: zero queries average the valid values, one valid key returns its value,
  no valid key returns zeros;
* the attention is unchanged when every slot is moved to another physical place as long as the
  logical layout is kept (ring rotation with the block index);
* on the tiny layout the float64 oracle agrees with an independent long-double computation to
  1e-12 (its own rounding, nothing more).
"""
import cmath
import math

import numpy as np
import pytest

import oracle
import synth


def _sizes(cfg):
    lf = cfg["grid_h"] * cfg["grid_w"]
    return lf, cfg["frames_per_block"] * lf, cfg["ref_frames"] * lf


def _logical_rows(cfg):
    """Physical row of each logical key, in logical order, with its validity.

    Written from the slot diagram directly: ref rows first, then the static block, the dynamic
    block, then the ring blocks from oldest (b-R+1) to newest (b), block b' living in ring slot
    b' mod R.
    """
    lf, lblk, lref = _sizes(cfg)
    R = cfg["ring_slots"]
    b = cfg["block_index"]
    m = cfg["valid_mask"]
    rows = []
    rows += [(r, bool(m & 1)) for r in range(lref)]
    rows += [(lref + r, bool(m & 2)) for r in range(lblk)]
    rows += [(lref + lblk + r, bool(m & 4)) for r in range(lblk)]
    for bb in range(b - R + 1, b + 1):
        s = bb % R
        start = lref + (2 + s) * lblk
        rows += [(start + r, bool(m & (8 << s))) for r in range(lblk)]
    return rows


def _rotate(cfg, x, idx):
    """Rotate list ``x`` at logical token index ``idx`` by complex multiplication per pair."""
    lf, _, _ = _sizes(cfg)
    d = cfg["head_dim"]
    base = cfg["rope_base"]
    if cfg["rope_mode"] == 1:
        axes = [(0, d, idx)]
    else:
        t, tok = divmod(idx, lf)
        h, w = divmod(tok, cfg["grid_w"])
        a, bb, c = cfg["rope_split"]
        axes = [(0, a, t), (a, bb, h), (a + bb, c, w)]
    out = list(x)
    for off, da, p in axes:
        for j in range(da // 2):
            z = complex(x[off + 2 * j], x[off + 2 * j + 1]) * cmath.exp(1j * p * base ** (-2 * j / da))
            out[off + 2 * j], out[off + 2 * j + 1] = z.real, z.imag
    return out


def _brute_attention(cfg, q, k, v):
    lf, lblk, _ = _sizes(cfg)
    d = cfg["head_dim"]
    rows = _logical_rows(cfg)
    n_log = len(rows)
    out = np.zeros((lblk, cfg["n_heads"], d))
    for h in range(cfg["n_heads"]):
        keys = [(_rotate(cfg, list(k[h][r]), i), list(v[h][r]))
                for i, (r, ok) in enumerate(rows) if ok]
        for qi in range(lblk):
            qr = _rotate(cfg, list(q[qi][h]), n_log - lblk + qi)
            sc = [sum(a * b for a, b in zip(qr, kr)) / math.sqrt(d) for kr, _ in keys]
            mx = max(sc)
            w = [math.exp(s - mx) for s in sc]
            tot = sum(w)
            for dd in range(d):
                out[qi, h, dd] = sum(wi * vv[dd] for wi, (_, vv) in zip(w, keys)) / tot
    return out


def _inputs(cfg, seed):
    lf, lblk, lref = _sizes(cfg)
    T = lref + (2 + cfg["ring_slots"]) * lblk
    H, d = cfg["n_heads"], cfg["head_dim"]
    q = synth.normal_bf16((lblk, H, d), seed, 0).double().numpy()
    k = synth.normal_bf16((H, T, d), seed, 1).double().numpy()
    v = synth.normal_bf16((H, T, d), seed, 2).double().numpy()
    return q, k, v


SMALL_3D = dict(n_heads=2, head_dim=12, grid_h=2, grid_w=3, frames_per_block=2, ref_frames=1,
                ring_slots=3, rope_mode=3, rope_split=(4, 4, 4), rope_base=10000.0)


@pytest.mark.parametrize("b,mask", [(7, 0b111111), (1, 0b011011), (0, 0b001001),
                                    (5, 0b101011)])
def test_tiny_1d_matches_bruteforce(b, mask):
    cfg = synth.preset("tiny", block_index=b, valid_mask=mask)
    q, k, v = _inputs(cfg, seed=1)
    got, lse = oracle.attention(cfg, q, k, v)
    ref = _brute_attention(cfg, q, k, v)
    assert np.max(np.abs(got - ref)) <= 1e-12
    assert np.all(np.isfinite(lse))


@pytest.mark.parametrize("b,mask,R", [(4, 0b111111, 3), (9, 0b110101, 3), (6, 0b1111111, 4),
                                      (2, 0b0110111, 4)])
def test_small_3d_matches_bruteforce(b, mask, R):
    cfg = dict(SMALL_3D, block_index=b, valid_mask=mask, ring_slots=R)
    q, k, v = _inputs(cfg, seed=3)
    got, _ = oracle.attention(cfg, q, k, v)
    ref = _brute_attention(cfg, q, k, v)
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_softmax_rows_sum_to_one_and_skip_invalid():
    cfg = synth.preset("tiny", block_index=9, valid_mask=0b101101)
    q, k, _ = _inputs(cfg, seed=4)
    p, valid = oracle.attention_probs(cfg, q, k, head=0)
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(p[:, ~valid] == 0)
    assert np.all(p[:, valid] > 0)


def test_lse_matches_probabilities():
    cfg = synth.preset("tiny", block_index=9, valid_mask=0b111111)
    q, k, v = _inputs(cfg, seed=5)
    out, lse = oracle.attention(cfg, q, k, v)
    p, valid = oracle.attention_probs(cfg, q, k, head=0)
    # out = P V, and exp(score - lse) = P for every valid key
    assert np.max(np.abs(out[:, 0, :] - p @ v[0])) <= 1e-12
    kpos, _ = oracle.key_positions(cfg)
    qr = oracle.rope_rotate(cfg, q[:, 0, :], oracle.query_positions(cfg))
    kr = oracle.rope_rotate(cfg, k[0], kpos)
    sc = qr @ kr.T / math.sqrt(cfg["head_dim"])
    assert np.max(np.abs(np.exp(sc[:, valid] - lse[0][:, None]) - p[:, valid])) <= 1e-12


def test_zero_queries_average_the_valid_values():
    cfg = synth.preset("tiny", block_index=3, valid_mask=0b110011)
    q, k, v = _inputs(cfg, seed=6)
    out, lse = oracle.attention(cfg, np.zeros_like(q), k, v)
    _, valid = oracle.key_positions(cfg)
    assert np.max(np.abs(out[:, 0, :] - v[0][valid].mean(axis=0))) <= 1e-13
    assert np.allclose(lse, math.log(valid.sum()), atol=1e-13)


def test_single_valid_key_returns_its_value():
    cfg = dict(n_heads=3, head_dim=16, grid_h=1, grid_w=1, frames_per_block=1, ref_frames=1,
               ring_slots=3, rope_mode=1, rope_split=(16, 0, 0), rope_base=10000.0,
               block_index=4, valid_mask=0b0000100)           # only the dynamic slot: 1 key
    q, k, v = _inputs(cfg, seed=7)
    out, _ = oracle.attention(cfg, q, k, v)
    a, _ = oracle.slot_ranges(cfg)[oracle.SLOT_DYNAMIC]
    for h in range(3):
        assert np.array_equal(out[:, h, :], np.broadcast_to(v[h, a], out[:, h, :].shape))


def test_no_valid_key_gives_zero_output():
    cfg = synth.preset("tiny", block_index=3, valid_mask=0)
    q, k, v = _inputs(cfg, seed=8)
    out, lse = oracle.attention(cfg, q, k, v)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_same_logical_layout_same_output_after_ring_moves():
    """Advancing the block index by R leaves the slot permutation unchanged; advancing it by one
    moves every ring block to another rank.  Rebuild the cache so that each logical block is
    the same, at b and at b+1: the outputs must agree."""
    cfg0 = synth.preset("tiny", block_index=6, valid_mask=0b111111)
    q, k, v = _inputs(cfg0, seed=9)
    cfg1 = dict(cfg0, block_index=7)
    lf, lblk, lref = _sizes(cfg0)
    R = cfg0["ring_slots"]
    k1, v1 = k.copy(), v.copy()
    for rank in range(R):   # logical block at rank r lives in slot (b-R+1+r) mod R
        s0 = (6 - R + 1 + rank) % R
        s1 = (7 - R + 1 + rank) % R
        a0, a1 = lref + (2 + s0) * lblk, lref + (2 + s1) * lblk
        k1[:, a1:a1 + lblk] = k[:, a0:a0 + lblk]
        v1[:, a1:a1 + lblk] = v[:, a0:a0 + lblk]
    o0, _ = oracle.attention(cfg0, q, k, v)
    o1, _ = oracle.attention(cfg1, q, k1, v1)
    assert np.max(np.abs(o0 - o1)) <= 1e-13
    # and moving the blocks without re-laying them out does change the result
    o2, _ = oracle.attention(cfg1, q, k, v)
    assert np.max(np.abs(o0 - o2)) > 1e-3


def test_rows_and_heads_subsets_match_full():
    cfg = dict(SMALL_3D, block_index=5, valid_mask=0b111111)
    q, k, v = _inputs(cfg, seed=10)
    full, lse = oracle.attention(cfg, q, k, v)
    rows = np.array([0, 3, 11])
    sub, lse_s = oracle.attention(cfg, q, k, v, rows=rows, heads=[1])
    assert np.max(np.abs(sub[:, 0] - full[rows, 1])) <= 1e-14
    assert np.max(np.abs(lse_s[0] - lse[1, rows])) <= 1e-14


def test_position_probe_catches_one_misplaced_key(monkeypatch):
    """The adversarial probe of the GPU position tests is sensitive: moving ONE key of the
    cache one grid column (3-D) or one token (1-D) changes the output far beyond the
    attention tolerance."""
    import oracle.prsink_oracle as po
    from tests._probe import probe_inputs
    for name, S, H in [("tiny", 300.0, 1), ("480x480", 1000.0, 1)]:
        cfg = synth.preset(name, block_index=1000, valid_mask=0xFF, n_heads=H)
        q, k, v = (t.double().numpy() for t in probe_inputs(cfg, S))
        rows = np.arange(0, oracle.layout_sizes(cfg)["L_blk"], 97)
        good, _ = oracle.attention(cfg, q, k, v, rows=rows)
        orig = po.key_positions

        def shifted(c):
            pos, valid = orig(c)
            pos = pos.copy()
            if c["rope_mode"] == 3:
                pos[127, 2] += 1
            else:
                pos[127] += 1
            return pos, valid

        monkeypatch.setattr(po, "key_positions", shifted)
        bad, _ = oracle.attention(cfg, q, k, v, rows=rows)
        monkeypatch.setattr(po, "key_positions", orig)
        assert np.abs(bad - good).max() > 0.25, name


def _longdouble_attention(cfg, q, k, v):
    """The tiny 1-D layout in numpy long double (80-bit on x86-64): gather the logical sequence,
    rotate every pair by its position's angle, textbook softmax.  Independent of the oracle's
    code; it bounds the oracle's float64 rounding."""
    ld = np.longdouble
    lf, lblk, _ = _sizes(cfg)
    d = cfg["head_dim"]
    rows = _logical_rows(cfg)
    n_log = len(rows)
    j = np.arange(d // 2, dtype=ld)
    inv = np.power(ld(cfg["rope_base"]), -2 * j / ld(d))

    def rot(x, pos):
        ang = np.asarray(pos, dtype=ld)[:, None] * inv[None, :]
        c, s = np.cos(ang), np.sin(ang)
        x0, x1 = x[:, 0::2], x[:, 1::2]
        out = np.empty_like(x)
        out[:, 0::2] = x0 * c - x1 * s
        out[:, 1::2] = x0 * s + x1 * c
        return out

    valid = [(r, i) for i, (r, ok) in enumerate(rows) if ok]
    phys = [r for r, _ in valid]
    logi = [i for _, i in valid]
    out = np.zeros((lblk, cfg["n_heads"], d), dtype=ld)
    for h in range(cfg["n_heads"]):
        kk = rot(k[h][phys].astype(ld), logi)
        vv = v[h][phys].astype(ld)
        qq = rot(q[:, h].astype(ld), [n_log - lblk + i for i in range(lblk)])
        sc = (qq @ kk.T) / np.sqrt(ld(d))
        sc -= sc.max(axis=1, keepdims=True)
        w = np.exp(sc)
        out[:, h] = (w @ vv) / w.sum(axis=1, keepdims=True)
    return out


@pytest.mark.skipif(np.finfo(np.longdouble).eps >= np.finfo(np.float64).eps,
                    reason="long double is not wider than double on this platform")
@pytest.mark.parametrize("b,mask", [(7, 0b111111), (2, 0b011011)])
def test_float64_oracle_within_rounding_of_long_double(b, mask):
    cfg = synth.preset("tiny", block_index=b, valid_mask=mask)
    q, k, v = _inputs(cfg, 21 + b)
    got, _ = oracle.attention(cfg, q, k, v)
    ref = _longdouble_attention(cfg, q, k, v)
    assert np.abs(got - ref.astype(np.float64)).max() < 1e-12
