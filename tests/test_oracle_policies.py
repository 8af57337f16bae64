"""Pins of the oracle's bank-policy variants (the digest's weaknesses 3 and 5): each reduces to
the pages' own rule at its neutral setting, and each is checked against an independent
formulation (closed forms, enumeration, exact rational arithmetic)."""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth


def _unit_rows(g, n, dim=558):
    x = g.standard_normal((n, dim))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def _stream(seed=5, n=40):
    kp, ok, _ = synth.pose_stream(seed, n, fail_frac=0.2)
    phis = [oracle.fingerprint(kp[b][:, :62], ok[b]) for b in range(n)]
    return phis, [list(o) for o in ok]


def _key(d):
    return (d["r"], d["copy"], d["dyn_src"], d["action"], d["count"], tuple(d["bank_src"]))


# ------------------------------------------------------------------ fallback (weakness 5)

def test_fallback_off_is_plain_retrieval():
    g = np.random.default_rng(0)
    for _ in range(20):
        bank = _unit_rows(g, 5)
        phi = _unit_rows(g, 1)[0]
        src = g.permutation(50)[:5]
        ok = list(g.integers(0, 2, 3))
        assert oracle.retrieve_fallback(phi, ok, 0, bank, src, 5, int(src[0])) == \
            oracle.retrieve(phi, bank, src, 5, int(src[0]))


@pytest.mark.parametrize("min_detected", range(4))
def test_fallback_by_enumerating_detection_patterns(min_detected):
    g = np.random.default_rng(min_detected)
    bank = _unit_rows(g, 5)
    phi = _unit_rows(g, 1)[0]
    src = np.arange(5)
    for ok in itertools.product([0, 1], repeat=3):
        r, sc = oracle.retrieve_fallback(phi, ok, min_detected, bank, src, 5, -1)
        if sum(ok) < min_detected:
            assert (r, sc) == (-1, -np.inf)
        else:
            assert r == int(np.argmax(bank @ phi))


def test_fallback_stream_empties_the_dynamic_sink_on_failed_blocks():
    phis, oks = _stream()
    dec = oracle.stream_decisions_policy(phis, oks, min_detected=3)
    failed = [b for b, ok in enumerate(oks) if sum(ok) < 3]
    assert failed
    for b in failed:
        assert dec[b]["r"] == -1 and not dec[b]["copy"] and dec[b]["dyn_src"] == -1
    base = oracle.stream_decisions_policy(phis, oks, min_detected=0)
    assert [_key(d) for d in base] == [_key(d) for d in oracle.stream_decisions(phis)]


# ------------------------------------------------------------------ gated refresh (weakness 3)

def test_distance_matches_the_unit_vector_closed_form():
    g = np.random.default_rng(1)
    bank = _unit_rows(g, 5)
    phi = _unit_rows(g, 1)[0]
    d = oracle.fingerprint_distances(phi, bank, 5)
    assert np.allclose(d, np.sqrt(np.maximum(2.0 - 2.0 * bank @ phi, 0.0)), atol=1e-12)
    assert oracle.fingerprint_distances(np.zeros(558), bank, 5) == pytest.approx(np.ones(5))


def test_gate_closed_is_the_frozen_bank_and_gate_open_never_freezes():
    phis, oks = _stream()
    frozen = oracle.stream_decisions_policy(phis, oks, policy="frozen")
    closed = oracle.stream_decisions_policy(phis, oks, policy="gated", gate=2.5)   # > max distance
    assert [_key(d) for d in closed] == [_key(d) for d in frozen]
    opened = oracle.stream_decisions_policy(phis, oks, policy="gated", gate=-1.0)
    never = oracle.stream_decisions(phis, write_blocks=len(phis))
    assert [_key(d) for d in opened] == [_key(d) for d in never]


def test_gate_lets_a_far_block_into_a_frozen_bank():
    g = np.random.default_rng(2)
    base = _unit_rows(g, 1)[0]
    bank = np.array([base + 0.05 * r for r in g.standard_normal((5, 558))])
    bank /= np.linalg.norm(bank, axis=1, keepdims=True)
    src = np.arange(5)
    far = _unit_rows(g, 1)[0]                                  # ~orthogonal: distance ~ sqrt(2)
    near = bank[2] + 0.01 * g.standard_normal(558)
    near /= np.linalg.norm(near)
    a, phi2, src2, c = oracle.bank_update_gated(bank, src, 5, 5, far, 30, 20, gate=1.0)
    assert a >= 0 and src2[a] == 30 and np.allclose(phi2[a], far)
    a, phi2, src2, c = oracle.bank_update_gated(bank, src, 5, 5, near, 30, 20, gate=1.0)
    assert a == -1 and np.array_equal(phi2, bank) and np.array_equal(src2, src)


# ------------------------------------------------------------------ decayed writes (weakness 3)

def test_decay_off_is_the_frozen_bank():
    phis, oks = _stream()
    frozen = oracle.stream_decisions_policy(phis, oks, policy="frozen")
    off = oracle.stream_decisions_policy(phis, oks, policy="decay", alpha=0.0)
    assert [_key(d) for d in off] == [_key(d) for d in frozen]


def test_nearest_entry_is_the_sorted_maximum():
    g = np.random.default_rng(3)
    for _ in range(20):
        bank = _unit_rows(g, 7)
        phi = _unit_rows(g, 1)[0]
        j, sc = oracle.nearest_entry(phi, bank, 7)
        assert j == sorted(range(7), key=lambda i: (-float(bank[i] @ phi), i))[0]
    assert oracle.nearest_entry(phi, bank, 0) == (-1, -np.inf)


def test_full_weight_blend_is_a_store():
    cfg = synth.preset("tiny", block_index=4, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    cache = synth.normal_bf16((2, 2, 1, s["T"], 64), 3, 0).double().numpy()
    bank = synth.normal_bf16((2, 5, 2, 1, s["L_blk"], 64), 3, 1).double().numpy()
    assert np.array_equal(oracle.bank_blend_kv(cfg, cache, bank, 1, 3, 1.0),
                          oracle.bank_store(cfg, cache, bank, 1, 3))
    assert np.array_equal(oracle.bank_blend_kv(cfg, cache, bank, 1, 3, 0.0), bank)
    g = np.random.default_rng(4)
    bp = _unit_rows(g, 5)
    phi = _unit_rows(g, 1)[0]
    a, mode, bp2, src2, _ = oracle.bank_update_decay(bp, np.arange(5), 5, 5, phi, 25, 20, 1.0)
    assert mode == "blend" and np.allclose(bp2[a], phi, atol=1e-15) and src2[a] == 25


def test_blend_is_the_rounded_exact_average():
    """Against exact rational arithmetic: the float32 products and sum are within float32
    rounding of (1 - alpha) x + alpha z, and the bf16 result within half a bf16 ulp of that."""
    cfg = synth.preset("tiny", block_index=4, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    cache = synth.normal_bf16((1, 2, 1, s["T"], 64), 6, 0).double().numpy()
    bank = synth.normal_bf16((1, 5, 2, 1, s["L_blk"], 64), 6, 1).double().numpy()
    alpha = 0.3
    out = oracle.bank_blend_kv(cfg, cache, bank, 0, 2, alpha)
    a, _ = oracle.slot_ranges(cfg)[oracle.SLOT_RING0]
    w_old, w_new = oracle.blend_weights(alpha)
    g = np.random.default_rng(5)
    for _ in range(300):
        kv, t, c = int(g.integers(2)), int(g.integers(s["L_blk"])), int(g.integers(64))
        x, z = bank[0, 2, kv, 0, t, c], cache[0, kv, 0, a + t, c]
        exact = Fraction(float(w_old)) * Fraction(x) + Fraction(float(w_new)) * Fraction(z)
        got = out[0, 2, kv, 0, t, c]
        assert abs(Fraction(got) - exact) <= Fraction(2.0 ** -8) * abs(exact) + Fraction(2.0 ** -130)
        assert got == float(torch.tensor(got).to(torch.bfloat16).item())    # a bf16 value


def test_repeated_blends_decay_geometrically():
    cfg = synth.preset("tiny", block_index=4, valid_mask=0xFF)
    s = oracle.layout_sizes(cfg)
    bank = synth.normal_bf16((1, 1, 2, 1, s["L_blk"], 64), 7, 1).double().numpy()
    cache = np.zeros((1, 2, 1, s["T"], 64))
    a, e = oracle.slot_ranges(cfg)[oracle.SLOT_RING0]
    cache[:, :, :, a:e] = 1.0
    x0 = bank.copy()
    alpha, k = 0.25, 4
    for _ in range(k):
        bank = oracle.bank_blend_kv(cfg, cache, bank, 0, 0, alpha)
    want = (1 - alpha) ** k * x0 + (1 - (1 - alpha) ** k) * 1.0
    assert np.abs(bank - want).max() <= k * 2.0 ** -8 * (np.abs(x0).max() + 1.0)


def test_blended_fingerprint_is_unit_and_between_its_sources():
    g = np.random.default_rng(8)
    bp = _unit_rows(g, 5)
    phi = 0.8 * bp[1] + 0.6 * _unit_rows(g, 1)[0]
    phi /= np.linalg.norm(phi)
    a, mode, bp2, _, _ = oracle.bank_update_decay(bp, np.arange(5), 5, 5, phi, 21, 20, 0.25)
    assert a == 1 and mode == "blend"
    assert abs(np.linalg.norm(bp2[1]) - 1.0) <= 1e-12
    assert bp2[1] @ phi > bp[1] @ phi and bp2[1] @ bp[1] > bp[1] @ phi
    for j in (0, 2, 3, 4):
        assert np.array_equal(bp2[j], bp[j])
