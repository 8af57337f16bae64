"""Plant plausible mistakes in the oracle (on the CPU) and check that its pins catch each one.

Every mutation below is a slip that could be made while writing the oracle from the pages: a
reversed rotation, the other RoPE pairing convention, a dropped factor in the frequencies, an
off-by-one in the ring order, a wrong attention scale, queries placed on the wrong slot, a
missing normalisation, the b-1 exclusion forgotten, maximising instead of minimising the bank
similarity, and a block written into the neighbouring slot.  For each one at least one pin
must fail.
"""
import numpy as np
import pytest

import oracle
import oracle.prsink_oracle as po
import tests.test_oracle_attention as ta
import tests.test_oracle_layout_rope as tl
import tests.test_oracle_pose as tp


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(po, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def _rope_reversed(cfg, x, pos):
    x = np.asarray(x, dtype=np.float64)
    ang = po.rope_angles(cfg, pos)
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * c + x[..., 1::2] * s
    out[..., 1::2] = -x[..., 0::2] * s + x[..., 1::2] * c
    return out


def _rope_half_split(cfg, x, pos):
    x = np.asarray(x, dtype=np.float64)
    ang = po.rope_angles(cfg, pos)
    c, s = np.cos(ang), np.sin(ang)
    h = x.shape[-1] // 2
    out = np.empty_like(x)
    out[..., :h] = x[..., :h] * c - x[..., h:] * s
    out[..., h:] = x[..., :h] * s + x[..., h:] * c
    return out


def _angles_no_two(cfg, pos):
    base = float(cfg["rope_base"])
    pos = np.asarray(pos)
    parts = []
    for ax, (_, da) in enumerate(po._rope_axes(cfg)):
        j = np.arange(da // 2, dtype=np.float64)
        p = pos[..., ax] if cfg["rope_mode"] == 3 else pos
        parts.append(p.astype(np.float64)[..., None] * base ** (-j / da))
    return np.concatenate(parts, axis=-1)


_orig_attention = po.attention
_orig_query_positions = po.query_positions
_orig_fingerprint = po.fingerprint
_orig_kv_append = po.kv_append


def _attention_scale_d(cfg, q, k, v, rows=None, heads=None):
    # scores divided by d instead of sqrt(d): same as scaling q by 1/sqrt(d)
    return _orig_attention(cfg, np.asarray(q) / np.sqrt(cfg["head_dim"]), k, v, rows, heads)


def _query_positions_oldest(cfg):
    s = po.layout_sizes(cfg)
    return _orig_query_positions(cfg) - (s["R"] - 1) * cfg["frames_per_block"] * (
        1 if cfg["rope_mode"] == 3 else s["L_f"]) * (
        np.array([1, 0, 0]) if cfg["rope_mode"] == 3 else 1)


def _fingerprint_unnormalised(kp, ok):
    v = _orig_fingerprint(kp, ok)
    kpa = np.asarray(kp, dtype=np.float64).reshape(-1)
    return v * np.linalg.norm(kpa)


def _fingerprint_no_zero_fill(kp, ok):
    return _orig_fingerprint(kp, np.ones(3, np.uint8))


def _retrieve_no_exclusion(phi_b, bank_phi, bank_src, count, exclude):
    best, best_s = -1, -np.inf
    for i in range(int(count)):
        sc = float(np.dot(bank_phi[i], phi_b))
        if best < 0 or sc > best_s:
            best, best_s = i, sc
    return best, best_s


def _bank_objective_negated(phis):
    import itertools
    phis = [np.asarray(p, dtype=np.float64) for p in phis]
    pairs = list(itertools.combinations(range(len(phis)), 2))
    return -sum(float(np.dot(phis[i], phis[j])) for i, j in pairs) / max(len(pairs), 1)


def _kv_append_next_slot(cfg, k_new, v_new, k_cache, v_cache, slot):
    n = len(po.slot_ranges(cfg))
    return _orig_kv_append(cfg, k_new, v_new, k_cache, v_cache, (slot + 1) % n
                           if po.slot_ranges(cfg)[(slot + 1) % n][1] - po.slot_ranges(cfg)[
                               (slot + 1) % n][0] == np.asarray(k_new).shape[0] else slot - 1)


MUTATIONS = {
    "rope_reversed": [("rope_rotate", _rope_reversed)],
    "rope_half_split": [("rope_rotate", _rope_half_split)],
    "rope_freq_missing_2": [("rope_angles", _angles_no_two)],
    "ring_rank_off_by_one": [("ring_rank", lambda s, b, R: (s - (b - R + 1) + 1) % R)],
    "scale_1_over_d": [("attention", _attention_scale_d)],
    "queries_on_oldest_slot": [("query_positions", _query_positions_oldest)],
    "fingerprint_unnormalised": [("fingerprint", _fingerprint_unnormalised)],
    "fingerprint_no_zero_fill": [("fingerprint", _fingerprint_no_zero_fill)],
    "retrieve_no_exclusion": [("retrieve", _retrieve_no_exclusion)],
    "bank_maximises_similarity": [("bank_objective", _bank_objective_negated)],
    "append_wrong_slot": [("kv_append", _kv_append_next_slot)],
}


def _pins():
    """Every pin, as a zero-argument callable (one representative case per parametrisation)."""
    return [
        tl.test_rope_closed_forms,
        tl.test_rope_position_zero_is_identity_and_norm_kept,
        lambda: tl.test_rope_relative_invariance("480x480"),
        lambda: tl.test_ring_rank_is_age_order(3),
        lambda: tl.test_positions_tile_the_logical_layout("tiny", 7),
        lambda: tl.test_positions_tile_the_logical_layout("480x480", 1000),
        tl.test_valid_mask_early_blocks,
        lambda: ta.test_tiny_1d_matches_bruteforce(7, 0b111111),
        lambda: ta.test_small_3d_matches_bruteforce(4, 0b111111, 3),
        ta.test_zero_queries_average_the_valid_values,
        ta.test_same_logical_layout_same_output_after_ring_moves,
        tp.test_fingerprint_layout_closed_form,
        tp.test_fingerprint_failed_frames_are_zero_filled,
        tp.test_retrieve_ties_exclusion_and_empty,
        lambda: [tp.test_retrieve_matches_sort(s) for s in range(20)],
        lambda: [tp.test_bank_update_matches_subset_enumeration(s) for s in range(25)],
        tp.test_bank_update_insert_ties_and_freeze,
        tp.test_kv_append_places_rows_bit_exact,
        tp.test_stream_decisions_invariants,
    ]


def test_unmutated_oracle_passes_every_pin():
    for pin in _pins():
        pin()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    for attr, fn in MUTATIONS[name]:
        _patch(monkeypatch, attr, fn)
    caught = 0
    for pin in _pins():
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {name}"
