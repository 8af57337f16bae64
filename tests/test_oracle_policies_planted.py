"""Plant plausible mistakes in the oracle's bank-policy variants (on the CPU) and check that the
pins of ``tests/test_oracle_policies.py`` catch each one: the fallback comparison inverted, the
gate compared on similarity instead of distance, a refreshed entry stamped with the wrong
source block, the moving-average weights swapped, the nearest entry taken as the farthest, the
blended fingerprint left unnormalised."""
import math

import numpy as np
import pytest

import oracle
import oracle.prsink_oracle as po
import tests.test_oracle_policies as tpp

_orig_bank_update = po.bank_update
_orig_retrieve = po.retrieve


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(po, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def _fallback_inverted(phi_b, ok, min_detected, bank_phi, bank_src, count, exclude):
    if po.detected_frames(ok) >= min_detected and min_detected > 0:
        return -1, -np.inf
    return _orig_retrieve(phi_b, bank_phi, bank_src, count, exclude)


def _gated_on_similarity(bank_phi, bank_src, count, M, phi_b, b, write_blocks, gate):
    if b < write_blocks:
        return _orig_bank_update(bank_phi, bank_src, count, M, phi_b, b, write_blocks)
    sims = [float(np.dot(np.asarray(bank_phi[i], dtype=np.float64), phi_b)) for i in range(count)]
    if count > 0 and not max(sims) > gate:
        return -1, np.array(bank_phi, dtype=np.float64), np.array(bank_src), count
    return _orig_bank_update(bank_phi, bank_src, count, M, phi_b, b, b + 1)


def _gated_wrong_source(bank_phi, bank_src, count, M, phi_b, b, write_blocks, gate):
    if b < write_blocks:
        return _orig_bank_update(bank_phi, bank_src, count, M, phi_b, b, write_blocks)
    d = po.fingerprint_distances(phi_b, bank_phi, count)
    if count > 0 and not float(d.min()) > gate:
        return -1, np.array(bank_phi, dtype=np.float64), np.array(bank_src), count
    return _orig_bank_update(bank_phi, bank_src, count, M, phi_b, 0, 1)     # stamps block 0


def _decay_variant(swap=False, farthest=False, normalise=True):
    def fn(bank_phi, bank_src, count, M, phi_b, b, write_blocks, alpha):
        if b < write_blocks:
            a, bp, bs, c = _orig_bank_update(bank_phi, bank_src, count, M, phi_b, b, write_blocks)
            return a, ("store" if a >= 0 else None), bp, bs, c
        bank_phi = np.array(bank_phi, dtype=np.float64, copy=True)
        bank_src = np.array(bank_src, copy=True)
        if not alpha > 0.0 or count == 0:
            return -1, None, bank_phi, bank_src, count
        sims = [float(np.dot(bank_phi[i], phi_b)) for i in range(count)]
        j = int(np.argmin(sims)) if farthest else int(np.argmax(sims))
        w_old, w_new = po.blend_weights(alpha)
        if swap:
            w_old, w_new = w_new, w_old
        t = float(w_old) * bank_phi[j] + float(w_new) * np.asarray(phi_b, dtype=np.float64)
        n = math.sqrt(float(np.dot(t, t)))
        bank_phi[j] = t / n if (normalise and n > 0) else t
        bank_src[j] = b
        return j, "blend", bank_phi, bank_src, count
    return fn


MUTATIONS = {
    "fallback_inverted": [("retrieve_fallback", _fallback_inverted)],
    "gate_on_similarity": [("bank_update_gated", _gated_on_similarity)],
    "gate_wrong_source_block": [("bank_update_gated", _gated_wrong_source)],
    "decay_weights_swapped": [("bank_update_decay", _decay_variant(swap=True))],
    "decay_farthest_entry": [("bank_update_decay", _decay_variant(farthest=True))],
    "decay_unnormalised": [("bank_update_decay", _decay_variant(normalise=False))],
}


def _pins():
    return [
        tpp.test_fallback_off_is_plain_retrieval,
        lambda: [tpp.test_fallback_by_enumerating_detection_patterns(m) for m in range(4)],
        tpp.test_fallback_stream_empties_the_dynamic_sink_on_failed_blocks,
        tpp.test_distance_matches_the_unit_vector_closed_form,
        tpp.test_gate_closed_is_the_frozen_bank_and_gate_open_never_freezes,
        tpp.test_gate_lets_a_far_block_into_a_frozen_bank,
        tpp.test_decay_off_is_the_frozen_bank,
        tpp.test_nearest_entry_is_the_sorted_maximum,
        tpp.test_full_weight_blend_is_a_store,
        tpp.test_blended_fingerprint_is_unit_and_between_its_sources,
    ]


def test_unmutated_policies_pass_every_pin():
    for pin in _pins():
        pin()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_policy_mistake_is_caught(name, monkeypatch):
    for attr, fn in MUTATIONS[name]:
        _patch(monkeypatch, attr, fn)
    caught = 0
    for pin in _pins():
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {name}"
