"""The prefill attention kernel's barrier protocol under random schedules (CPU; see attention_protocol).

The kernel as built (one query tile per CTA, P buffers by pair % 2) must finish every schedule with no
buffer hazard, for one and for two value slots and for every chunk-union size up to 17.  The earlier
design, with the P buffers tied to the value slots, must be caught racing with a single value slot:
a softmax warp that skipped pairs passes its P-buffer wait one phase early.  The persistent variant
(several tiles per CTA, bookkeeping double-buffered, O released by O_EMPTY) is checked as well.
"""
import random

import pytest

from attention_protocol import Protocol


def _failures(make, runs):
    bad = []
    for seed in range(runs):
        try:
            make(seed).run()
        except AssertionError as e:
            bad.append(str(e))
    return bad


@pytest.mark.parametrize("n_value_slots", [1, 2])
def test_one_tile_per_cta_is_race_and_deadlock_free(n_value_slots):
    bad = _failures(lambda seed: Protocol([1 + seed % 17], n_value_slots, seed=seed, lone_by_count=False), 170)
    assert not bad, bad[:3]


def test_p_buffers_tied_to_one_value_slot_race():
    bad = _failures(lambda seed: Protocol([3 + seed % 14], 1, seed=seed, p_mod_2=False, lone_by_count=False), 100)
    assert any("P buffer overwritten" in b for b in bad), bad[:3]


def test_p_buffers_tied_to_two_value_slots_were_safe():
    bad = _failures(lambda seed: Protocol([1 + seed % 17], 2, seed=seed, p_mod_2=False, lone_by_count=False), 170)
    assert not bad, bad[:3]


@pytest.mark.parametrize("n_value_slots", [1, 2])
def test_persistent_cta_is_race_and_deadlock_free(n_value_slots):
    r = random.Random(5 + n_value_slots)
    cases = [[r.randint(1, 11) for _ in range(r.randint(2, 6))] for _ in range(120)]
    bad = _failures(lambda seed: Protocol(cases[seed], n_value_slots, seed=1000 + seed), len(cases))
    assert not bad, bad[:3]


def test_persistent_cta_needs_the_lone_chunk_counted_twice():
    # with the value loader standing in for a lone chunk's missing warps, the next tile's S buffer
    # never becomes free: the protocol stalls
    cases = [[3, 4], [5, 2, 2], [1, 1]]
    bad = _failures(lambda seed: Protocol(cases[seed % 3], 2, seed=seed, lone_by_count=False), 30)
    assert any("deadlock" in b or "more arrivals" in b for b in bad), bad[:3]
