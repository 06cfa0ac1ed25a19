"""The attention kernel's mbarrier protocol, checked on a host-side model (no GPU).

tests/attn_protocol_model.py runs attn_kernel's warp roles with the kernel's
barrier counts and phase parities and random timing of copies and MMA commits.
"""
import random

import attn_protocol_model as M


def test_valid_items_never_deadlock_or_race():
    """Every item of a valid layer has at least one key block (k >= 1)."""
    rng = random.Random(11)
    for _ in range(150):
        items = M.random_items(rng, allow_empty=False)
        assert M.run(items, rng) == "ok", items


def test_items_without_key_blocks_can_alias_the_list_slot():
    """Known issue in the current kernel: with an item that has no key blocks (only a rejected
    item on a layer without prefix tiles), the list slot can be refilled twice before the S
    issuer has seen it; its parity wait then never passes (the kernel's bounded wait times out).
    Starving the S issuer and the V producer shows it deterministically."""
    rng = random.Random(3)
    r = M.run([0, 1, 0, 1], rng, starve=("S issuer", "producer V", "tmaV"))
    assert r.startswith("deadlock"), r
    assert "S issuer waits LFULL0" in r


def test_every_slot_reader_releasing_the_slot_fixes_it():
    rng = random.Random(5)
    assert M.run([0, 1, 0, 1], rng, slot_readers_release=True,
                 starve=("S issuer", "producer V", "tmaV")) == "ok"
    for _ in range(150):
        items = M.random_items(rng, allow_empty=True)
        assert M.run(items, rng, slot_readers_release=True) == "ok", items


def _flagged(fault, trials, seed):
    rng = random.Random(seed)
    n = 0
    for _ in range(trials):
        try:
            n += M.run(M.random_items(rng, allow_empty=False), rng, faults=(fault,)) != "ok"
        except M.Hazard:
            n += 1
    return n


def test_model_catches_an_s_buffer_reused_before_pv():
    assert _flagged("s_skips_pv_done", 60, 2) > 0


def test_model_catches_a_wrong_phase_parity():
    assert _flagged("softmax_parity", 20, 4) == 20
