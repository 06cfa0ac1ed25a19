"""The attention kernel's mbarrier protocol, checked on a host-side model (no GPU).

tests/attn_protocol_model.py runs attn_kernel's warp roles with the kernel's
barrier counts and phase parities and random timing of copies and MMA commits,
including the bounded waits and the abort / drain path taken when one runs out.
"""
import random

import pytest

import attn_protocol_model as M


def test_valid_items_never_deadlock_or_race():
    """Every item of a valid layer has at least one key block (k >= 1)."""
    rng = random.Random(11)
    for _ in range(150):
        items = M.random_items(rng, allow_empty=False)
        assert M.run(items, rng) == "ok", items


def test_items_without_key_blocks_are_safe_with_the_kernels_slot_counts():
    """An item with no key blocks (a rejected item on a layer without prefix tiles): every role
    that reads the list slot releases it (13 arrivals), so the slot is never refilled before the
    S issuer or the V producer has seen it."""
    rng = random.Random(5)
    assert M.run([0, 1, 0, 1], rng, starve=("S issuer", "producer V", "tmaV")) == "ok"
    for _ in range(150):
        items = M.random_items(rng, allow_empty=True)
        assert M.run(items, rng) == "ok", items


def test_the_earlier_slot_counts_alias_and_time_out():
    """With the list-slot barrier counting only the eight softmax warps (the earlier kernel),
    the slot can be refilled twice before the S issuer has seen it; its parity wait then never
    passes, the bounded wait runs out and the CTA aborts (reported as a timeout, not a hang)."""
    rng = random.Random(3)
    r = M.run([0, 1, 0, 1], rng, slot_readers_release=False, starve=("S issuer", "producer V", "tmaV"))
    assert r.startswith("aborted") and "S issuer waits LFULL0" in r, r


@pytest.mark.parametrize("seed", range(6))
def test_hold_runs_out_and_drains_before_the_cta_ends(seed):
    """The kernel's test hold: the softmax warps wait on a barrier nothing arrives on. Every
    other role blocks in turn, the bounded wait runs out, and after the abort the producers'
    copies and the issuers' MMAs have all completed before the CTA ends."""
    rng = random.Random(100 + seed)
    for _ in range(25):
        items = M.random_items(rng, allow_empty=False)
        r = M.run(items, rng, hold=True)
        assert r.startswith("aborted") and "HOLD" in r, (items, r)


def _flagged(fault, trials, seed, timeout_p=0.0):
    rng = random.Random(seed)
    n = 0
    for _ in range(trials):
        try:
            r = M.run(M.random_items(rng, allow_empty=False), rng, faults=(fault,), timeout_p=timeout_p)
            n += not (r == "ok" or (timeout_p and r.startswith("aborted")))
        except M.Hazard:
            n += 1
    return n


@pytest.mark.parametrize("seed", range(4))
def test_a_wait_running_out_early_still_drains(seed):
    """A wait that runs out while copies and MMAs are in flight (a caller's short limit): the
    roles leave, the producers wait for their copies and the issuers for their MMAs, and
    nothing is in flight when the CTA ends."""
    rng = random.Random(200 + seed)
    aborted = 0
    for _ in range(40):
        r = M.run(M.random_items(rng, allow_empty=True), rng, timeout_p=0.02)
        assert r == "ok" or r.startswith("aborted"), r
        aborted += r.startswith("aborted")
    assert aborted > 0


def test_model_catches_an_s_buffer_reused_before_pv():
    assert _flagged("s_skips_pv_done", 60, 2) > 0


def test_model_catches_a_wrong_phase_parity():
    assert _flagged("softmax_parity", 20, 4) == 20


def test_model_catches_mma_issuers_leaving_without_draining():
    assert _flagged("mma_no_drain", 60, 6, timeout_p=0.02) > 0


def test_model_catches_producers_leaving_without_draining():
    assert _flagged("tma_no_drain", 60, 7, timeout_p=0.02) > 0
