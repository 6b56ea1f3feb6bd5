"""Host slot allocator / prefix cache (gdn_slot_cache_*), no GPU.

Scenarios check the semantics one by one.  A random-operation test checks two things after
every call: that reference counts are conserved, and that every planned index table meets
gdn_decode_step's preconditions, as judged by the oracle's brute-force check.
"""
import numpy as np
import pytest

import oracle
from hybrid_linear_attention_step_b200.slot_cache import SlotCache, SlotCacheError

CAPACITY = 6
INVALID = 1


def test_miss_then_in_place_updates():
    c = SlotCache(8)
    req, slot, matched, needs_init = c.open([5, 6, 7])
    assert matched == 0 and needs_init and c.refcount(slot) == 1
    for _ in range(3):
        src, dst = c.plan([req])
        assert src[0] == slot and dst[0, 0] == slot  # owned: in place
        assert c.commit([req])[0] == slot
    assert c.stats() == (7, 0, 1)
    c.close(req)
    assert c.stats() == (8, 0, 0)


def test_checkpoint_forks_copy_on_write():
    c = SlotCache(8)
    toks = [1, 2, 3, 4]
    req, s0, _, _ = c.open(toks)
    assert c.checkpoint(req, toks) == s0 and c.refcount(s0) == 2
    src, dst = c.plan([req])
    assert src[0] == s0 and dst[0, 0] != s0  # the checkpoint is read, a fresh slot written
    new = c.commit([req])[0]
    assert new == dst[0, 0] and c.refcount(s0) == 1 and c.refcount(new) == 1
    src, dst = c.plan([req])  # now owned again: in place
    assert src[0] == dst[0, 0] == new
    c.commit([req])
    # a second request extending the prefix starts from the checkpoint
    r2, s2, matched, needs_init = c.open(toks + [9, 9])
    assert (s2, matched, needs_init) == (s0, 4, False) and c.refcount(s0) == 2
    src, dst = c.plan([r2])
    assert src[0] == s0 and dst[0, 0] not in (s0, new)


def test_radix_matching_with_edge_splits():
    c = SlotCache(16)
    slots = {}
    for path in ([1, 2, 3, 4], [1, 2, 5], [1, 2], [7]):
        r, s, _, _ = c.open(path)
        slots[tuple(path)] = c.checkpoint(r, path)
        c.close(r)
    expect = {(1, 2, 3, 4, 9): (1, 2, 3, 4), (1, 2, 5, 6): (1, 2, 5), (1, 2, 7): (1, 2), (1, 2): (1, 2),
              (1, 2, 3): (1, 2), (7, 1): (7,)}
    for ctx, hit in expect.items():
        r, s, matched, needs_init = c.open(list(ctx))
        assert (s, matched, needs_init) == (slots[hit], len(hit), False), ctx
        c.close(r)
    for ctx in ([1, 3], [2], [1], []):
        r, s, matched, needs_init = c.open(ctx)
        assert matched == 0 and needs_init and s not in slots.values()
        c.close(r)
    assert c.stats()[1] == 4


def test_speculative_plan_and_commit():
    c = SlotCache(20)
    reqs = [c.open([i])[0] for i in range(3)]
    base = [c.plan([r])[0][0] for r in reqs]
    c.commit(reqs)
    src, cur = c.plan(reqs, T=4)
    assert list(src) == base and len(set(cur.ravel())) == 12 and not set(cur.ravel()) & set(base)
    assert c.stats()[0] == 20 - 3 - 12
    committed = c.commit(reqs, T=4, accept_len=[0, 2, 4])
    assert list(committed) == [base[0], cur[1, 1], cur[2, 3]]
    assert c.stats()[0] == 20 - 3  # rejected drafts and replaced slots are free again
    for s in (base[1], base[2]) + tuple(cur[0]) + (cur[1, 0], cur[1, 2], cur[1, 3]):
        assert c.refcount(int(s)) == 0
    # matches the device commit's rule on the same table
    want = np.array(base, np.int32)
    oracle.commit(np.array([0, 2, 4], np.int32), want, cur, 20)
    assert np.array_equal(committed, want)


def test_eviction_and_capacity():
    c = SlotCache(4)
    reqs = []
    for i in range(4):
        r, s, _, _ = c.open([100 + i])
        c.checkpoint(r, [100 + i])
        reqs.append(r)
    assert c.stats() == (0, 4, 4)
    with pytest.raises(SlotCacheError) as e:  # every checkpoint is still read by its request
        c.open([999])
    assert e.value.status == CAPACITY
    c.close(reqs[1])
    c.close(reqs[3])
    # [100] and [102] are still read by their requests; [101] and [103] only by the tree.
    r, s, _, _ = c.open([999])  # no free slot: evicts the least recently used free checkpoint, [101]
    assert c.stats()[1] == 3
    r103, _, matched, _ = c.open([103])
    assert matched == 1  # still cached
    c.close(r103)
    assert c.open([101])[2] == 0  # gone; this open evicts [103], the last evictable checkpoint
    assert c.stats()[1] == 2
    # a plan that cannot find slots changes nothing
    c2 = SlotCache(3)
    a = c2.open([1])[0]
    b = c2.open([2])[0]
    with pytest.raises(SlotCacheError):
        c2.plan([a, b], T=2)
    assert c2.stats() == (1, 0, 2)
    src, dst = c2.plan([a, b])  # single-token in place still works
    assert np.array_equal(src, dst[:, 0])


def test_failing_plan_keeps_evictable_checkpoints():
    """A plan that needs more fresh slots than free plus evictable ones fails before it
    takes a slot or evicts a checkpoint: the cached prefix is still a hit afterwards."""
    c = SlotCache(4)
    r1, s0, _, _ = c.open([1, 2])
    c.checkpoint(r1, [1, 2])
    c.close(r1)  # slot s0 is now held by the tree only: evictable
    r2 = c.open([3])[0]
    r3 = c.open([4])[0]
    before = c.stats()
    assert before == (1, 1, 2)
    with pytest.raises(SlotCacheError) as e:  # 4 draft slots wanted, 1 free + 1 evictable
        c.plan([r2, r3], T=2)
    assert e.value.status == CAPACITY
    assert c.stats() == before
    assert c.refcount(s0) == 1
    r4, s, matched, needs_init = c.open([1, 2, 9])
    assert (s, matched, needs_init) == (s0, 2, False)
    c.close(r4)
    # one draft each for a single request fits: 1 free + 1 evictable
    src, cur = c.plan([r2], T=2)
    assert len(set(cur.ravel())) == 2 and c.stats()[1] == 0


def test_invalid_sequences_are_rejected():
    c = SlotCache(8)
    r = c.open([1])[0]
    for bad in (lambda: c.plan([r, r]), lambda: c.commit([r]), lambda: c.plan([r + 1]), lambda: c.close(r + 5)):
        with pytest.raises(SlotCacheError) as e:
            bad()
        assert e.value.status == INVALID
    c.plan([r], T=2)
    with pytest.raises(SlotCacheError):
        c.commit([r], T=1)
    with pytest.raises(SlotCacheError):
        c.commit([r], T=2, accept_len=[3])
    with pytest.raises(SlotCacheError):
        c.checkpoint(r, [1])  # mid-step
    c.commit([r], T=2, accept_len=[1])
    with pytest.raises(SlotCacheError):
        SlotCache(0)


def test_random_operations_keep_invariants_and_preconditions():
    rng = np.random.default_rng(7)
    num_slots = 48
    c = SlotCache(num_slots)
    open_reqs = {}  # req -> token list
    vocab = 5
    for step in range(1500):
        op = rng.integers(0, 10)
        try:
            if op <= 2 or not open_reqs:
                base = list(open_reqs.values())[rng.integers(0, len(open_reqs))] if open_reqs and rng.random() < .7 else []
                ctx = base[: rng.integers(0, len(base) + 1)] + list(rng.integers(0, vocab, rng.integers(0, 4)))
                r, s, matched, needs = c.open(ctx)
                open_reqs[r] = ctx
            elif op <= 6:
                reqs = rng.choice(list(open_reqs), size=rng.integers(1, len(open_reqs) + 1), replace=False)
                T = int(rng.choice([1, 1, 2, 3]))
                src, dst = c.plan(reqs, T)
                # the plan meets every precondition of gdn_decode_step
                assert oracle.check_step(src, dst, num_slots) == 0
                acc = rng.integers(0, T + 1, size=len(reqs)).astype(np.int32)
                c.commit(reqs[::-1].copy(), T, acc[::-1].copy())
                for i, r in enumerate(reqs):
                    open_reqs[int(r)] = open_reqs[int(r)] + list(rng.integers(0, vocab, 1 if T == 1 else int(acc[i])))
            elif op == 7:
                r = int(rng.choice(list(open_reqs)))
                if open_reqs[r]:
                    c.checkpoint(r, open_reqs[r])
                    if rng.random() < 0.3:
                        # one state under a second, shorter prefix too: several checkpoints
                        # then name one slot, which the bookkeeping must still count right
                        c.checkpoint(r, open_reqs[r][: rng.integers(1, len(open_reqs[r]) + 1)])
            elif op == 8:
                r = int(rng.choice(list(open_reqs)))
                c.close(r)
                del open_reqs[r]
            else:
                c.evict(int(rng.integers(0, num_slots)))
        except SlotCacheError as e:
            assert e.status == CAPACITY
        free, ckpts, nreq = c.stats()
        refs = [c.refcount(s) for s in range(num_slots)]
        assert free == refs.count(0) and nreq == len(open_reqs)
        assert sum(refs) == nreq + ckpts  # each holder holds one reference
    for r in list(open_reqs):
        c.close(r)
    c.evict(num_slots)
    assert c.stats() == (num_slots, 0, 0)


def test_slot_named_by_several_checkpoints_is_freed_before_reuse():
    """Two checkpoints of one request name the same slot.  With no free slot left, a new
    request must get that slot only after both checkpoints are evicted: evicting one of
    them frees nothing, and handing the slot out then would let the request overwrite a
    cached prefix state."""
    c = SlotCache(1)
    req, s0, _, _ = c.open([1, 2, 3])
    assert c.checkpoint(req, [1, 2]) == s0 and c.checkpoint(req, [1, 2, 3]) == s0
    c.close(req)
    assert c.stats() == (0, 2, 0) and c.refcount(s0) == 2
    r2, s2, matched, needs_init = c.open([9])
    assert (s2, matched, needs_init) == (s0, 0, True)
    assert c.stats() == (0, 0, 1) and c.refcount(s0) == 1   # both checkpoints gone, slot owned once
    c.close(r2)
    _, _, matched, needs_init = c.open([1, 2, 3])              # the prefix is no longer cached
    assert matched == 0 and needs_init


def test_capacity_failure_with_shared_checkpoint_slot_changes_nothing():
    """Slot 0 is held by a request and a checkpoint; slot 1 by two checkpoints of another
    request.  A plan that needs two fresh slots fails (one evictable slot), and the
    evictable checkpoints survive the failure."""
    c = SlotCache(2)
    a, sa, _, _ = c.open([1])
    c.checkpoint(a, [1])
    b, sb, _, _ = c.open([5, 6])
    c.checkpoint(b, [5])
    c.checkpoint(b, [5, 6])
    c.close(b)
    assert c.stats() == (0, 3, 1)
    with pytest.raises(SlotCacheError) as e:
        c.plan([a], T=2)  # the checkpointed source needs T = 2 fresh slots; one can be made
    assert e.value.status == CAPACITY
    assert c.stats() == (0, 3, 1) and c.refcount(sb) == 2
