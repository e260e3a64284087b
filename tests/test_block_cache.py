"""The device block cache's slot policy (hga_block_cache_plan), on the host:
hits keep their slot, misses fill empty slots first, then evict the least
recently used slot that the current call does not need (ties: lowest slot);
bad requests leave the cache unchanged."""
import numpy as np
import pytest

from segmented_fine_tuning_b200 import BlockCache, HgaError


def test_hand_worked_sequence():
    c = BlockCache(10, 4)
    s, m = c.plan([1, 2, 3])
    assert s.tolist() == [0, 1, 2] and m.tolist() == [1, 2, 3]  # empty slots in order
    s, m = c.plan([2, 5])
    assert s.tolist() == [1, 3] and m.tolist() == [5]  # 2 is a hit; 5 takes the last empty slot
    s, m = c.plan([6, 7])
    # no empty slot: slots 0 (block 1) and 2 (block 3) were last used by call 1, slots 1, 3 by call 2
    assert s.tolist() == [0, 2] and m.tolist() == [6, 7]
    s, m = c.plan([0, 1, 2, 3])
    # 2 hits in slot 1; oldest free slot 3 (call 2), then slots 0 and 2 (call 3) in slot order
    assert s.tolist() == [3, 0, 1, 2] and m.tolist() == [0, 1, 3]
    assert c.block_of_slot.tolist() == [1, 2, 3, 0]
    assert c.slot_of_block[:4].tolist() == [3, 0, 1, 2] and (c.slot_of_block[4:] == -1).all()


def test_repeat_is_all_hits():
    c = BlockCache(64, 16)
    need = [3, 9, 10, 11, 40]
    s1, m1 = c.plan(need)
    s2, m2 = c.plan(need)
    assert m1.tolist() == need and m2.size == 0 and s1.tolist() == s2.tolist()


def _model(cap, slots, calls):
    """Straightforward restatement of the policy, for the random comparison."""
    where = {}
    owner = [-1] * slots
    last = [-1] * slots
    out = []
    for t, need in enumerate(calls, start=1):
        for n in need:
            if n in where:
                last[where[n]] = t
        res, miss = [], []
        for n in need:
            if n in where:
                res.append(where[n])
                continue
            free = [x for x in range(slots) if owner[x] < 0 and last[x] != t]
            if free:
                x = free[0]
            else:
                cand = [x for x in range(slots) if last[x] != t]
                x = min(cand, key=lambda y: (last[y], y))
            if owner[x] >= 0:
                del where[owner[x]]
            owner[x], where[n], last[x] = n, x, t
            res.append(x)
            miss.append(n)
        out.append((res, miss))
    return out


def test_random_sequences_match_the_policy():
    rng = np.random.default_rng(7)
    for trial in range(20):
        cap, slots = int(rng.integers(5, 60)), int(rng.integers(1, 20))
        calls = []
        for _ in range(30):
            k = int(rng.integers(0, min(slots, cap) + 1))
            calls.append(sorted(rng.choice(cap, size=k, replace=False).tolist()))
        c = BlockCache(cap, slots)
        for (res, miss), need in zip(_model(cap, slots, calls), calls):
            s, m = c.plan(need)
            assert s.tolist() == res and m.tolist() == miss


@pytest.mark.parametrize("need", [[0, 1, 2, 3, 4], [2, 1], [1, 1], [-1], [10]])
def test_bad_requests_leave_the_cache_unchanged(need):
    c = BlockCache(10, 4)
    c.plan([0, 5])
    before = (c.slot_of_block.copy(), c.block_of_slot.copy(), c.last_use.copy(), c.c.tick)
    with pytest.raises(HgaError):
        c.plan(need)
    assert (c.slot_of_block == before[0]).all() and (c.block_of_slot == before[1]).all()
    assert (c.last_use == before[2]).all() and c.c.tick == before[3]


def test_reset_empties():
    c = BlockCache(8, 3)
    c.plan([1, 2])
    c.reset()
    assert (c.slot_of_block == -1).all() and (c.block_of_slot == -1).all() and c.c.tick == 0
    assert c.plan([4])[1].tolist() == [4]


def test_spaco_sampler_picks_k_blocks_per_sequence_and_caps_the_factor():
    """Host sampler of the sparse backward: exactly k of the t query blocks
    of every sequence, reproducible from the generator's seed, factor t/k
    (the inverse of the inclusion probability), capped when asked."""
    import torch
    from segmented_fine_tuning_b200 import spaco_sample_blocks
    g = torch.Generator().manual_seed(3)
    mask, scale = spaco_sample_blocks(4, 16, 4, g)
    assert mask.dtype == torch.uint8 and tuple(mask.shape) == (4, 16)
    assert (mask.sum(dim=1) == 4).all() and scale == 4.0
    again, _ = spaco_sample_blocks(4, 16, 4, torch.Generator().manual_seed(3))
    assert torch.equal(mask, again)
    _, capped = spaco_sample_blocks(1, 16, 1, torch.Generator().manual_seed(0), cap=8.0)
    assert capped == 8.0
    # over many draws every block is chosen with probability k/t
    counts = torch.zeros(16)
    gen = torch.Generator().manual_seed(11)
    for _ in range(2000):
        m, _ = spaco_sample_blocks(1, 16, 4, gen)
        counts += m[0].float()
    assert ((counts / 2000 - 0.25).abs() < 0.04).all()
    with pytest.raises(ValueError):
        spaco_sample_blocks(1, 16, 0, gen)
