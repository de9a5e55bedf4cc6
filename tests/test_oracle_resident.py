"""Pins of the resident-page oracle: invariants any correct reuse policy must keep, and a
small hand-worked sequence."""
import numpy as np
import pytest

from oracle.resident import resident_update


def _state(n_blocks, n_slots):
    return np.full(n_blocks, -1, np.int64), np.full(n_slots, -1, np.int64)


def test_hand_worked_sequence():
    sob, bos = _state(10, 3)
    # first selection: everything misses, slots filled in order
    ps, cp = resident_update([2, 5, 7], sob, bos)
    assert ps.tolist() == [0, 1, 2] and cp == [(2, 0), (5, 1), (7, 2)]
    # 5 stays; 2 and 7 leave; 1 and 9 come into the freed slots 0 and 2 (ascending)
    ps, cp = resident_update([1, 5, 9], sob, bos)
    assert cp == [(1, 0), (9, 2)] and ps.tolist() == [0, 1, 2]
    assert sob[2] == -1 and sob[7] == -1 and bos.tolist() == [1, 5, 9]
    # the same selection again copies nothing
    ps, cp = resident_update([1, 5, 9], sob, bos)
    assert cp == [] and ps.tolist() == [0, 1, 2]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_invariants_over_random_sequences(seed):
    rng = np.random.default_rng(seed)
    n_blocks, n_slots, k = 300, 40, 32
    sob, bos = _state(n_blocks, n_slots)
    cur = np.sort(rng.choice(n_blocks, k, replace=False))
    total = 0
    for step in range(60):
        if step:  # drift: replace a few selected blocks
            keep = rng.choice(k, k - int(rng.integers(0, 6)), replace=False)
            pool = np.setdiff1d(np.arange(n_blocks), cur[keep])
            cur = np.sort(np.concatenate([cur[keep], rng.choice(pool, k - len(keep), replace=False)]))
        before = {int(b): int(sob[b]) for b in cur if sob[b] >= 0}
        ps, cp = resident_update(cur, sob, bos)
        total += len(cp)
        # every selected block is resident, in the slot the page list names
        assert all(bos[s] == b for b, s in zip(cur, ps))
        # the maps are inverse to each other
        for s in range(n_slots):
            if bos[s] >= 0:
                assert sob[bos[s]] == s
        assert int((sob >= 0).sum()) == int((bos >= 0).sum())
        # hits keep their slot; copies are exactly the misses
        assert all(sob[b] == s for b, s in before.items())
        assert sorted(b for b, _ in cp) == sorted(set(int(b) for b in cur) - set(before))
        assert len({s for _, s in cp}) == len(cp)
    assert total < 60 * k  # reuse happened


def test_refuses_too_few_slots():
    sob, bos = _state(10, 2)
    with pytest.raises(AssertionError):
        resident_update([1, 2, 3], sob, bos)
