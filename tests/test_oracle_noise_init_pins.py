"""Pins of the coordinated noise initialisation oracle (oracle/noise_init.py): a hand-worked
selection, the structural properties the reading fixes, and a planted mistake per rule."""
import numpy as np
import pytest

import oracle as O
import oracle.noise_init as N
from workloads import make_noise_permutations


def pin_hand_worked_selection():
    # pool of 6 frames, previous block used frames 1 and 4, permutation 4 0 1 5 3 2
    assert N.coordinated_frames(6, 2, [1, 4], [4, 0, 1, 5, 3, 2]) == [0, 5]
    assert N.coordinated_frames(6, 3, [], [4, 0, 1, 5, 3, 2]) == [4, 0, 1]


def pin_schedule_properties():
    frames = [2] * 40 + [1]
    W = 8
    perms = make_noise_permutations(len(frames), 16, seed=3)
    sched = N.coordinated_schedule(frames, W, perms)
    assert [len(f) for f in sched] == frames
    assert sched[:W] == [[2 * b, 2 * b + 1] for b in range(W)]      # the pool itself, in order
    for b in range(W, len(frames)):
        f = sched[b]
        assert len(set(f)) == len(f) and all(0 <= x < 16 for x in f)
        assert not set(f) & set(sched[b - 1])                        # adjacent blocks share no frame
        order = [x for x in perms[b] if x not in set(sched[b - 1])]
        assert f == order[:len(f)]                                   # the permutation's order
    used = {x for f in sched[W:] for x in f}
    assert used == set(range(16))                                    # the full pool is drawn from


def pin_gather_is_the_pool_frames():
    pool = np.arange(5 * 3 * 2, dtype=np.float64).reshape(5, 3, 2)
    got = N.gather_frames(pool, [4, 1])
    assert np.array_equal(got, np.concatenate([pool[4], pool[1]]))


PINS = [pin_hand_worked_selection, pin_schedule_properties, pin_gather_is_the_pool_frames]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_rejects_small_pools_and_bad_permutations():
    with pytest.raises(ValueError):
        N.coordinated_frames(3, 2, [0, 1], [0, 1, 2])
    with pytest.raises(ValueError):
        N.coordinated_frames(3, 1, [], [0, 0, 2])


def _mutants():
    cf, cs, gf = N.coordinated_frames, N.coordinated_schedule, N.gather_frames

    def no_exclusion(pool_frames, block_frames, prev, perm):
        return [int(f) for f in perm][:block_frames]

    def sorted_pick(pool_frames, block_frames, prev, perm):
        ex = set(prev)
        return sorted(f for f in perm if f not in ex)[:block_frames]

    def window_shuffled(block_frames, W, perms):
        out = cs(block_frames, W, perms)
        out[1] = list(reversed(out[1]))
        return out

    def gather_reversed(pool, frames):
        return gf(pool, list(reversed(frames)))

    return [("coordinated_frames", no_exclusion), ("coordinated_frames", sorted_pick),
            ("coordinated_schedule", window_shuffled), ("gather_frames", gather_reversed)]


@pytest.mark.parametrize("idx", range(4))
def test_planted_mistake_fails_a_pin(idx, monkeypatch):
    name, fn = _mutants()[idx]
    monkeypatch.setattr(N, name, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {fn.__name__}"
