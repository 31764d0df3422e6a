"""Host logic of the multi-level padded decode (no GPU): level choice and the
padded slot list the kernels receive."""
import pytest

from linear_attention_13_b200.decode_batch import DEFAULT_LEVELS, padded_slots, pick_level, validate_levels


def test_pick_level_smallest_that_fits():
    assert pick_level(1) == 1
    assert pick_level(3) == 4
    assert pick_level(4) == 4
    assert pick_level(129) == 256
    assert pick_level(5, levels=(16, 8)) == 8
    for n in range(1, max(DEFAULT_LEVELS) + 1):
        lv = pick_level(n)
        assert lv >= n and all(x < n or x >= lv for x in DEFAULT_LEVELS)


@pytest.mark.parametrize("n", [0, -1, 257])
def test_pick_level_rejects(n):
    with pytest.raises(ValueError):
        pick_level(n)


def test_padded_slots():
    assert padded_slots([5, 2, 7], 4, num_slots=8) == [5, 2, 7, -1]
    assert padded_slots([0], 1, num_slots=1) == [0]
    assert padded_slots([], 2, num_slots=1) == [-1, -1]


@pytest.mark.parametrize("slots,level,num", [([1, 1], 2, 4), ([4], 1, 4), ([-1], 1, 4), ([0, 1, 2], 2, 4)])
def test_padded_slots_rejects(slots, level, num):
    with pytest.raises(ValueError):
        padded_slots(slots, level, num)


def test_validate_levels():
    assert validate_levels((8, 1, 4)) == (1, 4, 8)
    for bad in ((), (0, 4), (4, 4)):
        with pytest.raises(ValueError):
            validate_levels(bad)
