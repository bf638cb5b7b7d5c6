"""Direct pins of the oracle's small helpers (token -> frame / partition,
KV-group offsets, a group's keys, the token-level frame mask), each against
values worked out by hand."""
import numpy as np
import pytest

from oracle import groups, masks, step


def test_frame_and_partition_of_tokens_at_the_boundaries():
    off = [0, 3, 7, 10]
    assert masks.frame_of([0, 2, 3, 6, 7, 9], off).tolist() == [0, 0, 1, 1, 2, 2]
    assert [step.partition_of(t, off) for t in (0, 2, 3, 6, 7, 9)] == [0, 0, 1, 1, 2, 2]


def test_uniform_groups_and_their_checks():
    assert groups.uniform_group_off(10, 4) == [0, 4, 8, 10]
    assert groups.uniform_group_off(3, 0) == [0, 1, 2, 3]
    assert groups.check_group_off([0, 4], 4) == [0, 4]
    for bad in ([0, 2, 2, 4], [1, 4], [0, 3], [0, 3, 2, 4]):
        with pytest.raises(ValueError):
            groups.check_group_off(bad, 4)


def test_keys_of_a_group_span_its_partitions():
    po, go = [0, 5, 9, 20], [0, 2, 3]
    assert groups.unit_keys(po, go, 0).tolist() == list(range(9))
    assert groups.unit_keys(po, go, 1).tolist() == list(range(9, 20))


def test_token_mask_of_the_frame_tile_pattern():
    # 4 frames of 2 tokens; frame f sees f-1, f, f+1 and 0
    fo = [0, 2, 4, 6, 8]
    fm = [[1 if (abs(f - g) <= 1 or g == 0) else 0 for g in range(4)] for f in range(4)]
    allowed = masks.token_allowed(np.arange(8), np.arange(8), fo, fm)
    want = np.array([[1, 1, 1, 1, 0, 0, 0, 0],
                     [1, 1, 1, 1, 0, 0, 0, 0],
                     [1, 1, 1, 1, 1, 1, 0, 0],
                     [1, 1, 1, 1, 1, 1, 0, 0],
                     [1, 1, 1, 1, 1, 1, 1, 1],
                     [1, 1, 1, 1, 1, 1, 1, 1],
                     [1, 1, 0, 0, 1, 1, 1, 1],
                     [1, 1, 0, 0, 1, 1, 1, 1]], dtype=bool)
    assert (allowed == want).all()
    assert masks.token_allowed([0, 1], [5, 6, 7]).all()          # no mask: everything
