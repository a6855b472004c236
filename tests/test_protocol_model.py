"""The attention kernel's mbarrier protocol, modelled on the CPU (see
protocol_model.py), over shapes that exercise ragged tiles, one-tile and
jobless items, interleaved and shared stage rings, and forced chunk counts,
for both kernel configurations (two row tiles on 128-row key/value tiles with
two column shares per row for the split passes, three on 64-row tiles for
the decode)."""
import pytest

from protocol_model import check

SHAPES = [(1, 2, 1024, 16, 16), (1, 1, 1, 1, 16), (1, 2, 7, 5, 16), (2, 1, 129, 17, 32),
          (1, 3, 300, 64, 64), (3, 2, 513, 64, 16), (1, 1, 4097, 256, 32), (1, 2, 2000, 512, 64),
          (1, 1, 640, 100, 32), (1, 2, 1500, 384, 64)]


@pytest.mark.parametrize("nw", [2, 3])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_protocol(shape, nw):
    check(*shape, NW=nw, grid=37)


@pytest.mark.parametrize("nw", [2, 3])
@pytest.mark.parametrize("force", [1, 2, 7])
def test_protocol_forced_chunks(nw, force):
    check(2, 2, 3001, 128, 32, force_chunks=force, NW=nw, grid=37)


def test_per_warpgroup_rings_on_the_16641_token_workload():
    check(2, 8, 16641, 128, 32, NW=3, grid=148, mode="split")
    check(2, 8, 16641, 128, 32, NW=2, grid=148, mode="split")


def test_model_catches_the_shared_ring_race():
    """With one shared stage ring in interleaved mode, consecutive fills of a
    stage can belong to different warpgroups and a parity wait can pass on the
    wrong fill; the model must see a stage holding the wrong tile.  The chunk
    count is pinned to 37 (592 items of 8 tiles), a split in which the model
    interleaves the warpgroups closely enough to show the race."""
    with pytest.raises(AssertionError, match="kv stage holds wrong tile"):
        check(2, 8, 16641, 128, 32, NW=3, grid=148, mode="split", shared_ring=True, force_chunks=37)


def test_column_shares_in_split_and_single_share_decode():
    """The split passes on 128-column jobs run two column shares per row (their
    exchange pairs the same job), the decode one; both write each output once."""
    res = check(1, 2, 1500, 384, 64, NW=2, grid=37, mode="split")
    assert res
    check(1, 2, 1500, 384, 32, NW=2, grid=37, mode="split")      # D <= 32: one warp per row
    check(1, 2, 1500, 384, 32, NW=2, grid=37, mode="split", CS=2)  # two shares at D = 32 (not launched)
    check(1, 2, 700, 64, 64, NW=2, grid=37, mode="split")        # interleaved, two shares per stream


def test_model_catches_a_score_buffer_released_by_one_share():
    """If the next score MMA waited for one share only, it could overwrite the
    scores the other share has not read yet; the model must see it."""
    with pytest.raises(AssertionError, match="S overwritten before read"):
        for seed in range(6):
            check(1, 2, 3000, 256, 64, NW=2, grid=5, mode="split", seed=seed, plant="sfree_one_share")
