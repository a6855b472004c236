"""The backward kernel's mbarrier protocol, modelled on the CPU (see
protocol_model_bwd.py): both sides (latent rows over token chunks, token rows
over all latents), row or column statistics, the fused (dual) token side with
one row slot, two warpgroups (D <= 64) and one (D = 128), ragged shapes,
one-tile items and forced chunk counts."""
import pytest

from protocol_model_bwd import check

SHAPES = [(1, 2, 1000, 48, 16), (1, 1, 1, 1, 16), (2, 1, 530, 70, 128), (1, 2, 777, 300, 32),
          (2, 2, 1500, 128, 64), (1, 3, 1100, 200, 16), (1, 2, 650, 96, 128), (1, 1, 33, 129, 64)]
USES = [("latent", True, False), ("latent", False, False), ("token", True, False), ("token", False, False),
        ("token", True, True)]


@pytest.mark.parametrize("use", USES, ids=lambda u: f"{u[0]}-{'col' if u[1] else 'row'}{'-dual' if u[2] else ''}")
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_backward_protocol(shape, use):
    side, col_stats, dual = use
    check(*shape, side=side, col_stats=col_stats, dual=dual, grid=23)


@pytest.mark.parametrize("force", [1, 2, 7])
def test_backward_protocol_forced_chunks(force):
    check(1, 2, 3000, 64, 64, side="latent", col_stats=True, force_chunks=force, grid=23)
    check(1, 2, 3000, 64, 64, side="latent", col_stats=False, force_chunks=force, grid=23)


def test_backward_protocol_many_items_per_cta():
    """Several items per CTA (row slots reused, accumulators reset per item)."""
    check(2, 3, 2100, 300, 64, side="token", col_stats=True, dual=True, grid=5)
    check(2, 3, 2100, 300, 64, side="latent", col_stats=True, grid=5, force_chunks=9)


def test_model_catches_a_missing_pfree_wait():
    """Storing P/dS without waiting for the previous job's accumulating MMAs is
    the race the pfree barrier prevents; the model must see it."""
    with pytest.raises(AssertionError, match="P/dS overwritten"):
        check(1, 2, 3000, 64, 64, side="latent", col_stats=True, grid=23, skip_pfree_wait=True)


def test_model_catches_an_epilogue_before_the_last_accumulation():
    # planted: the item's epilogue reads the accumulators as soon as its last
    # P/dS is released, without waiting for that accumulating MMA
    with pytest.raises(AssertionError, match="last accumulation|still runs"):
        for seed in range(20):
            check(1, 2, 3000, 512, 64, side="token", col_stats=False, grid=7, seed=seed, dual=True,
                  no_deferred_wait=True)
