"""The measurement-only microbenchmarks (include/mcs_micro.h) run and give
plausible rates: the MMA timing covers every MMA (no completion wait ran out)
and stays at or below the nominal peak (well above a floor when nothing else
runs); the exponential rate is positive and at most the SM's lane count per
cycle."""
import pytest
import torch

from sparse_attention_diffusion_mcs_b200 import micro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", list(micro.MMA_SHAPES))
@pytest.mark.parametrize("load", list(micro.MMA_LOADS))
@pytest.mark.parametrize("chains", [1, 2])
def test_mma_rate_is_plausible(shape, load, chains):
    r = micro.mma_rate(shape, load, chains=chains, batches=256)
    # at most the nominal dense bf16 rate of one SM (8192 FLOP/cycle); alone, not absurdly slow
    assert 0 < r["flop_per_sm_per_cycle"] <= 8192 * 1.02, r
    if load == "none":
        assert r["flop_per_sm_per_cycle"] > 1000, r


def test_ex2_rate_is_plausible():
    r = micro.ex2_rate(16, iters=512)
    assert 1.0 < r["ex2_per_sm_per_cycle"] <= 128.0, r
