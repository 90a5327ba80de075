"""Head-block partition of one layer (shard.py), host only: the blocks cover
every flattened head exactly once, in order, contiguous, sizes differing by
at most one; a block is a view at its head offset, not a copy."""
import pytest
import torch

from sparse_attention_diffusion_mcs_b200 import shard


@pytest.mark.parametrize("BH,world", [(24, 1), (24, 2), (24, 8), (7, 3), (3, 8), (0, 2), (48, 5)])
def test_blocks_partition_the_heads(BH, world):
    ranges = [shard.head_range(BH, world, r) for r in range(world)]
    covered = []
    for start, count in ranges:
        covered.extend(range(start, start + count))
    assert covered == list(range(BH))
    counts = [c for _, c in ranges]
    assert max(counts) - min(counts) <= 1
    assert counts == sorted(counts, reverse=True)       # the larger blocks come first


def test_bad_partitions_are_refused():
    for args in [(4, 0, 0), (4, 2, 2), (4, 2, -1), (-1, 2, 0)]:
        with pytest.raises(ValueError):
            shard.head_range(*args)


def test_shard_is_a_view_at_the_head_offset():
    B, H, N, d = 2, 3, 5, 4
    x = torch.arange(B * H * N * d, dtype=torch.float32).view(B, H, N, d)
    for world in (1, 2, 4):
        parts = []
        for r in range(world):
            v = shard.shard(x, world, r)
            start, count = shard.head_range(B * H, world, r)
            assert v.shape == (1, count, N, d) and v.is_contiguous()
            if count:
                assert v.data_ptr() == x.data_ptr() + start * N * d * x.element_size()
            parts.append(v[0])
        assert torch.equal(torch.cat(parts), x.view(B * H, N, d))
    with pytest.raises(ValueError):
        shard.shard(x.transpose(2, 3), 2, 0)
