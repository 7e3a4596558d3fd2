"""The index samplers of the GPU parity tests (host logic, no GPU).

A sampler that loses the top of the range leaves the last token tiles and
output tiles of a full-size forward unchecked, so these pins run on the CPU."""
import numpy as np
import pytest

from gpu_util import sample_indices, stratified_indices


@pytest.mark.parametrize("n,k,tile", [(2048, 48, 128), (14336, 384, 128), (8192, 48, 128), (28672, 384, 128),
                                      (4096, 512, 128), (1000, 48, 128), (300, 40, 128), (130, 64, 128)])
def test_sample_keeps_ends_and_last_tile(n, k, tile):
    for seed in range(5):
        s = sample_indices(n, k, seed, tile)
        assert s.dtype == np.int64
        assert np.all(np.diff(s) > 0) and s[0] >= 0 and s[-1] < n
        assert len(s) >= k
        last_tile = (n - 1) // tile * tile
        for must in (0, 1, n - 2, n - 1, last_tile, tile - 1, tile):
            if must < n:
                assert must in s, (n, k, seed, must)
        # the seeded draws reach the top quarter of the range
        assert np.sum(s >= (3 * n) // 4) >= k // 8, (n, k, seed)


def test_sample_small_range_is_everything():
    np.testing.assert_array_equal(sample_indices(40, 48, 1), np.arange(40))
    np.testing.assert_array_equal(sample_indices(48, 48, 1), np.arange(48))


@pytest.mark.parametrize("n,block", [(2048, 16), (4096, 16), (8192, 16), (14336, 128), (28672, 128),
                                     (1000, 16), (1025, 128), (5, 16)])
def test_stratified_meets_every_block(n, block):
    s = stratified_indices(n, block, 3)
    assert np.all(np.diff(s) > 0) and s[0] >= 0 and s[-1] == n - 1
    hit = np.zeros((n + block - 1) // block, dtype=bool)
    hit[s // block] = True
    assert hit.all()
