"""The work plan of the 2-SM pair kernels, checked on the host (no GPU):
``slr_plan_check`` builds the plan for a shape as a launch would and walks
every pair's chunk sequence.  The layer's product is a sum over the K stages
of each output tile (LoSparse, section 3.2), so a sound plan covers every
(row tile, 16-token unit, K stage) exactly once and every tile's rank stages
exactly once, whether the last round of tiles is dealt whole, split by tokens
or split along K."""
import pytest

import sparse_rank_linear_02_b200 as slr

# (M, d_out, d_in, r): the benchmark layers and ragged shapes (rows past a
# tile, tokens past a unit, K stages fewer than pairs, one tile, long K).
SHAPES = [
    (2048, 14336, 4096, 64), (4096, 1024, 4096, 64), (4096, 4096, 4096, 64), (4096, 4096, 14336, 64),
    (1024, 8192, 28672, 64), (512, 8192, 28672, 128), (256, 8192, 28672, 256), (128, 8192, 28672, 64),
    (1024, 28672, 8192, 64), (65, 512, 256, 8), (129, 136, 384, 8), (300, 512, 640, 128),
    (513, 1024, 1024, 256), (250, 1000, 8192, 64), (700, 2048, 4096, 256), (100, 296, 1024, 64),
    (37, 200, 256, 16), (1000, 4096, 384, 8), (8192, 8192, 28672, 64), (1, 4096, 4096, 64),
]
PAIRS = [74, 66, 33, 7, 1]


@pytest.mark.parametrize("M,d_out,d_in,r", SHAPES)
def test_pair_plans_cover_every_stage_once(M, d_out, d_in, r):
    for kernel in ("2sm128", "2sm240", "2sm256", "2smtall"):
        tails = ("whole", "tokens", "k") if kernel == "2smtall" else ("whole", "tokens")
        for tail in tails:
            for pairs in PAIRS:
                for chu in (0, 10):
                    bad = slr.plan_check(M, d_out, d_in, r, kernel, tail, pairs, chu)
                    assert bad == 0, (kernel, tail, pairs, chu, bad)


def test_plan_check_arguments():
    assert slr.plan_check(2048, 14336, 4096, 64, "2sm240", "k", 74) == -1   # K split: 512-row kernel only
    assert slr.plan_check(2048, 14336, 4000, 64, "2smtall", "tokens", 74) == -1   # d_in % 128
    assert slr.plan_check(2048, 14336, 4096, 12, "2smtall", "tokens", 74) == -1   # r % 8
    assert slr.plan_check(0, 14336, 4096, 64, "2smtall", "tokens", 74) == -1
    assert slr.plan_check(2048, 14336, 4096, 64, "2smtall", "tokens", 0) == -1
    assert slr.plan_check(2048, 14336, 4096, 64, "2smtall", "tokens", 129) == -1
    assert slr.plan_check(1 << 20, 1 << 16, 1 << 14, 64, "2smtall", "tokens", 74) == -1   # too large to walk
