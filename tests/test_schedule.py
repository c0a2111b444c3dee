"""Host-only checks of the tensor-core GEMM's work split (include/gptq_testing.h): the tile
schedule of the persistent CTAs covers every tile exactly once for every K-range mode, and the
tile width choice follows the cost model's intent.  No GPU needed."""
import itertools

import pytest

from post_weight_quantization_16_b200 import gptq as G

KLO_NONE, KLO_COL, KLO_ROW = 0, 1, 2
KHI_NONE, KHI_COL = 0, 1

SHAPES = [(128, 128, 128), (4096, 896, 128), (300, 1024, 256), (2048, 2048, 2048), (1024, 640, 1024),
          (8192, 3072, 1024), (96, 64, 32)]
MODES = [(KLO_NONE, KHI_NONE, 0), (KLO_COL, KHI_NONE, 0), (KLO_ROW, KHI_NONE, 0), (KLO_NONE, KHI_COL, 0),
         (KLO_NONE, KHI_NONE, 1)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("modes", MODES)
def test_every_tile_exactly_once(shape, modes):
    M, N, K = shape
    klo, khi, upper = modes
    if upper and M != N:
        pytest.skip("upper-triangle products are square")
    for bn, ctas in itertools.product((64, 128, 256), (1, 3, 37, 148, 1000)):
        r = G.lib().gptq_test_tile_schedule(M, N, K, klo, khi, upper, bn, ctas)
        assert r == 0, (shape, modes, bn, ctas, r)


def test_schedule_rejects_bad_arguments():
    assert G.lib().gptq_test_tile_schedule(128, 128, 128, 0, 0, 0, 96, 4) == -1
    assert G.lib().gptq_test_tile_schedule(0, 128, 128, 0, 0, 0, 64, 4) == -1


def test_tile_width_choice():
    pick = G.lib().gptq_test_pick_tile_n
    # a large dense product keeps the widest tile (fewest bytes per flop)
    assert pick(4096, 4096, 4096, KLO_NONE, KHI_NONE, 0, 148) == 256
    # a product with too few wide tiles for the SMs takes narrower ones
    assert pick(1024, 1024, 1024, KLO_COL, KHI_NONE, 0, 148) == 64
    # the sweep's short update (K = 128) over many columns stays wide
    assert pick(4096, 896, 128, KLO_NONE, KHI_NONE, 0, 148) == 256
    for args in [(128, 128, 128, 0, 0, 0, 148), (2048, 2048, 2048, 1, 0, 0, 148), (4096, 128, 128, 0, 0, 0, 148)]:
        assert pick(*args) in (64, 128, 256)
    assert pick(0, 128, 128, 0, 0, 0, 148) == -1
