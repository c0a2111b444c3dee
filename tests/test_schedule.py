"""Host-only checks of the tensor-core GEMM's work split (include/gptq_testing.h): the tile
schedule of the persistent CTAs covers every tile exactly once for every K-range mode, and the
tile width choice follows the cost model's intent.  No GPU needed."""
import ctypes
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


def _factor_plan(n):
    cap = 4 * (n // 128) + 8
    nodes = (ctypes.c_int32 * (3 * cap))()
    spine = (ctypes.c_int32 * 64)()
    ns = ctypes.c_int()
    cnt = G.lib().gptq_test_factor_plan(n, nodes, cap, spine, 64, ctypes.byref(ns))
    assert 0 < cnt <= cap
    return [tuple(nodes[3 * i:3 * i + 3]) for i in range(cnt)], list(spine[:ns.value])


@pytest.mark.parametrize("n", [128, 256, 896, 1024, 1152, 2048, 2304, 3200, 4096, 5120, 7168, 11008, 14336, 28672, 32768])
def test_factor_plan_forms_every_slab_block_of_U(n):
    """The sweep reads U inside every aligned slab of 128-1024 columns (the update past a slab
    is D V U[slab, slab]): each such block must lie inside a node whose whole U the
    factorization forms.  Also: the leaves tile [0, n), every node is split into two parts that
    the plan holds, and the nodes left incomplete are exactly those gptq_get_factor completes,
    each after its left part is complete."""
    nodes, spine = _factor_plan(n)
    leaves = sorted((o, h) for o, h, _ in nodes if h == 128)
    assert [o for o, _ in leaves] == list(range(0, n, 128))
    full = {(o, h) for o, h, u in nodes if u}
    spans = {(o, h) for o, h, _ in nodes}
    for o, h, _ in nodes:
        if h > 128:  # a left part (o, h1) and a right part (o + h1, h - h1), both in the plan
            assert any((o, h1) in spans and (o + h1, h - h1) in spans for h1 in range(128, h, 128)), (o, h)
    for S in (128, 256, 512, 1024):
        for a in range(0, n, S):
            b = min(n, a + S)
            assert any(o <= a and b <= o + h for o, h in full), (S, a, b)
    incomplete = sorted(h for o, h, u in nodes if not u)
    assert all(o == 0 for o, h, u in nodes if not u)  # only the left edge
    assert sorted(spine) == incomplete and spine == sorted(spine)  # completed smallest first
    for h in spine:  # its left part is complete by the time it is completed
        left = max(hh for oo, hh in spans if oo == 0 and hh < h)
        assert (0, left) in full or left in spine[:spine.index(h)]
