"""Host-only check of gptq_rtn_quantize's percentile positions (include/gptq_testing.h): the ranks
and fp32 weights the call hands its kernel, applied to sorted fp32 values with the kernel's
interpolation, give np.percentile's result bit for bit (the clip ratio of "模型量化实战…" §3.1
takes its range from np.percentile).  No GPU needed."""
import ctypes

import numpy as np
import pytest

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import gptq as G


def _pos(p, k):
    lo, hi, t, omt = ctypes.c_int(), ctypes.c_int(), ctypes.c_float(), ctypes.c_float()
    assert G.lib().gptq_test_pct_position(p, k, ctypes.byref(lo), ctypes.byref(hi), ctypes.byref(t),
                                          ctypes.byref(omt)) == 0
    return lo.value, hi.value, np.float32(t.value), np.float32(omt.value)


def _lerp(a, b, t, omt):
    """The kernel's interpolation, one fp32 rounding per operation."""
    d = b - a
    return a + d * t if t < np.float32(0.5) else b - d * omt


@pytest.mark.parametrize("k", [1, 2, 3, 32, 128, 1000, 4096, 11008])
def test_positions_reproduce_numpy_percentile(k):
    rng = np.random.default_rng(k)
    v = np.sort(rng.standard_normal((16, k)).astype(np.float16).astype(np.float32), axis=1)
    ps = [0.0, 50.0, 100.0] + [float(x) for x in rng.uniform(0.0, 100.0, 20)]
    for c in (0.9, 0.95, 0.99, 0.999, 0.5, 0.3, 0.01):
        for sym in (True, False):
            ps += list(O.clip_percentiles(c, sym))
    for p in ps:
        lo, hi, t, omt = _pos(p, k)
        assert 0 <= lo <= hi <= k - 1 and hi - lo <= 1 and np.float32(1.0) - t == omt
        assert np.array_equal(_lerp(v[:, lo], v[:, hi], t, omt), np.percentile(v, p, axis=1)), p


def test_position_rejects_bad_arguments():
    lo, hi, t, omt = ctypes.c_int(), ctypes.c_int(), ctypes.c_float(), ctypes.c_float()
    args = (ctypes.byref(lo), ctypes.byref(hi), ctypes.byref(t), ctypes.byref(omt))
    for p, k in ((-1.0, 8), (100.5, 8), (float("nan"), 8), (50.0, 0)):
        assert G.lib().gptq_test_pct_position(p, k, *args) == -1
    assert G.lib().gptq_test_pct_position(50.0, 8, None, *args[1:]) == -1
