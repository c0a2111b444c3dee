"""Host-side checks of the C ABI (no GPU): the library loads, exports every function the
header declares, and validates arguments before touching the device."""
import ctypes
import os

import pytest

from post_weight_quantization_16_b200 import build as B
from post_weight_quantization_16_b200 import gptq as G


@pytest.fixture(scope="module")
def L():
    B.build()
    return G.lib()


def test_library_exports_every_header_function(L):
    names = G.header_functions()
    assert len(names) >= 13
    for nm in names:
        assert hasattr(L, nm), nm
    # and the binding declares a signature for each of them
    assert set(names) == set(G._SIGS)


def test_status_strings(L):
    for s in range(8):
        assert L.gptq_status_string(s)
    assert b"positive definite" in L.gptq_status_string(G.ERR_NOT_PD)


def test_workspace_bytes(L):
    n, m = 4096, 4096
    b = L.gptq_workspace_bytes(n, m)
    assert b >= 4 * n * n * 4 + m * n * 4
    assert L.gptq_workspace_bytes(100, 4) == 0        # n % 128
    assert L.gptq_workspace_bytes(4096, 0) == 0       # m_max
    assert L.gptq_workspace_bytes(65536, 1) == 0      # n too large
    assert L.gptq_workspace_bytes(28672, 8192) > 14e9


def test_create_rejects_bad_arguments_before_any_device_call(L):
    h = ctypes.c_void_p()
    assert L.gptq_create(ctypes.byref(h), 100, 16, 0, None) == G.ERR_ARG
    assert L.gptq_create(ctypes.byref(h), 512, 0, 0, None) == G.ERR_ARG
    assert L.gptq_create(ctypes.byref(h), 512, 16, -1, None) == G.ERR_ARG
    assert L.gptq_create(None, 512, 16, 0, None) == G.ERR_ARG


def test_create_reports_oom_without_allocating(L, monkeypatch):
    monkeypatch.setenv("GPTQ_MAX_WORKSPACE_BYTES", "1000")
    h = ctypes.c_void_p()
    assert L.gptq_create(ctypes.byref(h), 512, 16, 0, None) == G.ERR_OOM
    assert not h.value


def test_null_context_is_an_argument_error(L):
    assert L.gptq_hessian_accumulate(None, None, 0, 0) == G.ERR_ARG
    assert L.gptq_prepare(None, 0.01, 0, None) == G.ERR_ARG
    assert L.gptq_quantize_layer(None, None, 1, G.QParams(4, 128, 0), None, None, None, None, None) == G.ERR_ARG
    assert L.gptq_synchronize(None) == G.ERR_ARG
    assert L.gptq_reset(None) == G.ERR_ARG
    assert L.gptq_destroy(None) == G.OK


@pytest.mark.skipif(os.path.exists("/dev/nvidia0"), reason="checks the no-GPU behaviour")
def test_no_cpu_fallback_without_a_device(L):
    h = ctypes.c_void_p()
    assert L.gptq_create(ctypes.byref(h), 512, 16, 0, None) == G.ERR_CUDA


def test_binding_fails_loudly_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(G, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(G, "_LIB", None)
    with pytest.raises(RuntimeError, match="not built"):
        G.lib()


def test_new_calls_reject_a_null_context(L):
    assert L.gptq_get_dead_columns(None, None) == G.ERR_ARG
    assert L.gptq_set_profiling(None, 1) == G.ERR_ARG
    cnt = ctypes.c_int()
    assert L.gptq_get_profile(None, None, 0, ctypes.byref(cnt)) == G.ERR_ARG
    assert L.gptq_test_bounded_wait(None, 1000) == G.ERR_ARG


def test_dequant_matmul_workspace_is_a_pure_size_function(L):
    assert L.gptq_dequant_matmul_workspace_bytes(16, 4096, 4096, 1) >= 256 + 16 * 4096 * 2
    assert L.gptq_dequant_matmul_workspace_bytes(16, 4096, 4096, 0) < L.gptq_dequant_matmul_workspace_bytes(
        16, 4096, 4096, 1)
    assert L.gptq_dequant_matmul_workspace_bytes(16, 4096, 100, 0) == 0      # n % 128
    assert L.gptq_dequant_matmul_workspace_bytes(0, 4096, 4096, 0) == 0      # no tokens
    assert L.gptq_dequant_matmul(None, 1, None, None, None, None, 1, 128, G.QParams(4, 128, 0), None, None, 0, 0,
                                 None) == G.ERR_ARG


def test_rtn_quantize_rejects_bad_arguments_before_any_device_call(L):
    """Every case below is refused on the host, so no pointer is ever dereferenced."""
    p = ctypes.c_void_p(1 << 20)
    qp = G.QParams(8, -1, 1)
    assert L.gptq_rtn_quantize(None, 16, 512, qp, 0.99, None, p, p, p, None, 0, None) == G.ERR_ARG
    assert L.gptq_rtn_quantize(p, 16, 512, qp, 0.99, None, None, p, p, None, 0, None) == G.ERR_ARG
    for clip in (0.0, -0.5, 1.5, float("nan"), float("inf")):
        assert L.gptq_rtn_quantize(p, 16, 512, qp, clip, None, p, p, p, None, 0, None) == G.ERR_ARG, clip
    assert L.gptq_rtn_quantize(p, 16, 500, qp, 0.99, None, p, p, p, None, 0, None) == G.ERR_ARG      # n % 128
    assert L.gptq_rtn_quantize(p, 0, 512, qp, 0.99, None, p, p, p, None, 0, None) == G.ERR_ARG       # no rows
    assert L.gptq_rtn_quantize(p, 16, 512, G.QParams(5, -1, 1), 0.99, None, p, p, p, None, 0, None) == G.ERR_ARG
    assert L.gptq_rtn_quantize(p, 16, 512, G.QParams(4, 96, 0), 0.99, None, p, p, p, None, 0, None) == G.ERR_ARG


def test_sequential_keeps_one_context_per_width_and_grows_it(monkeypatch):
    """The binding's context bookkeeping for quantize_sequential, with a stand-in context class."""
    import types
    made = []

    class FakeContext:
        def __init__(self, n, m_max, device, stream):
            self.n, self.m_max, self.closed = n, m_max, False
            made.append(self)

        def close(self):
            self.closed = True

    monkeypatch.setattr(G, "GPTQContext", FakeContext)
    dev, st = types.SimpleNamespace(index=0), types.SimpleNamespace(cuda_stream=7)
    ctxs = {}
    a = G._sequential_context(ctxs, 256, 100, dev, st)
    assert G._sequential_context(ctxs, 256, 50, dev, st) is a              # fewer rows: reused
    b = G._sequential_context(ctxs, 256, 300, dev, st)                     # more rows: replaced
    assert b is not a and a.closed and b.m_max == 300 and not b.closed
    c = G._sequential_context(ctxs, 512, 10, dev, st)
    assert len(ctxs) == 2 and c.n == 512
    other = G._sequential_context(ctxs, 256, 10, dev, types.SimpleNamespace(cuda_stream=9))
    assert other is not b and len(ctxs) == 3                                # one per stream
    loose = G._sequential_context(None, 256, 10, dev, st)
    assert loose not in ctxs.values() and len(made) == 5
    G.close_contexts(ctxs)
    assert not ctxs and b.closed and c.closed and other.closed
