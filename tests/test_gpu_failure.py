"""Failure detection on the GPU without a GPU fault: a device-side bounded wait that runs out
(an mbarrier nothing arrives on, with a 1 ms limit) is reported as GPTQ_ERR_TIMEOUT by the
next gptq_synchronize and leaves the context usable; a host wait with a short limit returns
GPTQ_ERR_TIMEOUT while a kernel is still running.  Also the per-kernel instrumentation, which
must not change any result."""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import synth
from post_weight_quantization_16_b200 import gptq as G
from tests import gpu_helpers as GH

pytestmark = pytest.mark.gpu
TINY = synth.WORKLOADS["tiny_256x512"][0]


def _small_run(ctx, layer, qs, X, W):
    ctx.reset()
    ctx.accumulate_hessian(GH.bf16_to_dev(X))
    perm = ctx.prepare(qs.damp, qs.desc_act)
    out = ctx.quantize_layer(torch.from_numpy(W).to(GH.DEV), qs.bits, qs.group_size, qs.sym)
    ctx.synchronize()
    return perm.cpu().numpy(), {k: v.cpu().numpy() for k, v in out.items() if v is not None}


def test_device_wait_that_runs_out_is_reported_and_the_context_survives():
    layer = synth.scaled_layer(TINY, m=64, n=256, n_tok=512)
    qs = synth.QuantSetting(4, 128, False, 0.01, True)
    X, W = synth.make_x_bf16(layer), synth.make_w_fp16(layer)
    with G.GPTQContext(layer.n, layer.m, 0) as ctx:
        perm0, ref = _small_run(ctx, layer, qs, X, W)
        assert G.lib().gptq_test_bounded_wait(ctx._h, 1_000_000) == G.OK   # 1 ms
        with pytest.raises(G.GPTQError) as ei:
            ctx.synchronize()
        assert ei.value.status == G.ERR_TIMEOUT
        ctx.synchronize()                       # the status word was cleared
        perm1, out = _small_run(ctx, layer, qs, X, W)
        assert np.array_equal(perm0, perm1)
        for k in ref:
            assert np.array_equal(ref[k], out[k]), k


def test_host_wait_with_a_short_limit_returns_timeout(monkeypatch):
    with G.GPTQContext(256, 16, 0) as ctx:
        assert G.lib().gptq_test_bounded_wait(ctx._h, 300_000_000) == G.OK  # a 300 ms kernel
        monkeypatch.setenv("GPTQ_SYNC_TIMEOUT_MS", "5")
        with pytest.raises(G.GPTQError) as ei:
            ctx.synchronize()                   # the host gives up after 5 ms
        assert ei.value.status == G.ERR_TIMEOUT
        monkeypatch.delenv("GPTQ_SYNC_TIMEOUT_MS")
        with pytest.raises(G.GPTQError) as ei:
            ctx.synchronize()                   # the kernel itself gave up and said so
        assert ei.value.status == G.ERR_TIMEOUT
        ctx.synchronize()


def test_profiling_records_every_role_and_changes_no_result(monkeypatch):
    monkeypatch.setenv("GPTQ_SLAB_WIDTH", "256")
    layer = synth.scaled_layer(TINY, m=96, n=2304, n_tok=2048)
    qs = synth.QuantSetting(4, 128, False, 0.01, True)
    X, W = synth.make_x_bf16(layer), synth.make_w_fp16(layer)
    with G.GPTQContext(layer.n, layer.m, 0) as ctx:
        perm0, ref = _small_run(ctx, layer, qs, X, W)
        ctx.set_profiling(True)
        perm1, out = _small_run(ctx, layer, qs, X, W)
        prof = ctx.get_profile()
        ctx.set_profiling(False)
        assert ctx.get_profile() == {}
    assert np.array_equal(perm0, perm1)
    for k in ref:
        assert np.array_equal(ref[k], out[k]), k
    n = layer.n
    assert prof["hessian_syrk_pair"]["launches"] == 1
    assert prof["hessian_syrk_pair"]["flops"] == layer.n_tok * n * (n + 1)
    assert prof["leaf_chol_inv"]["launches"] == n // 128
    assert prof["sweep_slab"]["launches"] == (n + 255) // 256   # one per 256-column slab
    # the factorization's algorithmic work: n^3/3 for the Cholesky factor and n^3/3 for its
    # inverse, plus lower-order terms of the diagonals, less the two products of the root
    # (columns [0, 1024) + [1024, 2304)) that only the full U needs: T = V12 U22 and
    # U12 = -U11 T (h1 h2 (h2 + 1) and h2 h1 (h1 + 1) flops)
    h1, h2 = 1024, n - 1024
    skipped = h1 * h2 * (h2 + 1) + h2 * h1 * (h1 + 1)
    f = sum(v["flops"] for k, v in prof.items() if ":factor" in k or k == "leaf_chol_inv")
    assert 2 * n ** 3 / 3 - skipped <= f <= 1.02 * 2 * n ** 3 / 3 - skipped, f
    # the tensor-core trailing update: the columns past each 256-column slab (the updates
    # inside a slab run in the slab kernel) ...
    far = prof["gemm_tf32x3:trailing_far"]["flops"]
    assert far == 2 * layer.m * sum(min(256, n - s0) * (n - s0 - 256) for s0 in range(0, n - 256, 256))
    # ... with Vs = V blockdiag(U_SS): the rows above each 256-column block times its
    # upper-triangular U block, once per prepared factor
    vs = prof["gemm_tf32x3:trailing_vs"]
    assert vs["launches"] == 1
    assert vs["flops"] == 2 * sum(b0 * (256 * 257 // 2) for b0 in range(0, n, 256))
    assert all(v["ms"] > 0 for v in prof.values())
