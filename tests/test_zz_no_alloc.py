"""gptq_quantize_layer_noalloc — the quantize entry point for callers that cannot allocate
device memory themselves (a host that owns a fixed device-memory budget, or code where
cudaMalloc/cudaFree, which synchronize the device, are not allowed).  Its scratch is a fixed
array inside the library; these tests check it against the context-based
gptq_quantize_layer through the C ABI, on two calls in a row, and that requests beyond the
array's size are refused.

The file name sorts last so that a run that stops at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

from post_weight_quantization_16_b200 import gptq as G
from post_weight_quantization_16_b200 import synth


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_refuses_sizes_beyond_its_scratch():
    L = G.lib()
    qp = G.QParams(4, 128, 0)
    dummy = ctypes.c_void_p(16)  # never dereferenced: the size check comes first
    # m * n above 2^20
    assert L.gptq_quantize_layer_noalloc(dummy, 1024, 2048, dummy, dummy, None, qp, dummy, dummy, dummy,
                                         None, None, 0, None) == G.ERR_ARG
    # m above 4096
    assert L.gptq_quantize_layer_noalloc(dummy, 4097, 128, dummy, dummy, None, qp, dummy, dummy, dummy,
                                         None, None, 0, None) == G.ERR_ARG


@pytest.mark.gpu
def test_noalloc_matches_context_path_on_two_calls():
    from tests import gpu_helpers as GH

    layer = synth.scaled_layer(synth.WORKLOADS["tiny_256x512"][0], m=200, n=1024, n_tok=4096)
    qs = synth.QuantSetting(4, 128, False, 0.01, True)
    X = synth.make_x_bf16(layer)
    W = synth.make_w_fp16(layer)
    Wd = torch.from_numpy(W).to(GH.DEV)
    with G.GPTQContext(layer.n, layer.m, 0) as ctx:
        ctx.accumulate_hessian(GH.bf16_to_dev(X))
        perm = ctx.prepare(qs.damp, qs.desc_act)
        U = ctx.get_factor()
        ref = ctx.quantize_layer(Wd, qs.bits, qs.group_size, qs.sym)
        ctx.synchronize()

    L = G.lib()
    stream = torch.cuda.current_stream(GH.DEV)
    qp = G.QParams(qs.bits, qs.group_size, int(qs.sym))
    for call in range(2):
        out = {"codes": torch.full_like(ref["codes"], -1), "scales": torch.full_like(ref["scales"], float("nan")),
               "zeros": torch.full_like(ref["zeros"], float("nan")), "g_idx": torch.full_like(ref["g_idx"], -1),
               "w_hat": torch.full_like(ref["w_hat"], float("nan"))}
        st = L.gptq_quantize_layer_noalloc(_p(Wd), layer.m, layer.n, _p(U), _p(perm), None, qp, _p(out["codes"]),
                                           _p(out["scales"]), _p(out["zeros"]), _p(out["g_idx"]), _p(out["w_hat"]),
                                           GH.DEV.index, ctypes.c_void_p(stream.cuda_stream))
        assert st == G.OK, (call, G.STATUS.get(st))
        torch.cuda.synchronize(GH.DEV)
        same = (out["codes"] == ref["codes"]).float().mean().item()
        assert same >= GH.CODES_IDENTICAL, (call, same)
        sc_ref = ref["scales"].double()
        rel = ((out["scales"].double() - sc_ref).abs() / sc_ref.abs()).max().item()
        assert rel <= GH.SZ_REL, (call, rel)
        assert torch.equal(out["zeros"], ref["zeros"]), call
        assert torch.equal(out["g_idx"], ref["g_idx"]), call
        assert torch.allclose(out["w_hat"], ref["w_hat"], rtol=1e-6, atol=1e-9), call
