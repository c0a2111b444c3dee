"""gptq_quantize_layer_noalloc — the quantize entry point for callers that cannot allocate
device memory themselves: an engine or plugin host that hands out every byte of a fixed
device-memory budget, or code where cudaMalloc/cudaFree (which synchronize the whole device)
are not allowed.  Its scratch is a fixed array inside the library.

These tests call it through the C ABI on two calls in a row and check each call the way the
context path is checked: the oracle replays the sweep on the same factor (stage-isolated, the
oracle's U from the GPU's H) and the codes, scales and zeros must pass the replay; the outputs
must also agree with the context-based gptq_quantize_layer.  Requests beyond the array's size
are refused.  A layer with unexcited columns gets its `dead` mask from gptq_get_dead_columns.

The file name sorts last so that a run that stops at the first failure has already run every
other test."""
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


NOALLOC_CASES = [
    # bits, group, sym, want W_hat, dead columns
    (4, 128, False, True, False),
    (3, 64, False, True, False),
    (2, 32, True, True, False),
    (4, -1, False, False, False),
    (4, 128, False, True, True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("bits,g,sym,want_what,with_dead", NOALLOC_CASES)
def test_noalloc_matches_oracle_and_context_path_on_two_calls(bits, g, sym, want_what, with_dead):
    from oracle import gptq_oracle as O
    from tests import gpu_helpers as GH

    layer = synth.scaled_layer(synth.WORKLOADS["tiny_256x512"][0], m=200, n=1024, n_tok=4096)
    qs = synth.QuantSetting(bits, g, sym, 0.01, True)
    X = synth.make_x_bf16(layer)
    if with_dead:
        X[:, [3, 500, 1000]] = 0
    W = synth.make_w_fp16(layer)
    Wd = torch.from_numpy(W).to(GH.DEV)
    with G.GPTQContext(layer.n, layer.m, 0) as ctx:
        ctx.accumulate_hessian(GH.bf16_to_dev(X))
        H, _ = ctx.get_hessian()
        perm = ctx.prepare(qs.damp, qs.desc_act)
        U = ctx.get_factor()
        dead = ctx.get_dead_columns() if with_dead else None
        ref = ctx.quantize_layer(Wd, qs.bits, qs.group_size, qs.sym)
        ctx.synchronize()
    prep = O.prepare(H.cpu().numpy().astype(np.float64), qs.damp, qs.desc_act)
    assert np.array_equal(perm.cpu().numpy(), prep["perm"])
    if with_dead:
        assert np.array_equal(dead.cpu().numpy().astype(bool), prep["dead"])
        assert prep["dead"][[3, 500, 1000]].all()

    L = G.lib()
    stream = torch.cuda.current_stream(GH.DEV)
    qp = G.QParams(qs.bits, qs.group_size, int(qs.sym))
    for call in range(2):
        out = {"codes": torch.full_like(ref["codes"], -1), "scales": torch.full_like(ref["scales"], float("nan")),
               "zeros": torch.full_like(ref["zeros"], float("nan")), "g_idx": torch.full_like(ref["g_idx"], -1),
               "w_hat": torch.full_like(ref["w_hat"], float("nan")) if want_what else None}
        st = L.gptq_quantize_layer_noalloc(_p(Wd), layer.m, layer.n, _p(U), _p(perm), _p(dead), qp,
                                           _p(out["codes"]), _p(out["scales"]), _p(out["zeros"]), _p(out["g_idx"]),
                                           _p(out["w_hat"]), GH.DEV.index, ctypes.c_void_p(stream.cuda_stream))
        assert st == G.OK, (call, G.STATUS.get(st))
        torch.cuda.synchronize(GH.DEV)
        gpu = {"codes": O.unpack_codes(out["codes"].cpu().numpy().view(np.uint32), layer.n, qs.bits),
               "scales": out["scales"].cpu().numpy(), "zeros": out["zeros"].cpu().numpy()}
        # the oracle's replay of the sweep on the same inputs
        rs, rep = GH.check_sweep_replay(W, prep, gpu, qs)
        GH.assert_replay_ok(rs, rep, gpu)
        assert np.array_equal(out["g_idx"].cpu().numpy(), O.g_idx(prep["perm"], qs.group_size)), call
        # and the context path's outputs (codes compared one by one, not as packed words)
        ref_codes = O.unpack_codes(ref["codes"].cpu().numpy().view(np.uint32), layer.n, qs.bits)
        same = float(np.mean(gpu["codes"] == ref_codes))
        assert same >= GH.CODES_IDENTICAL, (call, same)
        assert torch.equal(out["zeros"], ref["zeros"]), call
        if want_what:
            # the dequantized weights are (code - zero) * scale of this call's own outputs, taken in
            # fp32 and stored in the original column order (the scales themselves were checked
            # against the oracle's replay above; the context path, which accumulates the
            # propagated errors in another order, may differ from this one by a scale tolerance
            # on each side, so its weights are not the yardstick here)
            what = out["w_hat"].cpu().numpy()
            gw = qs.group_size if qs.group_size > 0 else layer.n
            grp = np.arange(layer.n) // gw
            expect = np.empty_like(what)
            expect[:, prep["perm"]] = ((gpu["codes"].astype(np.float32) - gpu["zeros"][:, grp].astype(np.float32))
                                       * gpu["scales"][:, grp].astype(np.float32))
            assert np.array_equal(what, expect), call
            if with_dead:
                assert not what[:, [3, 500, 1000]].any()
