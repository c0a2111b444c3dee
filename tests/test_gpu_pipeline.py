"""gptq_quantize_layers: many layers in one pipelined call.  Every job's outputs must equal,
bit for bit, those of the same layer quantized alone through the context calls (the same
kernels on the same inputs; only the overlap between layers changes), and one shared-input
job is replayed by the oracle."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import gptq as G
from post_weight_quantization_16_b200 import synth
from tests import gpu_helpers as GH

TINY = synth.WORKLOADS["tiny_256x512"][0]


def test_pipeline_rejects_bad_jobs():
    L = G.lib()
    assert L.gptq_quantize_layers(None, 0, 0, None) == G.ERR_ARG
    jobs = (G.LayerJob * 1)()
    jobs[0].m, jobs[0].n = 4, 100          # n % 128
    assert L.gptq_quantize_layers(jobs, 1, 0, None) == G.ERR_ARG


def _alone(X, W, bits, g, sym, damp, desc_act):
    with G.GPTQContext(W.shape[1], W.shape[0], 0) as ctx:
        ctx.accumulate_hessian(X)
        perm = ctx.prepare(damp, desc_act)
        out = ctx.quantize_layer(W, bits, g, sym)
        ctx.synchronize()
        H, _ = ctx.get_hessian()
    return {k: v.cpu().numpy() for k, v in dict(out, perm=perm).items() if v is not None}, H.cpu().numpy()


@pytest.mark.gpu
def test_pipeline_equals_layers_quantized_alone():
    lay_a = synth.scaled_layer(TINY, m=96, n=512, n_tok=1500, name="a")
    lay_b = synth.scaled_layer(TINY, m=64, n=512, n_tok=900, name="b")
    lay_c = synth.scaled_layer(TINY, m=80, n=1152, n_tok=2000, name="c")
    import dataclasses
    lay_b = dataclasses.replace(lay_b, x_seed=5, w_seed=6)
    lay_c = dataclasses.replace(lay_c, x_seed=7, w_seed=8)
    Xa, Xb, Xc = (GH.bf16_to_dev(synth.make_x_bf16(l)) for l in (lay_a, lay_b, lay_c))
    Wa = torch.from_numpy(synth.make_w_fp16(lay_a)).to(GH.DEV)
    Wa2 = torch.from_numpy(synth.make_w_fp16(dataclasses.replace(lay_a, w_seed=11))).to(GH.DEV)
    Wb = torch.from_numpy(synth.make_w_fp16(lay_b)).to(GH.DEV)
    Wc = torch.from_numpy(synth.make_w_fp16(lay_c)).to(GH.DEV)
    layers = [
        dict(X=Xa, W=Wa, bits=4, group_size=128, sym=False, damp=0.01, desc_act=True, want_w_hat=True),
        dict(X=Xb, W=Wb, bits=3, group_size=64, sym=True, damp=0.1, desc_act=True),
        dict(X=Xa, W=Wa2, bits=2, group_size=-1, sym=False, damp=0.1, desc_act=True),   # shares X with job 0
        dict(X=Xc, W=Wc, bits=4, group_size=128, sym=False, damp=0.01, desc_act=False),
        dict(X=Xa, W=Wa, bits=8, group_size=128, sym=True, damp=0.01, desc_act=True),    # shares X and damp
    ]
    outs = G.quantize_layers(layers)
    torch.cuda.synchronize(GH.DEV)
    for L, o in zip(layers, outs):
        ref, H = _alone(L["X"], L["W"], L["bits"], L["group_size"], L["sym"], L["damp"], L["desc_act"])
        for k in ("codes", "scales", "zeros", "g_idx", "perm"):
            assert np.array_equal(o[k].cpu().numpy(), ref[k]), k
    # the oracle's replay of the shared-input job 2 (on the GPU's H)
    ref, H = _alone(Xa, Wa2, 2, -1, False, 0.1, True)
    prep = O.prepare(H.astype(np.float64), 0.1, True)
    gpu = {"codes": O.unpack_codes(outs[2]["codes"].cpu().numpy().view(np.uint32), 512, 2),
           "scales": outs[2]["scales"].cpu().numpy(), "zeros": outs[2]["zeros"].cpu().numpy()}
    st, rep = GH.check_sweep_replay(Wa2.cpu().numpy(), prep, gpu, synth.QuantSetting(2, -1, False, 0.1, True))
    GH.assert_replay_ok(st, rep, gpu)


@pytest.mark.gpu
def test_pipeline_handle_reused_for_two_batches():
    """One pipeline, two batches of different layers: each job equals the layer quantized alone."""
    import dataclasses
    lays = [dataclasses.replace(synth.scaled_layer(TINY, m=64, n=512, n_tok=1024, name=f"p{i}"), x_seed=20 + i,
                                w_seed=40 + i) for i in range(3)]
    Xs = [GH.bf16_to_dev(synth.make_x_bf16(l)) for l in lays]
    Ws = [torch.from_numpy(synth.make_w_fp16(l)).to(GH.DEV) for l in lays]
    with G.Pipeline({512: 64}) as pipe:
        for batch in ([0, 1], [2, 0]):
            layers = [dict(X=Xs[i], W=Ws[i], bits=4, group_size=128, sym=False, damp=0.01, desc_act=True)
                      for i in batch]
            outs = pipe.run(layers)
            torch.cuda.synchronize(GH.DEV)
            for i, o in zip(batch, outs):
                ref, _ = _alone(Xs[i], Ws[i], 4, 128, False, 0.01, True)
                for k in ("codes", "scales", "zeros", "g_idx", "perm"):
                    assert np.array_equal(o[k].cpu().numpy(), ref[k]), (batch, i, k)
        # a job wider than the pipeline's contexts is refused
        with pytest.raises(G.GPTQError) as ei:
            pipe.run([dict(X=Xs[0], W=torch.zeros((65, 512), dtype=torch.float16, device=GH.DEV), bits=4,
                           group_size=128, sym=False, damp=0.01, desc_act=True)])
        assert ei.value.status == G.ERR_ARG
