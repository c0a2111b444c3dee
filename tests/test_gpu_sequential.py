"""Sequential (cross-layer) quantization on the GPU ("GPTQ算法原理深度解析" §2.1: a layer's
quantization error reaches the next layer through its input): a three-layer ReLU stack where
each layer is calibrated on the outputs of the already-quantized layers before it.  Checked
stage by stage against the oracle: each layer's Hessian against 2 X^T X of the GPU's own
calibration inputs, its sweep replayed by the oracle on that Hessian, and the next layer's inputs
against ReLU of the oracle's product with the GPU's fp16-dequantized weights (tolerance: the
product's fp32 accumulation, as in the consumer's own tests, plus half a unit of the output
format's last place)."""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import gptq as G
from post_weight_quantization_16_b200 import synth
from tests import gpu_helpers as GH

pytestmark = pytest.mark.gpu


def _bits_to_f64(t, bf16):
    a = t.cpu().view(torch.int16).numpy().view(np.uint16) if bf16 else t.cpu().numpy()
    return (synth.bf16_bits_to_f32(a) if bf16 else a.astype(np.float32)).astype(np.float64)


def test_activation_convert_rounds_to_nearest():
    rng = np.random.default_rng(3)
    y = rng.normal(0, 3, 10007).astype(np.float32)
    y[:4] = [0.0, -0.0, 1e-30, -5.0]
    Y = torch.from_numpy(y).to(GH.DEV)
    xb, xh = G.activation_convert(Y, act=1)
    torch.cuda.synchronize(GH.DEV)
    relu = np.where(y > 0, y, np.float32(0))
    assert np.array_equal(xb.cpu().view(torch.int16).numpy().view(np.uint16), synth.f32_to_bf16_bits(relu))
    assert np.array_equal(xh.cpu().numpy(), relu.astype(np.float16))
    xb2, _ = G.activation_convert(Y, act=0, want_fp16=False)
    assert np.array_equal(xb2.cpu().view(torch.int16).numpy().view(np.uint16), synth.f32_to_bf16_bits(y))


def test_three_layer_relu_stack_stage_by_stage():
    N = 2048
    dims = [256, 512, 384, 256]
    lay0 = synth.scaled_layer(synth.WORKLOADS["tiny_256x512"][0], m=dims[1], n=dims[0], n_tok=N)
    X0 = GH.bf16_to_dev(synth.make_x_bf16(lay0))
    rng = np.random.default_rng(11)
    Ws = [(rng.standard_normal((dims[i + 1], dims[i])) * (1.0 / np.sqrt(dims[i]))).astype(np.float16)
          for i in range(3)]
    settings = [synth.QuantSetting(4, 128, False, 0.01, True), synth.QuantSetting(3, 64, True, 0.01, True),
                synth.QuantSetting(4, -1, False, 0.1, False)]
    layers = [dict(W=torch.from_numpy(W).to(GH.DEV), bits=q.bits, group_size=q.group_size, sym=q.sym, damp=q.damp,
                   desc_act=q.desc_act) for W, q in zip(Ws, settings)]
    res = G.quantize_sequential(X0, layers, act=1, keep_hessian=True)
    torch.cuda.synchronize(GH.DEV)
    x0 = synth.bf16_bits_to_f32(X0.cpu().view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(res[0]["X16"].cpu().numpy(), x0.astype(np.float16))
    for li, (W, qs, r) in enumerate(zip(Ws, settings, res)):
        n = dims[li]
        X = _bits_to_f64(r["X"], True)
        H = r["H"].cpu().numpy().astype(np.float64)
        Href = O.hessian(X)
        assert np.linalg.norm(H - Href) / np.linalg.norm(Href) <= GH.H_REL_FRO, li
        prep = O.prepare(H, qs.damp, qs.desc_act)
        assert np.array_equal(r["perm"].cpu().numpy(), prep["perm"]), li
        packed = r["codes"].cpu().numpy().view(np.uint32)
        gpu = {"codes": O.unpack_codes(packed, n, qs.bits), "scales": r["scales"].cpu().numpy(),
               "zeros": r["zeros"].cpu().numpy()}
        st, rep = GH.check_sweep_replay(W, prep, gpu, qs)
        GH.assert_replay_ok(st, rep, gpu)
        if li + 1 < len(res):
            X16 = _bits_to_f64(r["X16"], False)
            Y = O.dequant_matmul_fp16(X16.astype(np.float16), packed, gpu["scales"], gpu["zeros"], prep["perm"], n,
                                      qs.bits, qs.group_size)
            W16 = O.dequantize_packed_fp16(packed, gpu["scales"], gpu["zeros"], prep["perm"], n, qs.bits,
                                           qs.group_size)
            tol = (n / 16 + 8) * 2.0 ** -22 * (np.abs(X16) @ np.abs(W16.astype(np.float64)).T) + 1e-30
            relu = np.maximum(Y, 0.0)
            nxt_b = _bits_to_f64(res[li + 1]["X"], True)
            nxt_h = _bits_to_f64(res[li + 1]["X16"], False)
            assert np.all(np.abs(nxt_b - relu) <= tol + 2.0 ** -8 * np.abs(relu) + 1e-30), li
            assert np.all(np.abs(nxt_h - relu) <= tol + 2.0 ** -11 * np.abs(relu) + 2.0 ** -24), li
            assert (nxt_b >= 0).all() and (nxt_h >= 0).all()


def test_contexts_kept_between_calls_give_the_same_result():
    """quantize_sequential with a contexts dict: the first call creates the width-256 context, the
    third layer (384 rows) replaces it with a larger one, and a second call reuses it; every output
    equals the call that creates and closes its own contexts."""
    N = 1024
    dims = [256, 256, 256, 384]
    lay0 = synth.scaled_layer(synth.WORKLOADS["tiny_256x512"][0], m=dims[1], n=dims[0], n_tok=N)
    X0 = GH.bf16_to_dev(synth.make_x_bf16(lay0))
    rng = np.random.default_rng(12)
    layers = [dict(W=torch.from_numpy((rng.standard_normal((dims[i + 1], dims[i])) / 16).astype(np.float16)).to(GH.DEV),
                   bits=4, group_size=128, sym=bool(i % 2), damp=0.01, desc_act=True) for i in range(3)]
    ref = G.quantize_sequential(X0, layers, act=1)
    torch.cuda.synchronize(GH.DEV)
    ctxs = {}
    try:
        for _ in range(2):
            res = G.quantize_sequential(X0, layers, act=1, contexts=ctxs)
            torch.cuda.synchronize(GH.DEV)
            assert len(ctxs) == 1 and next(iter(ctxs.values())).m_max == 384
            for a, b in zip(ref, res):
                for key in ("codes", "scales", "zeros", "perm", "g_idx"):
                    assert torch.equal(a[key], b[key]), key
    finally:
        G.close_contexts(ctxs)
    assert not ctxs
