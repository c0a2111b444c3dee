"""AWQ channel scaling plus round-to-nearest on the GPU (gptq_awq_quantize, through the C ABI)
against the oracle's awq_quantize.  Both sides take every decision in the same arithmetic:
the channel sums are exact in fp64, the median and the mask compare the same fp64 values,
W' = fp32(W) * scale and the group parameters and codes use IEEE fp32 operations with
round-half-to-even; so the channel scales, codes, scales and zeros must be identical, and
the dequantized weights agree to fp32 rounding (1e-6 relative)."""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import gptq as G
from post_weight_quantization_16_b200 import synth
from tests import gpu_helpers as GH

pytestmark = pytest.mark.gpu
TINY = synth.WORKLOADS["tiny_256x512"][0]

CASES = [
    # m, n, n_tok, bits, g, sym, s
    (96, 512, 2048, 4, 128, False, 2.0),
    (64, 1152, 1000, 3, 64, True, 2.0),
    (40, 256, 500, 2, 32, False, 1.5),
    (64, 512, 777, 4, 128, False, 1.0),
    (33, 384, 64, 8, -1, True, 2.0),
    (32, 512, 0, 4, 128, False, 2.0),
]


def _check(layer, X_bits, bits, g, sym, s):
    W = synth.make_w_fp16(layer)
    Xd = GH.bf16_to_dev(X_bits) if X_bits.shape[0] else None
    out = G.awq_quantize(Xd, torch.from_numpy(W).to(GH.DEV), s, bits, g, sym)
    torch.cuda.synchronize(GH.DEV)
    X = synth.bf16_bits_to_f32(X_bits) if X_bits.shape[0] else np.zeros((1, layer.n))
    ref = O.awq_quantize(W.astype(np.float64), X, s, bits, g, sym)
    if X_bits.shape[0] == 0:
        ref = O.awq_quantize(W.astype(np.float64), np.zeros((1, layer.n)), s, bits, g, sym)
    assert np.array_equal(out["channel_scale"].cpu().numpy(), ref["channel_scale"])
    assert np.array_equal(out["codes"].cpu().numpy().view(np.uint32), ref["packed"])
    assert np.array_equal(out["scales"].cpu().numpy(), ref["scales"])
    assert np.array_equal(out["zeros"].cpu().numpy(), ref["zeros"])
    what = out["w_hat"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(what - ref["what"]) <= 1e-6 * np.abs(ref["what"]) + 1e-12)
    return ref


@pytest.mark.parametrize("m,n,n_tok,bits,g,sym,s", CASES)
def test_awq_matches_oracle(m, n, n_tok, bits, g, sym, s):
    layer = synth.scaled_layer(TINY, m=m, n=n, n_tok=max(n_tok, 1))
    X = synth.make_x_bf16(layer)[:n_tok]
    ref = _check(layer, X, bits, g, sym, s)
    if n_tok:
        # an even count: exactly half of the channels are protected (no ties in these draws)
        assert (ref["channel_scale"] != 1.0).sum() == (n // 2 if s != 1.0 else 0)


@pytest.mark.slow
def test_awq_q_proj_shape():
    """4096 x 4096 with 16384 calibration tokens of the q_proj recipe (0.5 % outlier channels x30)."""
    layer, _ = synth.WORKLOADS["q_proj_4096x4096"]
    X = synth.make_x_bf16(layer, 0, 16384)
    _check(layer, X, 4, 128, False, 2.0)
