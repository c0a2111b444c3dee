"""Round-to-nearest with a clipped range on the GPU (gptq_rtn_quantize, through the C ABI)
against the oracle's rtn with the same clip ratio ("模型量化实战…" §3.1 LinearQuantizer,
clip_ratio).  Both sides take every decision in the same arithmetic: the percentile's position
and weight in fp32 as numpy computes them, the order statistics exactly (they are values of the
group), the interpolation and the group parameters and codes in IEEE fp32 operations with
round-half-to-even; so codes, scales and zeros must be identical, and the dequantized weights
agree to fp32 rounding (1e-6 relative)."""
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
    # m, n, bits, g, sym, clip      (groups per row >= 8: one warp per group; fewer: the whole CTA)
    (64, 1024, 4, 128, False, 0.99),
    (64, 1024, 4, 128, True, 0.99),
    (48, 512, 8, -1, True, 0.99),        # the page's INT8 per-channel symmetric quantizer
    (48, 512, 8, -1, False, 0.99),
    (40, 2048, 3, 64, False, 0.9),
    (33, 384, 2, 32, True, 0.5),
    (32, 768, 4, 256, False, 0.95),      # 3 groups: CTA-wide selection
    (32, 512, 4, 128, True, 1.0),        # no clipping: the min-max quantizer
    (16, 4096, 8, -1, False, 0.999),
]


def _w(m, n, seed):
    """The tiny recipe's weights with a few large entries per row, so clipping matters."""
    layer = synth.scaled_layer(TINY, m=m, n=n, n_tok=1)
    W = synth.make_w_fp16(layer).astype(np.float32)
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, n, (m, max(1, n // 200)))
    np.put_along_axis(W, idx, rng.choice([-1.0, 1.0], idx.shape) * 0.3, axis=1)
    return W.astype(np.float16)


def _check(W, bits, g, sym, clip, scale=None):
    Wd = torch.from_numpy(W).to(GH.DEV)
    sd = None if scale is None else torch.from_numpy(scale).to(GH.DEV)
    out = G.rtn_quantize(Wd, bits, g, sym, clip, channel_scale=sd)
    torch.cuda.synchronize(GH.DEV)
    Ws = W.astype(np.float32) if scale is None else W.astype(np.float32) * scale[None, :]
    ref = O.rtn(Ws.astype(np.float64), bits, g, sym, clip)
    what_ref = ref["what"] if scale is None else ref["what"] / scale[None, :].astype(np.float64)
    assert np.array_equal(out["codes"].cpu().numpy().view(np.uint32), O.pack_codes(ref["codes"], bits))
    assert np.array_equal(out["scales"].cpu().numpy(), ref["scales"])
    assert np.array_equal(out["zeros"].cpu().numpy(), ref["zeros"])
    what = out["w_hat"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(what - what_ref) <= 1e-6 * np.abs(what_ref) + 1e-12)
    return ref


@pytest.mark.parametrize("m,n,bits,g,sym,clip", CASES)
def test_clipped_rtn_matches_oracle(m, n, bits, g, sym, clip):
    W = _w(m, n, 7 + m)
    ref = _check(W, bits, g, sym, clip)
    if clip < 1.0:
        mm = O.rtn(W.astype(np.float64), bits, g, sym)
        assert np.all(ref["scales"] <= mm["scales"])          # the clipped range lies inside the min-max one


def test_clipped_rtn_on_awq_scaled_weights():
    """The AWQ scales of gptq_awq_quantize passed on: W' = W * scale, W_hat = dequantized / scale."""
    m, n = 64, 1024
    layer = synth.scaled_layer(TINY, m=m, n=n, n_tok=512)
    X = synth.make_x_bf16(layer)
    W = _w(m, n, 3)
    awq = G.awq_quantize(GH.bf16_to_dev(X), torch.from_numpy(W).to(GH.DEV), 2.0, 4, 128, False, want_w_hat=False)
    torch.cuda.synchronize(GH.DEV)
    scale = awq["channel_scale"].cpu().numpy()
    assert (scale == 2.0).sum() == n // 2
    _check(W, 4, 128, False, 0.99, scale)


def test_clipped_rtn_ties_and_zero_rows():
    """Rows of repeated values, all-zero rows and rows of signed zeros: the order statistics are
    ties, and the scale falls to its 1e-8 floor."""
    m, n = 24, 512
    rng = np.random.default_rng(9)
    W = np.round(rng.normal(0, 2, (m, n))).astype(np.float16)
    W[3] = 0
    W[4] = np.float16(-0.0)
    W[5, ::2] = np.float16(-0.0)
    W[6] = 1.5
    for sym in (False, True):
        _check(W, 4, 128, sym, 0.9)
        _check(W, 8, -1, sym, 0.99)


@pytest.mark.slow
def test_clipped_rtn_q_proj_shape():
    """The page's INT8 quantizer (8 bits, per-channel, symmetric, clip 0.99) on a 4096 x 4096 layer,
    and 4-bit groups of 128 with asymmetric clipping."""
    layer, _ = synth.WORKLOADS["q_proj_4096x4096"]
    W = synth.make_w_fp16(layer)
    _check(W, 8, -1, True, 0.99)
    _check(W, 4, 128, False, 0.99)
