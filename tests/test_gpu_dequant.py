"""The packed result's consumer on the GPU: Y = X W16^T from codes, scales, zeros and perm
(gptq_dequant_matmul, through the C ABI), against the oracle's dequant_matmul_fp16.

Tolerance: the fp16 weights are formed identically on both sides (fp32 product, then round to
nearest fp16), every fp16 x fp16 product is exact in fp32, and the kernel accumulates in fp32:
one rounding per 16-wide MMA step plus the split-K additions.  So element by element
|Y - Y_oracle| <= (n/16 + 8) * 2^-22 * sum_k |X[t][perm[k]] W16[r][k]|."""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import gptq as G
from post_weight_quantization_16_b200 import synth
from tests import gpu_helpers as GH

pytestmark = pytest.mark.gpu


def _tol(X16, W16, n):
    a = np.abs(X16.astype(np.float64)) @ np.abs(W16.astype(np.float64)).T
    return (n / 16 + 8) * 2.0 ** -22 * a + 1e-30


def _random_layer(rng, m, n, bits, g):
    gw = n if g == -1 else g
    codes = rng.integers(0, 1 << bits, (m, n))
    s = rng.uniform(1e-3, 0.02, (m, n // gw)).astype(np.float32)
    z = rng.integers(0, 1 << bits, (m, n // gw)).astype(np.float32)
    return O.pack_codes(codes, bits), s, z


def _run(X16, packed, s, z, perm, bits, g):
    dev = GH.DEV
    Xd = torch.from_numpy(X16).to(dev)
    cd = torch.from_numpy(packed.view(np.int32)).to(dev)
    sd, zd = torch.from_numpy(s).to(dev), torch.from_numpy(z).to(dev)
    pd = None if perm is None else torch.from_numpy(np.asarray(perm, dtype=np.int32)).to(dev)
    Y = G.dequant_matmul(Xd, cd, sd, zd, pd, bits, g)
    torch.cuda.synchronize(dev)
    return Y.cpu().numpy().astype(np.float64)


CASES = [
    # T, m, n, bits, g, act_order
    (1, 128, 512, 4, 128, True),
    (5, 200, 1152, 4, 128, True),
    (16, 256, 1024, 4, 64, False),
    (33, 64, 512, 3, 32, True),
    (100, 384, 768, 2, 128, True),
    (300, 256, 512, 8, -1, True),
    (16, 130, 4096, 4, 128, True),
    (256, 512, 1024, 3, 64, False),
]


@pytest.mark.parametrize("T,m,n,bits,g,act", CASES)
def test_dequant_matmul_matches_oracle(T, m, n, bits, g, act):
    rng = np.random.default_rng(T * 1000 + m + n + bits)
    packed, s, z = _random_layer(rng, m, n, bits, g)
    perm = rng.permutation(n) if act else None
    X16 = rng.normal(0, 1, (T, n)).astype(np.float16)
    Y = _run(X16, packed, s, z, perm, bits, g)
    Yo = O.dequant_matmul_fp16(X16, packed, s, z, np.arange(n) if perm is None else perm, n, bits, g)
    W16 = O.dequantize_packed_fp16(packed, s, z, np.arange(n) if perm is None else perm, n, bits, g)
    assert np.all(np.abs(Y - Yo) <= _tol(X16, W16, n)), np.max(np.abs(Y - Yo) / _tol(X16, W16, n))


def test_dequant_matmul_after_quantizing_a_layer():
    """The consumer of a layer the path has just quantized (act-order, groups of 128)."""
    layer = synth.scaled_layer(synth.WORKLOADS["tiny_256x512"][0], m=192, n=1024, n_tok=2048)
    qs = synth.QuantSetting(4, 128, False, 0.01, True)
    gpu = GH.run_path(layer, qs)
    rng = np.random.default_rng(7)
    X16 = rng.normal(0, 1, (24, layer.n)).astype(np.float16)
    Y = _run(X16, gpu["packed"], gpu["scales"], gpu["zeros"], gpu["perm"], qs.bits, qs.group_size)
    Yo = O.dequant_matmul_fp16(X16, gpu["packed"], gpu["scales"], gpu["zeros"], gpu["perm"], layer.n, qs.bits,
                               qs.group_size)
    W16 = O.dequantize_packed_fp16(gpu["packed"], gpu["scales"], gpu["zeros"], gpu["perm"], layer.n, qs.bits,
                                   qs.group_size)
    assert np.all(np.abs(Y - Yo) <= _tol(X16, W16, layer.n))
    # and close to the product with the path's own fp32 dequantized weights
    ref = X16.astype(np.float64) @ gpu["w_hat"].T
    assert np.max(np.abs(Y - ref)) <= 1e-2 * np.max(np.abs(ref))


@pytest.mark.slow
@pytest.mark.parametrize("T", [16, 4096])
def test_dequant_matmul_70b_shape_sampled_rows(T):
    """The 70B-shaped down_proj (8192 x 28672, 4-bit, groups of 128, act-order): every output
    computed on the GPU, 48 sampled rows (and at T = 4096, 64 sampled tokens) by the oracle."""
    m, n, bits, g = 8192, 28672, 4, 128
    rng = np.random.default_rng(T)
    packed, s, z = _random_layer(rng, m, n, bits, g)
    perm = rng.permutation(n)
    X16 = rng.normal(0, 1, (T, n)).astype(np.float16)
    Y = _run(X16, packed, s, z, perm, bits, g)
    rows = np.sort(rng.choice(m, 48, replace=False))
    toks = np.arange(T) if T <= 64 else np.sort(rng.choice(T, 64, replace=False))
    Yo = O.dequant_matmul_fp16(X16[toks], packed[rows], s[rows], z[rows], perm, n, bits, g)
    W16 = O.dequantize_packed_fp16(packed[rows], s[rows], z[rows], perm, n, bits, g)
    got = Y[np.ix_(toks, rows)]
    assert np.all(np.abs(got - Yo) <= _tol(X16[toks], W16, n))
    assert np.isfinite(Y).all()


def test_dequant_matmul_rejects_bad_arguments():
    L = G.lib()
    qp = G.QParams(4, 128, 0)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=GH.DEV)
    dummy = torch.empty(4096, dtype=torch.float32, device=GH.DEV)
    p = lambda t: None if t is None else __import__("ctypes").c_void_p(t.data_ptr())
    # n not a multiple of 128
    assert L.gptq_dequant_matmul(p(dummy), 4, p(dummy), p(dummy), p(dummy), None, 8, 100, qp, p(dummy), p(ws),
                                 ws.numel(), 0, None) == G.ERR_ARG
    # workspace too small
    need = L.gptq_dequant_matmul_workspace_bytes(4, 8, 256, 1)
    assert L.gptq_dequant_matmul(p(dummy), 4, p(dummy), p(dummy), p(dummy), p(dummy), 8, 256, qp, p(dummy), p(ws),
                                 need - 256, 0, None) == G.ERR_ARG
