"""Unit checks of individual CUDA kernels through the C ABI test hooks (include/gptq_testing.h)."""
import ctypes

import numpy as np
import pytest
import torch

from post_weight_quantization_16_b200 import gptq as G

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def tf32_rn(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0xFFF + ((u >> 13) & 1)) & 0xFFFFE000
    return u.astype(np.uint32).view(np.float32)


def split(x):
    x = np.asarray(x, dtype=np.float32)
    hi = tf32_rn(x)
    lo = tf32_rn(x - hi)
    return hi, lo


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def run_gemm(A, B, alpha=1.0, beta=0, C0=None, klo=0, khi=0, upper=0, plain=True, hilo=False, trans=False, chunk=1,
             tile=0, reduce=0):
    M, K = A.shape
    N = B.shape[0]
    ah, al = split(A)
    bh, bl = split(B)
    Ah, Al, Bh, Bl = dev(ah), dev(al), dev(bh), dev(bl)
    C = dev(C0 if C0 is not None else np.zeros((M, N))) if plain else None
    if hilo:
        c0 = C0 if C0 is not None else np.zeros((M, N))
        h0, l0 = split(c0)
        Ch, Cl = dev(h0), dev(l0)
    else:
        Ch = Cl = None
    Cth = torch.zeros((N, M), dtype=torch.float32, device=DEV) if trans else None
    Ctl = torch.zeros((N, M), dtype=torch.float32, device=DEV) if trans else None
    st = G.lib().gptq_test_gemm_tf32x3(M, N, K, p(Ah), p(Al), K, p(Bh), p(Bl), K, float(alpha), int(beta), klo, khi,
                                       upper, p(C), N, p(Ch), p(Cl), N, p(Cth), p(Ctl), M, chunk, tile, reduce, 0,
                                       ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream))
    assert st == G.OK, G.STATUS.get(st)
    out = {}
    if plain:
        out["C"] = C.cpu().numpy().astype(np.float64)
    if hilo:
        out["Chilo"] = Ch.cpu().numpy().astype(np.float64) + Cl.cpu().numpy().astype(np.float64)
    if trans:
        out["Ct"] = Cth.cpu().numpy().astype(np.float64) + Ctl.cpu().numpy().astype(np.float64)
    return out


def ref(A, B, alpha, beta, C0):
    R = alpha * (np.asarray(A, np.float64) @ np.asarray(B, np.float64).T)
    if beta:
        R += np.asarray(C0, np.float64)
    scale = np.abs(alpha) * (np.abs(A).astype(np.float64) @ np.abs(B).astype(np.float64).T) + (np.abs(C0) if beta else 0)
    return R, scale


@pytest.mark.parametrize("M,N,K,chunk", [(128, 256, 32, 1), (200, 320, 96, 1), (64, 64, 128, 4), (384, 512, 2048, 1),
                                         (4096, 768, 128, 4), (300, 1024, 256, 2)])
@pytest.mark.parametrize("beta", [0, 1])
@pytest.mark.parametrize("tile", [0, 64, 128, 256, 512])
def test_gemm_outputs_match_fp64(M, N, K, chunk, beta, tile):
    r = np.random.default_rng(M + N + K + beta)
    A = r.standard_normal((M, K)).astype(np.float32)
    B = r.standard_normal((N, K)).astype(np.float32)
    C0 = r.standard_normal((M, N)).astype(np.float32)
    out = run_gemm(A, B, alpha=-0.75, beta=beta, C0=C0, plain=True, hilo=True, trans=(beta == 0), chunk=chunk,
                   tile=tile)
    R, scale = ref(A, B, -0.75, beta, C0)
    for k in out:
        got = out[k].T if k == "Ct" else out[k]
        err = np.abs(got - R) / scale
        assert err.max() <= 2e-6, (k, err.max())


@pytest.mark.parametrize("tile", [64, 128, 256, 512])
def test_gemm_triangular_k_ranges(tile):
    r = np.random.default_rng(7)
    n = 512
    # B lower in K-major form (B[c][k] = 0 for k < c): K from the tile's first column
    A = r.standard_normal((256, n)).astype(np.float32)
    B = np.triu(r.standard_normal((n, n)).astype(np.float32))
    R, scale = ref(A, B, 1.0, 0, None)
    got = run_gemm(A, B, klo=1, tile=tile)["C"]
    assert (np.abs(got - R) / scale).max() <= 2e-6
    # B upper in K-major form (B[c][k] = 0 for k > c): K up to the tile's last column
    B2 = np.tril(r.standard_normal((n, n)).astype(np.float32))
    R, scale = ref(A, B2, 1.0, 0, None)
    got = run_gemm(A, B2, khi=1, tile=tile)["C"]
    assert (np.abs(got - R) / scale).max() <= 2e-6
    # A upper (A[r][k] = 0 for k < r): K from the tile's first row
    A3 = np.triu(r.standard_normal((n, n)).astype(np.float32))
    B3 = r.standard_normal((384, n)).astype(np.float32)
    R, scale = ref(A3, B3, 1.0, 0, None)
    got = run_gemm(A3, B3, klo=2, tile=tile)["C"]
    assert (np.abs(got - R) / scale).max() <= 2e-6


@pytest.mark.parametrize("kblk,tile", [(128, 64), (128, 128), (256, 128), (256, 256), (512, 256), (1024, 0)])
def test_gemm_block_diagonal_k_ranges(kblk, tile):
    """k_lo_mode 3 + log2(kblk / 128): K over the output column's aligned kblk block only, cut at
    the tile's last column (B block-diagonal with upper-triangular blocks): the rows above each
    block equal the fp64 product with that masked B, in the plain and the transposed output."""
    r = np.random.default_rng(kblk + tile)
    n = 1536
    A = r.standard_normal((n, n)).astype(np.float32)
    B = r.standard_normal((n, n)).astype(np.float32)
    col = np.arange(n)[:, None]
    k = np.arange(n)[None, :]
    Bm = np.where((k // kblk == col // kblk) & (k <= col), B, np.float32(0))
    mode = 3 + int(np.log2(kblk // 128))
    out = run_gemm(A, Bm, klo=mode, khi=1, upper=1, plain=True, trans=True, tile=tile)
    R, scale = ref(A, Bm, 1.0, 0, None)
    rows_above = np.arange(n)[:, None] < (np.arange(n)[None, :] // kblk) * kblk
    for key in ("C", "Ct"):
        got = out[key].T if key == "Ct" else out[key]
        err = np.abs(got - R) / (scale + 1e-30)
        assert err[rows_above].max() <= 2e-6, (key, err[rows_above].max())


def test_gemm_block_diagonal_rejects_wide_tiles():
    A = np.ones((256, 256), np.float32)
    Ah, Al = dev(A), dev(np.zeros_like(A))
    st = G.lib().gptq_test_gemm_tf32x3(256, 256, 256, p(Ah), p(Al), 256, p(Ah), p(Al), 256, 1.0, 0, 3, 1, 1, p(Ah), 256,
                                       None, None, 256, None, None, 256, 1, 256, 0, 0,
                                       ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream))
    assert st == G.ERR_ARG


@pytest.mark.parametrize("tile", [64, 128, 256, 512])
def test_gemm_upper_only_updates_upper_triangle(tile):
    r = np.random.default_rng(9)
    n, K = 640, 128
    V = r.standard_normal((n, K)).astype(np.float32)
    C0 = r.standard_normal((n, n)).astype(np.float32)
    out = run_gemm(V, V, alpha=-1.0, beta=1, C0=C0, upper=1, plain=False, hilo=True, tile=tile)
    R, scale = ref(V, V, -1.0, 1, C0)
    iu = np.triu_indices(n)
    err = np.abs(out["Chilo"][iu] - R[iu]) / scale[iu]
    assert err.max() <= 2e-6


@pytest.mark.parametrize("M,N,K,chunk", [(4096, 896, 128, 4), (300, 320, 1024, 4), (128, 64, 32, 1), (1000, 3072, 256, 4)])
@pytest.mark.parametrize("tile", [64, 128, 256, 512])
def test_gemm_reduce_add_epilogue(M, N, K, chunk, tile):
    """C += alpha A B^T through TMA reduce-add boxes: equals the fp64 result, and C's columns
    right of the product (inside the same allocation) are untouched."""
    r = np.random.default_rng(M + N + K + tile)
    A = r.standard_normal((M, K)).astype(np.float32)
    B = r.standard_normal((N, K)).astype(np.float32)
    pad = 96  # C lives in a wider matrix: the product covers its first N columns
    C0 = r.standard_normal((M, N + pad)).astype(np.float32)
    ah, al = split(A)
    bh, bl = split(B)
    Ah, Al, Bh, Bl = dev(ah), dev(al), dev(bh), dev(bl)
    C = dev(C0)
    st = G.lib().gptq_test_gemm_tf32x3(M, N, K, p(Ah), p(Al), K, p(Bh), p(Bl), K, -1.0, 1, 0, 0, 0, p(C), N + pad,
                                       None, None, 0, None, None, 0, chunk, tile, 1, 0,
                                       ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream))
    assert st == G.OK, G.STATUS.get(st)
    got = C.cpu().numpy().astype(np.float64)
    R, scale = ref(A, B, -1.0, 1, C0[:, :N])
    assert (np.abs(got[:, :N] - R) / scale).max() <= 2e-6
    assert np.array_equal(got[:, N:], C0[:, N:].astype(np.float64))


def test_sweep_division_equals_ieee_division():
    """The sweep's reciprocal-plus-correction quotient is the correctly rounded x / s,
    bit for bit, on 2^30 pairs: random operands and quotients next to code boundaries."""
    mism = ctypes.c_uint64(0)
    ex = (ctypes.c_float * 2)()
    st = G.lib().gptq_test_div_rn(12345, 1 << 30, ctypes.byref(mism), ex, 0, None)
    assert st == 0, G.lib().gptq_status_string(st).decode()
    assert mism.value == 0, f"{mism.value} differing quotients, e.g. x={ex[0]!r} s={ex[1]!r}"
