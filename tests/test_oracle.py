"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU).

Each test pins the oracle to something other than its own formulas: a worked example
printed on a page, a closed form, an invariant, a special case that reduces to a
textbook routine, or brute force on tiny inputs.
"""
import itertools

import numpy as np
import pytest
import scipy.linalg

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import synth
from tests.conftest import read_golden


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(a):
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.asarray(a, dtype=np.float32)))


def _spd(n, seed, cond_boost=0.0):
    """A random symmetric positive definite matrix shaped like a calibration Hessian."""
    r = _rng(seed)
    X = _bf16(r.standard_normal((4 * n + 8, n)).astype(np.float32))
    if cond_boost:
        X[:, r.integers(0, n)] *= cond_boost
    H = O.hessian(X)
    return H


# ----------------------------------------------------------------------------------
# quantizer
# ----------------------------------------------------------------------------------
def test_worked_int8_example_codes_and_scale():
    g = read_golden("sym_int8_worked_example.txt")
    bits = int(g["bits"][0])
    w = np.array([float(x) for x in g["w"]], dtype=np.float32)[None, :]
    want = np.array([int(x) for x in g["codes"]])
    r = O.rtn(w.astype(np.float64), bits, -1, True)
    signed = r["codes"][0] - (1 << (bits - 1))
    assert signed.tolist() == want.tolist()
    s_want = np.float32(float(g["scale_numerator"][0])) / np.float32(int(g["scale_denominator"][0]))
    assert r["scales"][0, 0] == s_want
    # the same row through the GPTQ sweep with a diagonal H (no compensation) gives the same codes
    sw = O.gptq_sweep(w.astype(np.float64), np.eye(5), bits, -1, True)
    assert (sw["codes"][0] - 128).tolist() == want.tolist()


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_asym_grid_endpoints_and_roundtrip(bits):
    r = _rng(bits)
    w = r.normal(0, 0.02, size=(64, 128))
    s, z, _ = O.group_params(w, bits, False)
    qmax = (1 << bits) - 1
    w32 = w.astype(np.float32)
    lo = np.minimum(w32.min(1), 0)
    hi = np.maximum(w32.max(1), 0)
    u_lo, _, _ = O.quantize_values(lo, s, z, bits, False)
    u_hi, _, _ = O.quantize_values(hi, s, z, bits, False)
    assert (u_lo == 0).all()
    assert (u_hi == qmax).all()
    assert (z == np.rint(z)).all() and (z >= 0).all() and (z <= qmax).all()
    for j in range(w.shape[1]):
        u, _, wq = O.quantize_values(w[:, j], s, z, bits, False)
        assert (u >= 0).all() and (u <= qmax).all()
        # inside the range the round trip is within half a step (plus float32 slack)
        assert (np.abs(w[:, j] - wq) <= 0.5 * s * (1 + 1e-5) + 1e-12).all()


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_sym_grid(bits):
    r = _rng(10 + bits)
    w = r.normal(0, 0.02, size=(32, 64))
    s, z, _ = O.group_params(w, bits, True)
    assert (z == (1 << (bits - 1))).all()
    amax = np.abs(w.astype(np.float32)).max(1)
    j = np.abs(w.astype(np.float32)).argmax(1)
    u, _, wq = O.quantize_values(w[np.arange(32), j], s, z, bits, True)
    # the largest-magnitude value lands on +-(2^(b-1)-1) and round-trips within float32 error
    assert (np.abs(u - (1 << (bits - 1))) == (1 << (bits - 1)) - 1).all()
    assert np.allclose(np.abs(wq), amax, rtol=1e-6)


def test_zero_group_does_not_divide_by_zero():
    w = np.zeros((3, 8))
    for sym in (False, True):
        r = O.rtn(w, 4, 8, sym)
        assert np.all(r["what"] == 0)
        assert np.all(r["scales"] == np.float32(1e-8))


# ----------------------------------------------------------------------------------
# Hessian
# ----------------------------------------------------------------------------------
def test_hessian_small_integer_case():
    X = np.array([[1.0, 2.0], [3.0, 4.0]])
    # x1 x1^T + x2 x2^T = [[1+9, 2+12], [2+12, 4+16]], times 2
    assert O.hessian(X).tolist() == [[20.0, 28.0], [28.0, 40.0]]


def test_hessian_equals_sum_of_token_outer_products():
    r = _rng(1)
    X = _bf16(r.standard_normal((37, 9)).astype(np.float32)).astype(np.float64)
    acc = np.zeros((9, 9))
    for t in range(X.shape[0]):
        for a in range(9):
            for b in range(9):
                acc[a, b] += 2.0 * X[t, a] * X[t, b]
    assert np.array_equal(O.hessian(X), acc)  # bf16 products and these short sums are exact


def test_hessian_batches_accumulate():
    r = _rng(2)
    X = _bf16(r.standard_normal((100, 16)).astype(np.float32))
    acc = O.HessianAccumulator(16)
    for a, b in [(0, 13), (13, 64), (64, 100)]:
        acc.add(X[a:b])
    assert acc.n_tok == 100
    assert np.allclose(acc.H, O.hessian(X), rtol=1e-14, atol=0)
    assert np.allclose(acc.H, acc.H.T)
    assert np.linalg.eigvalsh(acc.H).min() > -1e-9


# ----------------------------------------------------------------------------------
# prepare: U
# ----------------------------------------------------------------------------------
@pytest.mark.parametrize("n", [1, 5, 16, 130])
def test_U_is_upper_cholesky_of_inverse(n):
    H = _spd(n, n, cond_boost=20.0)
    p = O.prepare(H, 0.01, False)
    U = p["U"]
    assert np.allclose(np.tril(U, -1), 0)
    assert (np.diag(U) > 0).all()
    # U^T U H = I
    assert np.allclose(U.T @ U @ p["Hd"], np.eye(n), rtol=0, atol=1e-10)
    # the textbook route: upper Cholesky factor of the explicit inverse
    ref = scipy.linalg.cholesky(np.linalg.inv(p["Hd"]), lower=False)
    assert np.allclose(U, ref, rtol=1e-10, atol=1e-14 * np.abs(ref).max())


def test_damping_adds_relative_multiple_of_identity():
    H = _spd(12, 3)
    p = O.prepare(H, 0.1, False)
    d = np.diag(H).mean()
    assert np.allclose(p["Hd"] - H, 0.1 * d * np.eye(12), rtol=0, atol=1e-12 * d)


def test_not_positive_definite_raises():
    H = np.zeros((4, 4))
    H[0, 0] = 1.0
    H[0, 1] = H[1, 0] = 5.0
    H[1, 1] = 1.0
    H[2, 2] = H[3, 3] = 1.0
    with pytest.raises(O.NotPositiveDefinite):
        O.prepare(H, 0.0, False)


def test_dead_columns_fixed_and_zeroed():
    r = _rng(4)
    X = _bf16(r.standard_normal((64, 16)).astype(np.float32))
    X[:, [3, 11]] = 0
    H = O.hessian(X)
    W = r.normal(0, 0.02, (8, 16))
    res = O.quantize_layer(W, H, 4, 8, False, 0.01, True, block=None)
    assert res["dead"].tolist() == [i in (3, 11) for i in range(16)]
    assert np.all(res["what_orig"][:, [3, 11]] == 0)


# ----------------------------------------------------------------------------------
# act-order
# ----------------------------------------------------------------------------------
def test_act_order_sorts_descending_and_is_stable():
    H = np.diag([3.0, 7.0, 3.0, 9.0, 1.0, 7.0])
    assert O.act_order(H).tolist() == [3, 1, 5, 0, 2, 4]


@pytest.mark.parametrize("sym", [False, True])
def test_diagonal_H_with_act_order_equals_rtn_in_permuted_groups(sym):
    r = _rng(5)
    n = 64
    d = r.uniform(1, 10, n)
    W = r.normal(0, 0.02, (16, n))
    res = O.quantize_layer(W, np.diag(d), 4, 16, sym, 0.01, True, block=None)
    perm = np.argsort(-d, kind="stable")
    assert res["perm"].tolist() == perm.tolist()
    ref = O.rtn(W[:, perm], 4, 16, sym)
    assert np.array_equal(res["codes"], ref["codes"])
    assert np.array_equal(res["scales"], ref["scales"])
    assert np.array_equal(res["zeros"], ref["zeros"])
    assert np.array_equal(res["what_orig"], O.unpermute_columns(ref["what"], perm))


# ----------------------------------------------------------------------------------
# sweep
# ----------------------------------------------------------------------------------
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("g", [8, 32, -1])
def test_diagonal_H_collapses_to_rtn(sym, g):
    r = _rng(6)
    W = r.normal(0, 0.02, (24, 32))
    U = np.diag(1.0 / np.sqrt(r.uniform(0.5, 3.0, 32)))  # diagonal H => diagonal U
    sw = O.gptq_sweep(W, U, 4, g, sym)
    ref = O.rtn(W, 4, g, sym)
    for k in ("codes", "scales", "zeros", "what"):
        assert np.array_equal(sw[k], ref[k]), k


def _obs_sweep(W, Hd, bits, g, sym):
    """Sequential OBS form: full inverse, error scaled by its diagonal, then the inverse
    is downdated to remove the quantized column (independent of the Cholesky-row form)."""
    W = np.array(W, dtype=np.float64)
    m, n = W.shape
    g = n if g == -1 else g
    Hinv = np.linalg.inv(Hd)
    codes = np.zeros((m, n), dtype=np.int64)
    what = np.zeros((m, n))
    for q in range(n):
        if q % g == 0:
            s, z, _ = O.group_params(W[:, q:q + g], bits, sym)
        u, _, wq = O.quantize_values(W[:, q], s, z, bits, sym)
        codes[:, q], what[:, q] = u, wq
        err = (W[:, q] - wq) / Hinv[q, q]
        W[:, q + 1:] -= np.outer(err, Hinv[q, q + 1:])
        Hinv = Hinv - np.outer(Hinv[:, q], Hinv[q, :]) / Hinv[q, q]
    return codes, what


@pytest.mark.parametrize("n,g,sym,bits", [(8, 4, False, 4), (16, 8, True, 3), (12, -1, False, 2), (16, 16, False, 4)])
def test_obs_sequential_equals_cholesky_row_form(n, g, sym, bits):
    for seed in range(5):
        H = _spd(n, 100 + seed, cond_boost=10.0)
        p = O.prepare(H, 0.01, False)
        W = _rng(seed).normal(0, 0.02, (20, n))
        sw = O.gptq_sweep(W, p["U"], bits, g, sym)
        codes, what = _obs_sweep(W, p["Hd"], bits, g, sym)
        assert np.array_equal(sw["codes"], codes)
        assert np.allclose(sw["what"], what, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("n,B,g", [(256, 128, 128), (256, 128, 64), (512, 128, 256), (200, 64, -1), (96, 32, 32)])
def test_blocked_equals_unblocked(n, B, g):
    H = _spd(n, 7, cond_boost=15.0)
    p = O.prepare(H, 0.01, True)
    W = _rng(8).normal(0, 0.02, (16, n))
    Wp = W[:, p["perm"]]
    a = O.gptq_sweep(Wp, p["U"], 4, g, False)
    b = O.gptq_sweep(Wp, p["U"], 4, g, False, block=B)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.allclose(a["scales"], b["scales"], rtol=1e-6, atol=0)
    assert np.allclose(a["what"], b["what"], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("n,g,sym,block", [(256, 64, False, None), (384, 128, True, 128), (320, -1, False, 64)])
def test_sweep_errors_satisfy_E_U_equals_W_minus_Q(n, g, sym, block):
    """Column i's weight after the updates of the columns before it is w_i - sum_{k<i} e_k U[k, i],
    and e_i U[i, i] is its rounding residual, so E U = W - Q exactly (W the weights the sweep
    starts from, Q the dequantized values): a dropped, transposed or mis-signed update breaks
    it.  Consequence used by the CUDA path: the errors of all columns before a column block S
    reach it as -E[:, <S] U[<S, S] = (W - Q)[:, <S] V[<S, S] U[S, S] with V = U^-1."""
    H = _spd(n, 31, cond_boost=20.0)
    p = O.prepare(H, 0.01, True)
    Wp = _rng(32).normal(0, 0.02, (24, n))[:, p["perm"]]
    sw = O.gptq_sweep(Wp, p["U"], 3, g, sym, block=block)
    U = p["U"]
    D = Wp - sw["what"]
    assert np.allclose(sw["err"] @ U, D, rtol=0, atol=1e-12 * np.abs(Wp).max())
    V = np.linalg.inv(U)
    for s0, s1 in ((128, 256), (64, 192), (n - 64, n)):
        lhs = -sw["err"][:, :s0] @ U[:s0, s0:s1]
        rhs = D[:, :s0] @ V[:s0, s0:s1] @ U[s0:s1, s0:s1]
        assert np.allclose(lhs, rhs, rtol=0, atol=1e-10 * np.abs(lhs).max())


def test_brute_force_optimum_and_gptq_beats_rtn_on_average():
    bits, n = 4, 4
    e_gptq, e_rtn = [], []
    grid = np.array(list(itertools.product(range(16), repeat=n)))  # 65536 code vectors
    for seed in range(200):
        r = _rng(1000 + seed)
        A = r.standard_normal((n, n))
        H = A @ A.T + 0.05 * np.eye(n) + 0.5 * np.ones((n, n))   # correlated columns
        w = r.normal(0, 0.02, (1, n))
        U = O.upper_cholesky_of_inverse(H)
        sw = O.gptq_sweep(w, U, bits, -1, False)       # per-channel: one static (s, z)
        s = np.float64(sw["scales"][0, 0])
        z = np.float64(sw["zeros"][0, 0])
        d_opt = w - (grid - z) * s
        opt = np.einsum("ij,jk,ik->i", d_opt, H, d_opt).min()
        d = w - sw["what"]
        eg = float((d @ H @ d.T)[0, 0])
        rt = O.rtn(w, bits, -1, False)
        dr = w - rt["what"]
        er = float((dr @ H @ dr.T)[0, 0])
        assert rt["scales"][0, 0] == sw["scales"][0, 0]
        assert eg >= opt * (1 - 1e-12)
        e_gptq.append(eg)
        e_rtn.append(er)
    assert np.mean(e_gptq) < np.mean(e_rtn)


def test_last_column_keeps_its_own_error():
    n = 24
    H = _spd(n, 9, cond_boost=5.0)
    p = O.prepare(H, 0.01, False)
    W = _rng(10).normal(0, 0.02, (10, n))
    sw = O.gptq_sweep(W, p["U"], 4, 8, False)
    U = p["U"]
    # the value the last column is quantized from is the original minus every earlier compensation
    w_last = W[:, -1] - sw["err"][:, :-1] @ U[:-1, -1]
    s, z = sw["scales"][:, -1], sw["zeros"][:, -1]
    u, _, wq = O.quantize_values(w_last, s, z, 4, False)
    assert np.array_equal(u, sw["codes"][:, -1])
    assert np.allclose(sw["err"][:, -1], (w_last - wq) / U[-1, -1], rtol=1e-12)
    # and nothing depends on it: changing the last column of W leaves earlier columns alone
    W2 = W.copy()
    W2[:, -1] += 0.05
    sw2 = O.gptq_sweep(W2, p["U"], 4, 8, False)
    assert np.array_equal(sw2["codes"][:, :16], sw["codes"][:, :16])


def test_gptq_layer_error_below_rtn_on_outlier_layer():
    layer = synth.scaled_layer(synth.WORKLOADS["tiny_256x512"][0], m=64, n=256, n_tok=1024)
    X = synth.bf16_bits_to_f32(synth.make_x_bf16(layer))
    W = synth.make_w_fp16(layer).astype(np.float64)
    H = O.hessian(X)
    res = O.quantize_layer(W, H, 4, 128, False, 0.01, True)
    e_gptq = O.layer_error(W, res["what_orig"], H)
    e_rtn = O.layer_error(W, O.rtn(W, 4, 128, False)["what"], H)
    assert e_gptq < 0.8 * e_rtn


# ----------------------------------------------------------------------------------
# metrics and outputs
# ----------------------------------------------------------------------------------
def test_layer_error_identity_matches_direct_product():
    r = _rng(11)
    X = _bf16(r.standard_normal((300, 32)).astype(np.float32)).astype(np.float64)
    W = r.normal(0, 0.02, (8, 32))
    What = W + r.normal(0, 0.001, W.shape)
    direct = np.sum(((W - What) @ X.T) ** 2) / np.sum((W @ X.T) ** 2)
    assert np.isclose(O.layer_error(W, What, O.hessian(X)), direct, rtol=1e-12)


def test_pack_known_words():
    c = np.array([[1, 2, 3, 4, 5, 6, 7, 8]])
    assert O.pack_codes(c, 4).tolist() == [[0x87654321]]
    c2 = np.array([[3, 0, 1, 2] * 4])
    assert O.pack_codes(c2, 2).tolist() == [[int("10010011" * 4, 2)]]
    c3 = np.zeros((1, 32), dtype=np.int64)
    c3[0, 10] = 7          # stream bits 30..32 straddle words 0 and 1
    assert O.pack_codes(c3, 3).tolist() == [[0xC0000000, 0x1, 0x0]]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_roundtrip(bits):
    r = _rng(bits)
    c = r.integers(0, 1 << bits, (7, 96))
    assert np.array_equal(O.unpack_codes(O.pack_codes(c, bits), 96, bits), c)


def test_g_idx_definition():
    perm = np.array([2, 0, 3, 1])
    assert O.g_idx(perm, 2).tolist() == [0, 1, 0, 1]


# ----------------------------------------------------------------------------------
# the parity checker itself (mistakes planted in the oracle's output, on the CPU)
# ----------------------------------------------------------------------------------
def test_replay_adopts_in_band_flip_and_flags_out_of_band_flip():
    n = 64
    H = _spd(n, 12, cond_boost=5.0)
    p = O.prepare(H, 0.01, False)
    W = _rng(13).normal(0, 0.02, (32, n))
    ref = O.gptq_sweep(W, p["U"], 4, 32, False)
    dist = O.boundary_distance(ref["pre"], 4, False)
    # make one column-0 value sit in the band by nudging W there, then plant a flip
    i = 5
    codes = ref["codes"].copy()
    st = O.ReplayStats()
    O.gptq_sweep(W, p["U"], 4, 32, False, ref_codes=codes, ref_zeros=ref["zeros"], stats=st)
    assert st.hard_mismatch == 0 and st.adopted == 0 and st.identical == st.total
    r, c = np.unravel_index(np.argmax(dist > 0.2), dist.shape)
    codes[r, c] += 1 if codes[r, c] < 15 else -1
    st = O.ReplayStats()
    O.gptq_sweep(W, p["U"], 4, 32, False, ref_codes=codes, ref_zeros=ref["zeros"], stats=st)
    assert st.hard_mismatch >= 1
    # an in-band flip is adopted: build one at a tiny distance from a boundary
    W2 = W.copy()
    s, z = ref["scales"][i, 0], ref["zeros"][i, 0]
    W2[i, 0] = (np.floor(ref["pre"][i, 0]) + 0.5 - z + 1e-4) * np.float64(s)
    ref2 = O.gptq_sweep(W2, p["U"], 4, 32, False)
    assert O.boundary_distance(ref2["pre"][i, 0], 4, False) < 1e-3
    codes2 = ref2["codes"].copy()
    codes2[i, 0] -= 1
    # a reference that took the other side of that one in-band decision and carried on
    # consistently from there (this is what a correct kernel with a slightly different
    # rounding of that value produces)
    planted = O.gptq_sweep(W2, p["U"], 4, 32, False, ref_codes=codes2, ref_zeros=ref2["zeros"])
    assert planted["codes"][i, 0] == codes2[i, 0]
    st = O.ReplayStats()
    out = O.gptq_sweep(W2, p["U"], 4, 32, False, ref_codes=planted["codes"], ref_zeros=planted["zeros"], stats=st)
    assert st.adopted == 1 and st.hard_mismatch == 0
    assert st.identical == st.total - 1
    assert np.array_equal(out["codes"], planted["codes"])


# ----------------------------------------------------------------------------------------
# the packed result's consumer: decoding the stream with its documented layout (LSB-first
# per row, sweep order, groups of g sweep positions, perm back to original columns) gives
# back exactly the dequantized weights the sweep formed, and the product with them
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("bits,g,sym,desc_act", [(4, 64, False, True), (3, 32, True, True), (2, -1, False, False),
                                                 (8, 128, True, True)])
def test_dequantize_packed_round_trip(bits, g, sym, desc_act):
    r = np.random.default_rng(bits * 10 + (g if g > 0 else 1))
    m, n, N = 12, 256, 600
    X = r.standard_normal((N, n))
    X[:, r.choice(n, 4, replace=False)] *= 15.0
    W = 0.02 * r.standard_normal((m, n))
    H = O.hessian(X)
    res = O.quantize_layer(W, H, bits, g, sym, 0.01, desc_act)
    What = O.dequantize_packed(res["packed"], res["scales"], res["zeros"], res["perm"], n, bits, g)
    assert np.array_equal(What, res["what_orig"])
    Y = O.dequant_matmul(X[:7], res["packed"], res["scales"], res["zeros"], res["perm"], n, bits, g)
    assert np.allclose(Y, X[:7] @ res["what_orig"].T, rtol=1e-12, atol=1e-12)
    if desc_act:  # the permutation matters: decoding without it does not give W_hat back
        wrong = O.dequantize_packed(res["packed"], res["scales"], res["zeros"], np.arange(n), n, bits, g)
        assert not np.array_equal(wrong, res["what_orig"])


# ----------------------------------------------------------------------------------------
# the replay's zero-point branch: a reference whose zero-point took the other side of an
# in-band rounding decision is adopted; one outside the band, or more than one step away,
# is a hard mismatch (asymmetric quantizer of "模型量化实战…" §3.1: z = -round(xmin / s))
# ----------------------------------------------------------------------------------------
def test_zero_boundary_distance_closed_form():
    t = np.array([-2.4999, 3.2, 0.5, -0.7, 7.0, -3.5, 1e-9])
    want = np.array([1e-4, 0.3, 0.0, 0.2, 0.5, 0.0, 0.5 - 1e-9])
    assert np.allclose(O.zero_boundary_distance(t), want, atol=1e-12)


def _zero_rows():
    """Three rows whose first 32-column group has xmax = 12.5 (4-bit: s close to 1) and an
    xmin that puts t = xmin / s at 8e-5 (row 0), 0.25 (row 1) and 8e-5 (row 2) from a
    half-integer; the remaining values are small and inside the range."""
    rng = _rng(77)
    W = rng.uniform(-1.0, 1.0, (3, 64))
    W[:, 1] = 12.5
    W[0, 0] = -2.5 + 1e-4
    W[1, 0] = -2.25
    W[2, 0] = -2.5 - 1e-4
    return W


def test_replay_adopts_in_band_zero_flip():
    W = _zero_rows()
    U = np.eye(W.shape[1])
    ref = O.gptq_sweep(W, U, 4, 32, False)
    s, z, t = O.group_params(W[:, :32], 4, False)
    assert O.zero_boundary_distance(t[0]) < 1e-3 and z[0] == 2.0
    planted = ref["zeros"].copy()
    planted[0, 0] = 3.0                      # the other side of row 0's in-band decision
    st = O.ReplayStats()
    out = O.gptq_sweep(W, U, 4, 32, False, ref_zeros=planted, stats=st)
    assert st.zero_adopted == 1 and st.zero_hard_mismatch == 0
    assert np.array_equal(out["zeros"], planted)
    # the group's codes and dequantized values are formed with the adopted zero-point
    w32 = W[0, :32].astype(np.float32)
    u = np.clip(np.rint(w32 / s[0] + np.float32(3.0)), 0, 15)
    assert np.array_equal(out["codes"][0, :32], u.astype(np.int64))
    assert np.allclose(out["what"][0, :32], (u - 3.0) * np.float64(s[0]), rtol=0, atol=0)
    # the other rows are untouched
    assert np.array_equal(out["codes"][1:], ref["codes"][1:])


def test_replay_flags_out_of_band_or_far_zero_flip():
    W = _zero_rows()
    U = np.eye(W.shape[1])
    ref = O.gptq_sweep(W, U, 4, 32, False)
    _, z, t = O.group_params(W[:, :32], 4, False)
    assert O.zero_boundary_distance(t[1]) > 0.2
    planted = ref["zeros"].copy()
    planted[1, 0] = z[1] + 1                 # row 1: one step away, but far from a boundary
    planted[2, 0] = z[2] - 2                 # row 2: in band, but two steps away
    st = O.ReplayStats()
    out = O.gptq_sweep(W, U, 4, 32, False, ref_zeros=planted, stats=st)
    assert st.zero_adopted == 0 and st.zero_hard_mismatch == 2
    assert np.array_equal(out["zeros"], ref["zeros"])  # the oracle keeps its own decisions


def test_replay_ignores_zeros_of_symmetric_codes():
    """Symmetric zero-points are the constant 2^(b-1); the replay has nothing to adopt."""
    W = _zero_rows()
    U = np.eye(W.shape[1])
    planted = np.full((3, 2), 7.0, dtype=np.float32)
    st = O.ReplayStats()
    out = O.gptq_sweep(W, U, 4, 32, True, ref_zeros=planted, stats=st)
    assert st.zero_adopted == 0 and st.zero_hard_mismatch == 0
    assert (out["zeros"] == 8.0).all()


def test_dequant_matmul_equals_sum_in_sweep_order():
    """Y[t, r] = sum_k X[t, perm[k]] (code[r, k] - z[r, k // g]) s[r, k // g]: the product
    taken in sweep order with the activations gathered by perm, on a tiny case by loops."""
    rng = _rng(31)
    m, n, g, bits = 5, 64, 16, 4
    codes = rng.integers(0, 16, (m, n))
    s = rng.uniform(0.01, 0.1, (m, n // g)).astype(np.float32)
    z = rng.integers(0, 16, (m, n // g)).astype(np.float32)
    perm = rng.permutation(n)
    X = rng.normal(0, 1, (3, n))
    packed = O.pack_codes(codes, bits)
    Y = O.dequant_matmul(X, packed, s, z, perm, n, bits, g)
    for t in range(3):
        for r in range(m):
            acc = 0.0
            for k in range(n):
                acc += X[t, perm[k]] * (codes[r, k] - float(z[r, k // g])) * float(s[r, k // g])
            assert abs(Y[t, r] - acc) <= 1e-12 * (1 + abs(acc))


# ----------------------------------------------------------------------------------------
# blocks of U without forming all of it (the full-width parity checks use them)
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("n,k", [(64, 16), (96, 32), (40, 40)])
def test_leading_and_trailing_blocks_of_U(n, k):
    H = _spd(n, 5, cond_boost=10.0)
    p = O.prepare(H, 0.01, True)
    U = p["U"]
    assert np.allclose(O.upper_cholesky_of_inverse_leading(p["Hd"], k), U[:k, :k], rtol=1e-10, atol=1e-14)
    assert np.allclose(O.upper_cholesky_of_inverse_trailing(p["Hd"], k), U[-k:, -k:], rtol=1e-10, atol=1e-14)


def test_prepare_order_is_prepare_without_the_factor():
    H = _spd(48, 8)
    H[7, :] = H[:, 7] = 0.0
    a, b = O.prepare_order(H, 0.1, True), O.prepare(H, 0.1, True)
    assert np.array_equal(a["perm"], b["perm"]) and np.array_equal(a["dead"], b["dead"])
    assert np.array_equal(a["Hd"], b["Hd"]) and a["mean_diag"] == b["mean_diag"]


# ----------------------------------------------------------------------------------------
# the fp16 weights of the dequantizing product ("模型量化实战…" §4.3: INT4 weights are turned
# back into FP16 before the product)
# ----------------------------------------------------------------------------------------
def test_fp16_dequant_is_within_half_an_fp16_ulp_and_exact_for_power_of_two_scales():
    rng = _rng(41)
    m, n, g, bits = 6, 128, 32, 4
    codes = rng.integers(0, 16, (m, n))
    s = rng.uniform(1e-3, 0.05, (m, n // g)).astype(np.float32)
    z = rng.integers(0, 16, (m, n // g)).astype(np.float32)
    perm = rng.permutation(n)
    packed = O.pack_codes(codes, bits)
    w64 = O.dequantize_packed(packed, s, z, perm, n, bits, g)
    w16 = O.dequantize_packed_fp16(packed, s, z, perm, n, bits, g)
    assert w16.dtype == np.float16
    # round to nearest fp16: within half an ulp of the exact value (all values are normal here)
    ulp = np.spacing(np.abs(w16).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(w16.astype(np.float64) - w64) <= 0.5 * ulp * (1 + 1e-6) + 1e-30)
    # power-of-two scales: every (code - zero) * scale is representable, so nothing rounds
    s2 = np.full_like(s, np.float32(2.0 ** -7))
    assert np.array_equal(O.dequantize_packed_fp16(packed, s2, z, perm, n, bits, g).astype(np.float64),
                          O.dequantize_packed(packed, s2, z, perm, n, bits, g))


def test_fp16_dequant_rounds_the_float32_product():
    """One weight whose exact product lies just past an fp16 rounding midpoint, but whose float32
    product lands exactly on it (then round-half-even decides): the fp16 value follows the
    float32 product, as the reading states."""
    # (u - z) = 5 and s = 13428327 * 2^-26 (exact in float32): 5 s = 1 + 2^-11 + 3 * 2^-26,
    # which float32 rounds to 1 + 2^-11, the fp16 midpoint between 1 and 1 + 2^-10
    s = np.float32(13428327 * 2.0 ** -26)
    assert float(s) == 13428327 * 2.0 ** -26
    exact = 5.0 * np.float64(s)
    f32 = np.float32(5.0) * s
    assert exact == 1 + 2.0 ** -11 + 3 * 2.0 ** -26 and f32 == np.float32(1 + 2.0 ** -11)
    codes = np.array([[5] + [0] * 31])
    packed = O.pack_codes(codes, 4)
    w16 = O.dequantize_packed_fp16(packed, np.array([[s]]), np.array([[0.0]], dtype=np.float32),
                                   np.arange(32), 32, 4, -1)
    # half-even from the float32 midpoint goes down to 1.0; the exact product would round up
    assert w16[0, 0] == np.float16(1.0)
    assert np.float16(exact) == np.float16(1 + 2.0 ** -10)


def test_dequant_matmul_fp16_by_loops():
    rng = _rng(43)
    m, n, g, bits = 4, 64, 16, 3
    codes = rng.integers(0, 8, (m, n))
    s = rng.uniform(0.01, 0.1, (m, n // g)).astype(np.float32)
    z = rng.integers(0, 8, (m, n // g)).astype(np.float32)
    perm = rng.permutation(n)
    X16 = rng.normal(0, 1, (3, n)).astype(np.float16)
    Y = O.dequant_matmul_fp16(X16, O.pack_codes(codes, bits), s, z, perm, n, bits, g)
    for t in range(3):
        for r in range(m):
            acc = 0.0
            for k in range(n):
                w = np.float16(np.float32(codes[r, k] - z[r, k // g]) * s[r, k // g])
                acc += float(X16[t, perm[k]]) * float(w)
            assert abs(Y[t, r] - acc) <= 1e-12 * (1 + abs(acc))


# ----------------------------------------------------------------------------------------
# AWQ ("大模型量化…", AWQ section): importance, the median mask, scaling before rounding
# ----------------------------------------------------------------------------------------
def test_awq_importance_and_median_mask_on_a_worked_case():
    X = np.array([[1.0, -2.0, 0.5, 4.0], [-3.0, 2.0, 0.5, 0.0]])
    imp = O.awq_channel_importance(X)
    assert imp.tolist() == [2.0, 2.0, 0.5, 2.0]
    # sorted 0.5, 2, 2, 2: the lower median is 2; no channel is strictly above it
    assert O.awq_channel_scale(imp, 2.0).tolist() == [1.0, 1.0, 1.0, 1.0]
    imp2 = np.array([3.0, 1.0, 4.0, 2.0])          # lower median 2: channels 0 and 2 above it
    assert O.awq_channel_scale(imp2, 2.0).tolist() == [2.0, 1.0, 2.0, 1.0]
    imp3 = np.array([5.0, 1.0, 3.0])               # odd count: the middle value 3
    assert O.awq_channel_scale(imp3, 1.5).tolist() == [1.5, 1.0, 1.0]


def test_awq_with_unit_scale_is_round_to_nearest():
    rng = _rng(61)
    W = rng.normal(0, 0.02, (16, 128)).astype(np.float16).astype(np.float64)
    X = rng.normal(0, 1, (64, 128))
    a = O.awq_quantize(W, X, 1.0, 4, 32, False)
    r = O.rtn(W, 4, 32, False)
    assert np.array_equal(a["codes"], r["codes"]) and np.array_equal(a["scales"], r["scales"])
    assert np.array_equal(a["what"], r["what"])


@pytest.mark.parametrize("sym", [False, True])
def test_awq_protected_channels_get_a_finer_step(sym):
    """Dividing by the scale after rounding: a protected channel's error is at most half a
    quantization step divided by s (the page's reason the method works), an unprotected one's
    at most half a step."""
    rng = _rng(62)
    W = rng.normal(0, 0.02, (32, 256)).astype(np.float16).astype(np.float64)
    X = rng.normal(0, 1, (128, 256)) * np.where(np.arange(256) % 7 == 0, 20.0, 1.0)[None, :]
    a = O.awq_quantize(W, X, 2.0, 4, 64, sym)
    sc = a["channel_scale"].astype(np.float64)
    assert (sc == 2.0).sum() == 128                                    # half of an even count
    step = np.repeat(a["scales"].astype(np.float64), 64, axis=1)
    err = np.abs(W - a["what"])
    assert np.all(err <= 0.5 * step / sc[None, :] * (1 + 1e-5) + 1e-12)


# ----------------------------------------------------------------------------------------
# Percentile clipping of the range ("模型量化实战…" §3.1 LinearQuantizer, clip_ratio) and the
# page's error measures (same section, quantization_error)
# ----------------------------------------------------------------------------------------
def test_percentile_matches_numpy_bit_for_bit():
    """The page takes the clipped range from np.percentile; the oracle's percentile is written
    out from its definition and must give numpy's float32 result exactly, on ties, signed zeros
    and the percentiles that the clip ratios produce."""
    rng = _rng(71)
    ps = [0.0, 0.5, 1.0, 25.0, 37.3, 50.0, 63.2, 99.0, 99.5, 100.0]
    for c in (0.9, 0.95, 0.99, 0.999, 0.5, 0.01):
        ps += list(O.clip_percentiles(c, True)) + list(O.clip_percentiles(c, False))
    for k in (2, 3, 32, 128, 1000, 4096):
        a = rng.standard_normal((40, k)).astype(np.float16).astype(np.float32)   # many ties
        a[:, : k // 4] = np.where(rng.random((40, k // 4)) < 0.5, -0.0, 0.0)  # signed zeros
        for p in ps:
            assert np.array_equal(O.percentile_f32(a, p), np.percentile(a, p, axis=1)), (k, p)


def test_percentile_closed_forms():
    rng = _rng(72)
    v = rng.permutation(129).astype(np.float32)[None, :]          # the values 0..128
    for p, want in ((0.0, 0.0), (25.0, 32.0), (50.0, 64.0), (100.0, 128.0)):
        assert O.percentile_f32(v, p)[0] == want
    # five values: the 90th percentile sits 0.6 of the way from the 4th to the 5th
    w = np.array([[5.0, 1.0, 4.0, 2.0, 3.0]], dtype=np.float32)
    assert abs(float(O.percentile_f32(w, 90.0)[0]) - 4.6) <= 1e-6
    assert O.clip_percentiles(0.99, True) == (float(np.float32(0.99)) * 100.0,)
    lo, hi = O.clip_percentiles(0.99, False)
    assert abs(lo - 0.5) < 1e-6 and abs(hi - 99.5) < 1e-6 and abs(lo + hi - 100.0) < 1e-12


@pytest.mark.parametrize("sym", [False, True])
def test_clip_ratio_one_is_the_min_max_quantizer(sym):
    rng = _rng(73)
    W = rng.normal(0, 0.02, (24, 256)).astype(np.float16).astype(np.float64)
    a, b = O.rtn(W, 4, 64, sym), O.rtn(W, 4, 64, sym, clip=1.0)
    for key in ("codes", "scales", "zeros", "what"):
        assert np.array_equal(a[key], b[key])


def test_clipped_symmetric_scale_ignores_the_outlier():
    """One outlier in a group of 128: the 99th percentile of |w| interpolates between the
    126th and 127th smallest magnitudes, so the outlier (the largest) no longer sets the
    step, and its code saturates at the top of the range."""
    rng = _rng(74)
    base = rng.uniform(-1.0, 1.0, 128).astype(np.float32)
    rows = []
    for big in (50.0, 5000.0):
        r = base.copy()
        r[5] = big
        rows.append(r)
    W = np.stack(rows).astype(np.float64)
    s, z, _ = O.group_params(W, 8, True, clip=0.99)
    assert s[0] == s[1]
    mags = np.sort(np.abs(base[np.arange(128) != 5]))
    assert mags[-2] / 127 <= s[0] <= mags[-1] / 127 * (1 + 1e-6)
    r = O.rtn(W, 8, -1, True, clip=0.99)
    assert np.all(r["codes"][:, 5] == 255)                          # +127 stored as 127 + 128
    s_mm, _, _ = O.group_params(W, 8, True)
    assert np.all(s_mm > 10 * s)


def test_clipped_asymmetric_range_excludes_the_tails():
    """Groups of 1000 with clip 0.99: the 0.5th and 99.5th percentiles sit between ranks 4 and
    5 from either end, so the four smallest and four largest values may move anywhere beyond
    them without changing the parameters; the clipped range lies inside the min-max range and
    narrows as the ratio falls."""
    rng = _rng(75)
    w = rng.normal(0.1, 1.0, 1000).astype(np.float32)
    order = np.argsort(w)
    w2 = w.copy()
    w2[order[:4]] -= 100.0
    w2[order[-4:]] += 100.0
    W = np.stack([w, w2]).astype(np.float64)
    s, z, _ = O.group_params(W, 4, False, clip=0.99)
    assert s[0] == s[1] and z[0] == z[1]
    prev = None
    for c in (1.0, 0.999, 0.99, 0.9, 0.5):
        s_c, _, _ = O.group_params(W[:1], 4, False, clip=c)
        if prev is not None:
            assert s_c[0] <= prev
        prev = s_c[0]


def test_clipping_lowers_the_error_of_the_bulk_on_an_outlier_layer():
    """The page's reason for the ratio: clipping the outliers shrinks the step for every other
    weight.  With one large weight per 128, the bulk's squared error falls well below the
    min-max quantizer's, while the outliers' rises."""
    rng = _rng(76)
    W = rng.normal(0, 0.02, (64, 512))
    W[:, ::128] = 0.5
    W = W.astype(np.float16).astype(np.float64)
    bulk = np.ones(W.shape, bool)
    bulk[:, ::128] = False
    a, b = O.rtn(W, 4, 128, True), O.rtn(W, 4, 128, True, clip=0.99)
    e_mm, e_cl = (W - a["what"]) ** 2, (W - b["what"]) ** 2
    assert e_cl[bulk].mean() < 0.2 * e_mm[bulk].mean()
    assert e_cl[~bulk].mean() > e_mm[~bulk].mean()


def test_quantization_error_closed_forms():
    W = np.array([[1.0, 0.0], [0.0, 2.0]])
    mse, cos = O.quantization_error(W, W)
    assert mse == 0.0 and abs(cos - 1.0) < 1e-8
    mse, cos = O.quantization_error(W, 2 * W)
    assert mse == np.mean(W ** 2) and abs(cos - 1.0) < 1e-8
    mse, cos = O.quantization_error(np.array([1.0, 0.0]), np.array([0.0, 1.0]))
    assert mse == 1.0 and cos == 0.0
    mse, cos = O.quantization_error(np.array([3.0, 4.0]), np.array([-3.0, -4.0]))
    assert mse == 50.0 and abs(cos + 1.0) < 1e-9


def test_percentile_equals_numpy_on_arbitrary_data():
    """Property check over arbitrary finite float32 groups (extreme magnitudes, subnormals, heavy
    ties) and percentiles: the oracle's written-out percentile is np.percentile's, bit for bit."""
    hyp = pytest.importorskip("hypothesis")
    st = pytest.importorskip("hypothesis.strategies")
    from hypothesis.extra import numpy as hnp

    @hyp.settings(max_examples=300, deadline=None, derandomize=True)
    @hyp.given(hnp.arrays(np.float32, hnp.array_shapes(min_dims=2, max_dims=2, min_side=1, max_side=70),
                          elements=st.floats(-float(np.float32(1e30)), float(np.float32(1e30)), width=32)),
               st.floats(0.0, 100.0, allow_nan=False))
    def check(a, p):
        want = np.percentile(a, p, axis=1)
        got = O.percentile_f32(a, p)
        assert np.array_equal(got, want, equal_nan=True)

    check()
