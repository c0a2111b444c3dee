"""Plain CPU oracle for GPTQ's per-layer quantization solve (numpy, float64 state).

TEST INFRASTRUCTURE.  Only the test-suite, the smoke check of the entry module and the
CPU-baseline leg of the benchmark may import this module.  The CUDA path never calls it
and shares no code with it: the two meet only in the seeded input generators, which
hold none of the method's arithmetic.

Page titles used in the citations below:

  [P3] "GPTQ算法原理深度解析" (the Llama-2 GPTQ walkthrough page)
  [P4] "模型量化实战：从 INT8 PTQ 到 GPTQ 的精度保持与推理加速全解析"
  [P5] "大模型量化：GPTQ/AWQ/GGUF 原理对比，4-bit 量化对推理精度的影响"
  [P1] "Qwen2.5模型GPTQ量化精度损失实测：对比分析报告"
  [P2] "GPTQ量化损失深度解析：原理、影响与优化策略"

Precision: every floating-point quantity of the sweep is kept in float64, except the
decisions that turn floating point into integers (the code ``round(w/s + z)``, the
zero-point ``round(xmin/s)``) and the scale that feeds them.  The pages compute those
in float32 ([P5] GPTQ section, ``W.copy().astype(np.float32)``; [P4] §3.2,
``weight.clone().float()``), so they are taken in float32 here, exactly as the CUDA
path takes them.

Readings of the pages that this oracle fixes (the pages are silent or contradict one
another on each of these):

* H is accumulated without the 1/N of [P3] §2.2.1 (H = E[x x^T]); [P4] §3.2
  ``accumulate_hessian`` adds 2 x^T x per batch, and every later step is invariant to
  a positive scale of H.
* Dead columns (diag H == 0) get H_ii = 1 and a zeroed weight column; the pages only
  skip an all-zero column ([P5] GPTQ sketch).
* act-order / desc_act ([P1] §三 "权重重排序", [P2] "按敏感度排序", [P3] §3.3
  ``desc_act``) is read as a stable sort of the columns by descending diag H taken
  after the dead-column fix and before damping; ties keep the lower index first.
* The factor of [P4] §3.2 ``prepare`` (Cholesky, Cholesky-inverse, then an upper
  Cholesky that the page applies twice) is read as ONE upper Cholesky factor U of the
  damped inverse: H^-1 = U^T U.
* Group scales are computed per output row over the group's CURRENT (already
  compensated) weights, when the sweep reaches the group's first column; groups run in
  sweep order; per-channel is one group spanning the whole row.
* The asymmetric range is widened to include 0 so the zero-point fits in b bits; the
  symmetric code range is [-2^(b-1), 2^(b-1)-1] ([P4] §3.1); both scales are floored
  at 1e-8 ([P4] §3.1).  Rounding is round-half-to-even.
"""
from __future__ import annotations

import numpy as np
import scipy.linalg


class NotPositiveDefinite(ValueError):
    """The damped (permuted) Hessian has no Cholesky factor."""


# ==================================================================================
# S1  Hessian accumulation  ([P4] §3.2 GPTQQuantizer.accumulate_hessian; [P3] §2.2.1)
# ==================================================================================
def hessian(X) -> np.ndarray:
    """H = 2 X^T X of one calibration batch X [tokens, n] (values widened to float64)."""
    X = np.asarray(X, dtype=np.float64)
    return 2.0 * (X.T @ X)


class HessianAccumulator:
    """Running H += 2 x^T x and token count, one call per calibration batch ([P4] §3.2)."""

    def __init__(self, n: int):
        self.H = np.zeros((n, n), dtype=np.float64)
        self.n_tok = 0

    def add(self, X) -> None:
        self.H += hessian(X)
        self.n_tok += int(np.shape(X)[0])


# ==================================================================================
# S2-S4  prepare: dead columns, act-order, damping, U = upper-Cholesky(H^-1)
# ==================================================================================
def dead_columns(H) -> np.ndarray:
    """Columns that no calibration token excites (diag H == 0)."""
    return np.diag(np.asarray(H)) == 0


def act_order(H_fixed) -> np.ndarray:
    """desc_act permutation: columns by descending diag H, stable (ties: lower index first)."""
    return np.argsort(-np.diag(np.asarray(H_fixed, dtype=np.float64)), kind="stable")


def upper_cholesky_of_inverse(Hd) -> np.ndarray:
    """U upper-triangular with positive diagonal and H^-1 = U^T U  ([P4] §3.2 prepare).

    Follows the page's route: lower Cholesky L of H, H^-1 = L^-T L^-1 (the
    "cholesky_inverse"), then the upper Cholesky factor of H^-1.
    """
    Hd = np.asarray(Hd, dtype=np.float64)
    n = Hd.shape[0]
    try:
        L = np.linalg.cholesky(Hd)
    except np.linalg.LinAlgError as exc:
        raise NotPositiveDefinite(str(exc)) from None
    Linv = scipy.linalg.solve_triangular(L, np.eye(n), lower=True)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    try:
        return np.linalg.cholesky(Hinv).T.copy()
    except np.linalg.LinAlgError as exc:
        raise NotPositiveDefinite(str(exc)) from None


def upper_cholesky_of_inverse_leading(Hd, k: int) -> np.ndarray:
    """The leading k x k block of U = upper_cholesky_of_inverse(Hd), without forming all of U.

    U is upper-triangular, so column j < k of U has no entries below row j and the leading
    block of H^-1 = U^T U is U[:k, :k]^T U[:k, :k]: U[:k, :k] is the upper Cholesky factor of
    (H^-1)[:k, :k], whose columns come from a Cholesky solve of H against the first k unit
    vectors.
    """
    Hd = np.asarray(Hd, dtype=np.float64)
    n = Hd.shape[0]
    try:
        c = scipy.linalg.cho_factor(Hd, lower=True)
    except np.linalg.LinAlgError as exc:
        raise NotPositiveDefinite(str(exc)) from None
    E = np.zeros((n, k))
    E[np.arange(k), np.arange(k)] = 1.0
    Y = scipy.linalg.cho_solve(c, E)[:k]
    Y = 0.5 * (Y + Y.T)
    return np.linalg.cholesky(Y).T.copy()


def upper_cholesky_of_inverse_trailing(Hd, k: int) -> np.ndarray:
    """The trailing k x k block of U = upper_cholesky_of_inverse(Hd), which depends only on
    the trailing k x k block of Hd: with H = V V^T, V upper, the trailing block of V V^T is
    V22 V22^T, and U = V^-1 has U22 = V22^-1, the factor of Hd[-k:, -k:] alone."""
    Hd = np.asarray(Hd, dtype=np.float64)
    return upper_cholesky_of_inverse(Hd[-k:, -k:])


def prepare_order(H, damp: float, desc_act: bool) -> dict:
    """Steps S2-S3 and the damping of S4 on an accumulated H (any scale): ``dead`` (bool [n]),
    ``perm`` (int [n]: sweep position k holds original column perm[k]), ``Hd`` (damped,
    permuted H) and ``mean_diag``.
    Damping: H += damp * mean(diag H) * I  ([P4] §3.2 prepare; [P3] §3.3 damp_percent).
    """
    H1 = np.array(H, dtype=np.float64)
    n = H1.shape[0]
    dead = dead_columns(H1)
    H1[dead, dead] = 1.0
    perm = act_order(H1) if desc_act else np.arange(n)
    mean_diag = float(np.mean(np.diag(H1)))
    H1[np.arange(n), np.arange(n)] += damp * mean_diag
    Hd = H1[np.ix_(perm, perm)]
    return {"dead": dead, "perm": perm, "Hd": Hd, "mean_diag": mean_diag}


def prepare(H, damp: float, desc_act: bool) -> dict:
    """Steps S2-S4 on an accumulated H (any scale): prepare_order, then U, the upper
    Cholesky factor of the damped, permuted H's inverse."""
    p = prepare_order(H, damp, desc_act)
    p["U"] = upper_cholesky_of_inverse(p["Hd"])
    return p


# ==================================================================================
# Min-max uniform quantizer  ([P4] §2.1 and §3.1 LinearQuantizer; [P5] 对称量化)
# ==================================================================================
def qrange(bits: int, sym: bool):
    """Integer code range (before the unsigned offset of symmetric codes)."""
    if sym:
        return -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    return 0, (1 << bits) - 1


def percentile_f32(v, p: float):
    """The p-th percentile (0 <= p <= 100) of each row of float32 values ``v`` [m, k], by
    linear interpolation between the two order statistics around the position (k - 1) q,
    q = p / 100 (the default method of the page's np.percentile, [P4] §3.1).  Arithmetic in
    float32, as numpy does it for float32 data: p rounded to float32 and divided by 100 in
    float32, h = (k - 1) q, the weight
    t = h - floor(h); the value a + (b - a) t for t < 1/2 and b - (b - a) (1 - t) otherwise,
    with a, b the order statistics of ranks floor(h) and floor(h) + 1 (the latter clamped to
    k - 1)."""
    v = np.asarray(v, dtype=np.float32)
    k = v.shape[1]
    srt = np.sort(v, axis=1)
    q = np.float32(p) / np.float32(100.0)
    h = np.float32(k - 1) * q
    lo = int(np.floor(h))
    hi = min(lo + 1, k - 1)
    t = h - np.float32(lo)
    a, b = srt[:, lo], srt[:, hi]
    d = b - a
    if t < np.float32(0.5):
        return a + d * t
    return b - d * (np.float32(1.0) - t)


def clip_percentiles(clip: float, sym: bool):
    """The percentiles that bound the clipped range ([P4] §3.1 ``clip_ratio``): the 100 c-th
    percentile of |w| for symmetric codes; the (1 - c) 50-th and the 100 - (1 - c) 50-th
    percentiles of w for asymmetric codes.  c is the clip ratio rounded to float32 (the
    library takes it as a float); the percentiles are formed in float64."""
    c = float(np.float32(clip))
    if sym:
        return (c * 100.0,)
    return ((1.0 - c) * 50.0, 100.0 - (1.0 - c) * 50.0)


def group_params(wg, bits: int, sym: bool, clip: float = 1.0):
    """Scale and zero-point of each row of a group of columns ``wg`` [m, k].

    The range is the group's min / max (|w| max for symmetric codes), or with clip < 1 the
    percentiles of ``clip_percentiles`` ([P4] §3.1: a clip ratio below 1 replaces the range
    by percentiles, so that outliers saturate instead of widening the step).
    Returns (s, z, t) in float32: s the scale, z the zero-point of the UNSIGNED code
    (2^(b-1) for symmetric), t the pre-round zero value xmin/s (asymmetric only, else
    NaN), used by the replay check.
    """
    w = np.asarray(wg, dtype=np.float64).astype(np.float32)
    m = w.shape[0]
    clipped = float(np.float32(clip)) < 1.0
    if sym:
        qpos = np.float32((1 << (bits - 1)) - 1)
        if clipped:
            amax = percentile_f32(np.abs(w), clip_percentiles(clip, True)[0])
        else:
            amax = np.max(np.abs(w), axis=1)
        s = np.maximum(amax / qpos, np.float32(1e-8))
        z = np.full(m, np.float32(1 << (bits - 1)), dtype=np.float32)
        t = np.full(m, np.nan, dtype=np.float32)
    else:
        qmax = np.float32((1 << bits) - 1)
        if clipped:
            p_lo, p_hi = clip_percentiles(clip, False)
            wlo, whi = percentile_f32(w, p_lo), percentile_f32(w, p_hi)
        else:
            wlo, whi = np.min(w, axis=1), np.max(w, axis=1)
        xmin = np.minimum(wlo, np.float32(0))
        xmax = np.maximum(whi, np.float32(0))
        s = np.maximum((xmax - xmin) / qmax, np.float32(1e-8))
        t = xmin / s
        z = -np.rint(t)
    return s.astype(np.float32), z.astype(np.float32), t.astype(np.float32)


def quantize_values(w, s, z, bits: int, sym: bool):
    """Quantize values w (one per row) with per-row (s, z).

    Returns (u, v, what): u the unsigned code, v the float32 pre-round value, what the
    dequantized value (u - z) * s in float64.
    """
    w32 = np.asarray(w, dtype=np.float64).astype(np.float32)
    lo, hi = qrange(bits, sym)
    if sym:
        v = w32 / s
        q = np.clip(np.rint(v), lo, hi)
        u = q - lo                       # unsigned storage: u = q + 2^(b-1)
    else:
        v = w32 / s + z
        u = np.clip(np.rint(v), lo, hi)
    what = (u.astype(np.float64) - z.astype(np.float64)) * s.astype(np.float64)
    return u.astype(np.int64), v.astype(np.float32), what


def boundary_distance(v, bits: int, sym: bool):
    """Distance of a pre-round value to the nearest rounding boundary inside the code range."""
    lo, hi = qrange(bits, sym)
    v = np.asarray(v, dtype=np.float64)
    b = np.clip(np.floor(v) + 0.5, lo + 0.5, hi - 0.5)
    return np.abs(v - b)


def zero_boundary_distance(t):
    t = np.asarray(t, dtype=np.float64)
    return np.abs(t - (np.floor(t) + 0.5))


# ==================================================================================
# S5-S6  column sweep with error compensation
#   [P5] GPTQ section (column loop, error pushed to the not-yet-quantized columns, the
#   last column keeps its own error); [P4] §3.2 quantize_block (block_size 128)
# ==================================================================================
def _group_width(group_size: int, n: int) -> int:
    return n if group_size in (-1, 0) else group_size


class ReplayStats:
    def __init__(self):
        self.total = 0
        self.identical = 0
        self.adopted = 0
        self.hard_mismatch = 0
        self.zero_adopted = 0
        self.zero_hard_mismatch = 0

    def as_dict(self):
        return dict(self.__dict__)


def gptq_sweep(Wp, U, bits: int, group_size: int, sym: bool, block: int | None = None,
               ref_codes=None, ref_zeros=None, band: float = 1e-3, stats: ReplayStats | None = None):
    """Quantize the columns of Wp (float64 [m, n], sweep order) with error compensation.

    For column i: when i starts a group, the group's (s, z) come from the current
    W[:, i:i+g]; u = Q(w_i); e = (w_i - what_i) / U[i, i]; W[:, j] -= e * U[i, j] for j > i.
    ``block=None`` applies every update immediately; ``block=B`` applies updates inside
    the current block of B columns immediately and the rest as one product per block,
    which changes nothing but the order of the float64 additions.

    Replay (``ref_codes``/``ref_zeros`` given): where this sweep's decision differs by
    one from the reference's and its pre-round value lies within ``band`` of a rounding
    boundary, the reference's integer is adopted and the sweep continues with it.

    Returns dict(codes [m,n] unsigned, scales [m,G] f32, zeros [m,G] f32, what [m,n] f64,
    pre [m,n] f32 pre-round values, err [m,n] f64 scaled errors e).
    """
    W = np.array(Wp, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    g = _group_width(group_size, n)
    if n % g:
        raise ValueError("group size must divide the number of columns")
    if block is not None and not (g == n or g % block == 0 or block % g == 0):
        raise ValueError("blocked sweep needs group size dividing or divided by the block")
    G = n // g
    codes = np.zeros((m, n), dtype=np.int64)
    scales = np.zeros((m, G), dtype=np.float32)
    zeros = np.zeros((m, G), dtype=np.float32)
    what = np.zeros((m, n), dtype=np.float64)
    pre = np.zeros((m, n), dtype=np.float32)
    errs = np.zeros((m, n), dtype=np.float64)
    B = n if block is None else block
    s = z = None
    for i1 in range(0, n, B):
        i2 = min(n, i1 + B)
        for i in range(i1, i2):
            if i % g == 0:
                s, z, t = group_params(W[:, i:i + g], bits, sym)
                if ref_zeros is not None and not sym:
                    rz = np.asarray(ref_zeros[:, i // g], dtype=np.float32)
                    diff = rz != z
                    ok = diff & (np.abs(rz - z) == 1) & (zero_boundary_distance(t) < band)
                    z = np.where(ok, rz, z).astype(np.float32)
                    if stats is not None:
                        stats.zero_adopted += int(ok.sum())
                        stats.zero_hard_mismatch += int((diff & ~ok).sum())
                scales[:, i // g] = s
                zeros[:, i // g] = z
            u, v, wq = quantize_values(W[:, i], s, z, bits, sym)
            if ref_codes is not None:
                rc = np.asarray(ref_codes[:, i], dtype=np.int64)
                diff = rc != u
                ok = diff & (np.abs(rc - u) == 1) & (boundary_distance(v, bits, sym) < band)
                if stats is not None:
                    stats.total += m
                    stats.identical += int((~diff).sum())
                    stats.adopted += int(ok.sum())
                    stats.hard_mismatch += int((diff & ~ok).sum())
                if ok.any():
                    u = np.where(ok, rc, u)
                    wq = (u.astype(np.float64) - z.astype(np.float64)) * s.astype(np.float64)
            codes[:, i] = u
            pre[:, i] = v
            what[:, i] = wq
            e = (W[:, i] - wq) / U[i, i]
            errs[:, i] = e
            if i + 1 < i2:
                W[:, i + 1:i2] -= np.outer(e, U[i, i + 1:i2])
        if i2 < n:
            W[:, i2:] -= errs[:, i1:i2] @ U[i1:i2, i2:]
    return {"codes": codes, "scales": scales, "zeros": zeros, "what": what, "pre": pre, "err": errs}


def rtn(W, bits: int, group_size: int, sym: bool, clip: float = 1.0):
    """Round-to-nearest with the same min-max groups and no compensation ([P5] "naive" 4-bit);
    with clip < 1 the groups' ranges are percentiles ([P4] §3.1 LinearQuantizer with
    ``clip_ratio``; the page's per-channel granularity is group_size -1 here).

    Returns dict(codes, scales, zeros, what) in the column order of W.
    """
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    g = _group_width(group_size, n)
    G = n // g
    codes = np.zeros((m, n), dtype=np.int64)
    scales = np.zeros((m, G), dtype=np.float32)
    zeros = np.zeros((m, G), dtype=np.float32)
    what = np.zeros((m, n), dtype=np.float64)
    for k in range(G):
        s, z, _ = group_params(W[:, k * g:(k + 1) * g], bits, sym, clip)
        scales[:, k], zeros[:, k] = s, z
        for j in range(k * g, (k + 1) * g):
            u, _, wq = quantize_values(W[:, j], s, z, bits, sym)
            codes[:, j], what[:, j] = u, wq
    return {"codes": codes, "scales": scales, "zeros": zeros, "what": what}


def quantization_error(W, What):
    """The page's two error measures of a quantized tensor ([P4] §3.1 ``quantization_error``):
    the mean squared error and the cosine similarity of W and its dequantized copy, the latter
    with 1e-8 added to the product of the norms.  float64."""
    W = np.asarray(W, dtype=np.float64)
    What = np.asarray(What, dtype=np.float64)
    mse = float(np.mean((W - What) ** 2))
    cos = float(np.sum(W * What) / (np.sqrt(np.sum(W * W)) * np.sqrt(np.sum(What * What)) + 1e-8))
    return mse, cos


# ==================================================================================
# S7  outputs: packed codes, g_idx, dequantized weights in original order
# ==================================================================================
def pack_codes(codes, bits: int) -> np.ndarray:
    """Pack unsigned b-bit codes [m, n] (sweep order) into a LSB-first bit stream per row.

    Code k of a row occupies stream bits k*b .. k*b+b-1; stream bit p is bit (p mod 32)
    of 32-bit word p div 32.  n*b must be a multiple of 32.
    """
    codes = np.asarray(codes, dtype=np.int64)
    m, n = codes.shape
    if (n * bits) % 32:
        raise ValueError("n * bits must be a multiple of 32")
    bitsm = ((codes[:, :, None] >> np.arange(bits)[None, None, :]) & 1).reshape(m, n * bits)
    words = (bitsm.reshape(m, n * bits // 32, 32).astype(np.uint64)
             << np.arange(32, dtype=np.uint64)[None, None, :]).sum(axis=2)
    return words.astype(np.uint32)


def unpack_codes(words, n: int, bits: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint32)
    m = words.shape[0]
    bitsm = ((words[:, :, None].astype(np.uint64) >> np.arange(32, dtype=np.uint64)) & 1)
    bitsm = bitsm.reshape(m, -1)[:, :n * bits].reshape(m, n, bits)
    return (bitsm.astype(np.int64) << np.arange(bits)[None, None, :]).sum(axis=2)


def g_idx(perm, group_size: int) -> np.ndarray:
    """Group of each ORIGINAL column: g_idx[perm[k]] = k // g."""
    perm = np.asarray(perm)
    n = perm.shape[0]
    g = _group_width(group_size, n)
    out = np.empty(n, dtype=np.int32)
    out[perm] = np.arange(n) // g
    return out


def unpermute_columns(Ap, perm) -> np.ndarray:
    """Column k of the sweep-order matrix goes back to original column perm[k]."""
    A = np.empty_like(Ap)
    A[:, np.asarray(perm)] = Ap
    return A


def layer_error(W, What, H0) -> float:
    """||(W - What) X||^2 / ||W X||^2 through the Hessian identity with the undamped H0 ([P3] §2.1)."""
    W = np.asarray(W, dtype=np.float64)
    D = W - np.asarray(What, dtype=np.float64)
    H0 = np.asarray(H0, dtype=np.float64)
    return float(np.sum((D @ H0) * D) / np.sum((W @ H0) * W))


# ==================================================================================
# the packed result's consumer (the step after the path: a layer that keeps its weights as
# codes and dequantizes them for the product: per [P4] §4.3, INT4 weights are turned back
# into FP16 values before the matrix product, and the gain is memory bandwidth)
# ==================================================================================
def dequantize_packed(packed, scales, zeros, perm, n: int, bits: int, group_size: int) -> np.ndarray:
    """W_hat in ORIGINAL column order from the packed output of the path: code k of a row
    (sweep order) belongs to group k // g and dequantizes as (code - zero) * scale ([P4] §3.1
    dequantize), formed exactly in float64 from the stored float32 scale and zero; sweep
    position k goes back to original column perm[k]."""
    codes = unpack_codes(packed, n, bits)
    grp = np.arange(n) // _group_width(group_size, n)
    s = np.asarray(scales, dtype=np.float32).astype(np.float64)[:, grp]
    z = np.asarray(zeros, dtype=np.float32).astype(np.float64)[:, grp]
    return unpermute_columns((codes.astype(np.float64) - z) * s, perm)


def dequant_matmul(X, packed, scales, zeros, perm, n: int, bits: int, group_size: int) -> np.ndarray:
    """Y = X W_hat^T for activations X [tokens, n] in original column order (float64)."""
    return np.asarray(X, dtype=np.float64) @ dequantize_packed(packed, scales, zeros, perm, n, bits, group_size).T


def dequantize_packed_fp16(packed, scales, zeros, perm, n: int, bits: int, group_size: int) -> np.ndarray:
    """The FP16 weights an INT4 layer is turned back into before its product ([P4] §4.3):
    (code - zero) * scale formed in float32, the precision the scales are stored in (the
    difference of two small integers is exact; the product is rounded to nearest), then
    rounded to nearest fp16.  ORIGINAL column order, like dequantize_packed."""
    codes = unpack_codes(packed, n, bits)
    grp = np.arange(n) // _group_width(group_size, n)
    s = np.asarray(scales, dtype=np.float32)[:, grp]
    z = np.asarray(zeros, dtype=np.float32)[:, grp]
    w32 = (codes.astype(np.float32) - z) * s
    return unpermute_columns(w32.astype(np.float16), perm)


def dequant_matmul_fp16(X16, packed, scales, zeros, perm, n: int, bits: int, group_size: int) -> np.ndarray:
    """Y = X W16^T in float64 for fp16 activations X16 [tokens, n] (original column order) and
    the fp16 weights of dequantize_packed_fp16: every product of two fp16 values is exact in
    float64 and the sum is taken in float64."""
    W16 = dequantize_packed_fp16(packed, scales, zeros, perm, n, bits, group_size)
    return np.asarray(X16, dtype=np.float16).astype(np.float64) @ W16.astype(np.float64).T


# ==================================================================================
# AWQ: activation-aware channel scaling before round-to-nearest ([P5] "AWQ：激活值感知 +
# 通道缩放，又快又好": importance = mean |x| per input channel; the channels above the median
# importance are multiplied by s (2.0 in the page's sketch); the scaled weights are quantized
# to nearest and the dequantized weights are divided by the scale again)
# ==================================================================================
def awq_channel_importance(X) -> np.ndarray:
    """Mean |x| of each input channel over the calibration tokens X [tokens, n] (float64)."""
    X = np.asarray(X, dtype=np.float64)
    return np.abs(X).sum(axis=0) / X.shape[0]


def awq_channel_scale(importance, s_protect: float) -> np.ndarray:
    """s_protect for the channels whose importance exceeds the median, 1 for the others.  The
    page's torch.median gives the lower of the two middle values of an even count."""
    v = np.asarray(importance, dtype=np.float64)
    med = np.sort(v)[(v.shape[0] - 1) // 2]
    return np.where(v > med, np.float32(s_protect), np.float32(1.0)).astype(np.float32)


def awq_quantize(W, X, s_protect: float, bits: int, group_size: int, sym: bool) -> dict:
    """The page's AWQ on one layer: W_scaled = W * scale (each input channel; float32 product),
    round-to-nearest of W_scaled with the min-max groups of this module (original column
    order), W_hat = dequantized / scale.  Returns rtn's dict plus channel_scale, importance,
    packed codes and what (float64, original order)."""
    imp = awq_channel_importance(X)
    scale = awq_channel_scale(imp, s_protect)
    Ws = np.asarray(W, dtype=np.float32) * scale[None, :]
    r = rtn(Ws.astype(np.float64), bits, group_size, sym)
    r["channel_scale"] = scale
    r["importance"] = imp
    r["what"] = r["what"] / scale[None, :].astype(np.float64)
    r["packed"] = pack_codes(r["codes"], bits)
    return r


# ==================================================================================
# whole layer
# ==================================================================================
def quantize_layer(W, H, bits: int, group_size: int, sym: bool, damp: float, desc_act: bool,
                   block: int | None = 128, prep: dict | None = None):
    """Steps S2-S7 for one layer from its accumulated H; W given in original column order."""
    W0 = np.asarray(W, dtype=np.float64)
    p = prepare(H, damp, desc_act) if prep is None else prep
    Wf = W0.copy()
    Wf[:, p["dead"]] = 0.0
    Wp = Wf[:, p["perm"]]
    r = gptq_sweep(Wp, p["U"], bits, group_size, sym, block=block)
    r["perm"] = p["perm"]
    r["U"] = p["U"]
    r["dead"] = p["dead"]
    r["g_idx"] = g_idx(p["perm"], group_size)
    r["what_orig"] = unpermute_columns(r["what"], p["perm"])
    r["packed"] = pack_codes(r["codes"], bits) if (W0.shape[1] * bits) % 32 == 0 else None
    return r
