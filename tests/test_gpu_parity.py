"""Parity of the CUDA path (through the C ABI) with the CPU oracle on seeded inputs."""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import synth
from post_weight_quantization_16_b200.gptq import GPTQContext, GPTQError, ERR_NOT_PD, ERR_STATE
from tests import gpu_helpers as GH

pytestmark = pytest.mark.gpu

TINY, TINY_Q = synth.WORKLOADS["tiny_256x512"]


def _h_rel(H, Href):
    return np.linalg.norm(H - Href) / np.linalg.norm(Href)


# ----------------------------------------------------------------------------------------
# S1 Hessian
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("n,n_tok", [(512, 2048), (384, 1000), (128, 64), (768, 4157)])
def test_hessian_matches_fp64(n, n_tok):
    layer = synth.scaled_layer(TINY, m=64, n=n, n_tok=n_tok)
    X = synth.make_x_bf16(layer)
    with GPTQContext(n, 64, 0) as ctx:
        ctx.accumulate_hessian(GH.bf16_to_dev(X))
        H, nt = ctx.get_hessian()
    H = H.cpu().numpy().astype(np.float64)
    Href = O.hessian(synth.bf16_bits_to_f32(X))
    assert nt == n_tok
    assert _h_rel(H, Href) <= GH.H_REL_FRO
    assert np.array_equal(H, H.T)


def test_hessian_batches_strides_and_chunks():
    layer = synth.scaled_layer(TINY, m=64, n=512, n_tok=6000)
    X = synth.make_x_bf16(layer)
    Href = O.hessian(synth.bf16_bits_to_f32(X))
    for chunk in (64, 1024, 1 << 20):
        with GPTQContext(512, 64, 0) as ctx:
            ctx.set_hessian_chunk(chunk)
            # batches of uneven sizes, the middle one taken from a wider (padded) buffer
            ctx.accumulate_hessian(GH.bf16_to_dev(X[:1000]))
            pad = np.zeros((3000, 512 + 64), dtype=np.uint16)
            pad[:, :512] = X[1000:4000]
            Xp = GH.bf16_to_dev(pad)
            ctx.accumulate_hessian(Xp[:, :512])
            ctx.accumulate_hessian(GH.bf16_to_dev(X[4000:]))
            H, nt = ctx.get_hessian()
        assert nt == 6000
        assert _h_rel(H.cpu().numpy().astype(np.float64), Href) <= GH.H_REL_FRO, chunk


# ----------------------------------------------------------------------------------------
# S2-S4 prepare
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("n,desc_act,damp", [(128, True, 0.01), (256, False, 0.1), (384, True, 0.01),
                                             (640, False, 0.01), (640, True, 0.1), (1024, True, 0.01),
                                             (2304, True, 0.01), (3200, False, 0.01)])
def test_prepare_perm_and_factor(n, desc_act, damp):
    """Past 1024 columns the factorization leaves out the U blocks of the recursion's left edge
    and gptq_get_factor completes them: the whole U is checked."""
    layer = synth.scaled_layer(TINY, m=64, n=n, n_tok=3000)
    X = synth.make_x_bf16(layer)
    with GPTQContext(layer.n, 64, 0) as ctx:
        ctx.accumulate_hessian(GH.bf16_to_dev(X))
        H, _ = ctx.get_hessian()
        perm = ctx.prepare(damp, desc_act).cpu().numpy()
        U = ctx.get_factor().cpu().numpy().astype(np.float64)
    H = H.cpu().numpy().astype(np.float64)
    prep = O.prepare(H, damp, desc_act)          # the oracle on the GPU's H
    assert np.array_equal(perm, prep["perm"])
    assert np.allclose(np.tril(U, -1), 0)
    err = np.abs(U - prep["U"]).max() / np.abs(prep["U"]).max()
    assert err <= 2e-5, err
    resid = np.abs(U.T @ U @ prep["Hd"] - np.eye(layer.n)).max()
    assert resid <= 1e-3, resid


def test_not_positive_definite_is_reported():
    n = 256
    H = np.eye(n, dtype=np.float32)
    H[3, 7] = H[7, 3] = 4.0       # 2x2 minor [[1,4],[4,1]] is indefinite
    with GPTQContext(n, 32, 0) as ctx:
        ctx.set_hessian(torch.from_numpy(H).to(GH.DEV), 10)
        with pytest.raises(GPTQError) as ei:
            ctx.prepare(0.0, False)
        assert ei.value.status == ERR_NOT_PD
        # not prepared: quantizing is a state error
        W = torch.zeros((32, n), dtype=torch.float16, device=GH.DEV)
        with pytest.raises(GPTQError) as ei:
            ctx.quantize_layer(W, 4, 128, False)
        assert ei.value.status == ERR_STATE
        # with enough damping the same H is positive definite: [[1,4],[4,1]] + 10*mean(diag)*I
        ctx.prepare(10.0, False)


def test_state_machine():
    layer = synth.scaled_layer(TINY, m=32, n=256, n_tok=512)
    X = GH.bf16_to_dev(synth.make_x_bf16(layer))
    with GPTQContext(256, 32, 0) as ctx:
        W = torch.zeros((32, 256), dtype=torch.float16, device=GH.DEV)
        with pytest.raises(GPTQError) as ei:
            ctx.quantize_layer(W, 4, 128, False)
        assert ei.value.status == ERR_STATE
        ctx.accumulate_hessian(X)
        ctx.prepare(0.01, True)
        with pytest.raises(GPTQError) as ei:
            ctx.accumulate_hessian(X)
        assert ei.value.status == ERR_STATE
        ctx.reset()
        ctx.accumulate_hessian(X)
        _, nt = ctx.get_hessian()
        assert nt == 512


# ----------------------------------------------------------------------------------------
# S5-S7 sweep (stage-isolated replay against the oracle on the GPU's H)
# ----------------------------------------------------------------------------------------
SWEEP_CASES = [
    # bits, group, sym, desc_act, damp
    (4, 128, False, False, 0.01),
    (4, 128, False, True, 0.01),
    (4, 128, True, True, 0.01),
    (3, 64, False, True, 0.1),
    (2, 32, False, True, 0.01),
    (2, -1, False, True, 0.1),
    (3, 256, True, False, 0.01),
    (8, 128, False, True, 0.01),
    (4, 64, True, True, 0.1),
]


@pytest.mark.parametrize("bits,g,sym,desc_act,damp", SWEEP_CASES)
def test_quantize_layer_parity(bits, g, sym, desc_act, damp):
    layer = synth.scaled_layer(TINY, m=96, n=512, n_tok=2048)
    qs = synth.QuantSetting(bits, g, sym, damp, desc_act)
    gpu = GH.run_path(layer, qs)
    prep = O.prepare(gpu["H"], damp, desc_act)
    assert np.array_equal(gpu["perm"], prep["perm"])
    st, rep = GH.check_sweep_replay(gpu["W"], prep, gpu, qs)
    GH.assert_replay_ok(st, rep, gpu)
    # g_idx and the dequantized weights in original order
    assert np.array_equal(gpu["g_idx"], O.g_idx(prep["perm"], g))
    what = O.unpermute_columns(rep["what"], prep["perm"])
    scale_ref = np.repeat(rep["scales"], (layer.n if g == -1 else g), axis=1)[:, np.argsort(prep["perm"])]
    # (u - z) * s in fp32 on the GPU vs float64 in the oracle, with scales equal to 1e-5
    assert np.all(np.abs(gpu["w_hat"] - what) <= 2e-7 * np.abs(what) + 1e-5 * scale_ref * (1 << bits) + 1e-12)
    # layer error within 1 % of the oracle's own (un-replayed) run, measured with the exact H
    Href = O.hessian(synth.bf16_bits_to_f32(gpu["X"]))
    own = O.quantize_layer(gpu["W"].astype(np.float64), gpu["H"], bits, g, sym, damp, desc_act)
    e_gpu = O.layer_error(gpu["W"], gpu["w_hat"], Href)
    e_own = O.layer_error(gpu["W"], own["what_orig"], Href)
    assert abs(e_gpu - e_own) <= GH.LAYER_ERR_REL * e_own, (e_gpu, e_own)


def test_end_to_end_tiny_config():
    """The tiny workload end to end: H against the oracle's own H, then the full replay."""
    gpu = GH.run_path(TINY, TINY_Q)
    Href = O.hessian(synth.bf16_bits_to_f32(gpu["X"]))
    assert _h_rel(gpu["H"], Href) <= GH.H_REL_FRO
    prep = O.prepare(gpu["H"], TINY_Q.damp, TINY_Q.desc_act)
    st, rep = GH.check_sweep_replay(gpu["W"], prep, gpu, TINY_Q)
    GH.assert_replay_ok(st, rep, gpu)
    assert np.array_equal(gpu["packed"], O.pack_codes(rep["codes"], TINY_Q.bits))


def test_dead_columns_on_gpu():
    layer = synth.scaled_layer(TINY, m=64, n=256, n_tok=1024)
    X = synth.make_x_bf16(layer)
    X[:, [5, 77, 200]] = 0
    qs = synth.QuantSetting(4, 128, False, 0.01, True)
    gpu = GH.run_path(layer, qs, X_bits=X)
    assert np.all(gpu["w_hat"][:, [5, 77, 200]] == 0)
    prep = O.prepare(gpu["H"], qs.damp, qs.desc_act)
    assert prep["dead"][[5, 77, 200]].all()
    st, rep = GH.check_sweep_replay(gpu["W"], prep, gpu, qs)
    GH.assert_replay_ok(st, rep, gpu)


def test_ragged_rows_and_wider_context():
    layer = synth.scaled_layer(TINY, m=45, n=384, n_tok=777)
    qs = synth.QuantSetting(4, 128, True, 0.01, True)
    gpu = GH.run_path(layer, qs, ctx_m=300)
    prep = O.prepare(gpu["H"], qs.damp, qs.desc_act)
    st, rep = GH.check_sweep_replay(gpu["W"], prep, gpu, qs)
    GH.assert_replay_ok(st, rep, gpu)


@pytest.mark.parametrize("n,g,sym,bits", [(2048, 128, False, 4), (1152, -1, False, 4), (1536, 384, True, 3),
                                          (2048, 256, False, 2), (1280, 64, True, 4), (2048, 1024, False, 4),
                                          (4096, 2048, False, 4)])
def test_quantize_layer_parity_across_super_blocks(n, g, sym, bits):
    """Layers wider than one super-block (the far columns are updated once per super-block),
    including a partial last super-block; groups of 256 and 1024 columns (the super-block
    widens to hold a whole group) and groups of 384 and 2048 columns (the update past a
    super-block taken as -E U on the completed factor, groups reaching past super-blocks)."""
    layer = synth.scaled_layer(TINY, m=80, n=n, n_tok=2 * n)
    qs = synth.QuantSetting(bits, g, sym, 0.01, True)
    gpu = GH.run_path(layer, qs)
    prep = O.prepare(gpu["H"], qs.damp, qs.desc_act)
    assert np.array_equal(gpu["perm"], prep["perm"])
    st, rep = GH.check_sweep_replay(gpu["W"], prep, gpu, qs)
    GH.assert_replay_ok(st, rep, gpu)


@pytest.mark.parametrize("slab", [128, 512, 1024])
def test_quantize_layer_parity_other_slab_widths(slab, monkeypatch):
    """The sweep's slab width (columns per launch, whose later columns are updated inside the
    launch) changes only the order of the fp32 updates: parity at other widths than the default."""
    monkeypatch.setenv("GPTQ_SLAB_WIDTH", str(slab))
    layer = synth.scaled_layer(TINY, m=80, n=2048, n_tok=4096)
    qs = synth.QuantSetting(4, 128, False, 0.01, True)
    gpu = GH.run_path(layer, qs)
    prep = O.prepare(gpu["H"], qs.damp, qs.desc_act)
    st, rep = GH.check_sweep_replay(gpu["W"], prep, gpu, qs)
    GH.assert_replay_ok(st, rep, gpu)


def test_quantize_before_and_after_the_factor_is_completed():
    """Quantizing needs only the diagonal super-blocks of U; completing U for gptq_get_factor
    changes no output, whichever form the update past a super-block takes."""
    layer = synth.scaled_layer(TINY, m=72, n=2304, n_tok=4608)
    X, W = synth.make_x_bf16(layer), synth.make_w_fp16(layer)
    Wd = torch.from_numpy(W).to(GH.DEV)
    for qs in (synth.QuantSetting(4, 128, False, 0.01, True), synth.QuantSetting(3, 384, True, 0.01, True)):
        with GPTQContext(layer.n, layer.m, 0) as ctx:
            ctx.accumulate_hessian(GH.bf16_to_dev(X))
            H, _ = ctx.get_hessian()
            ctx.prepare(qs.damp, qs.desc_act)
            a = ctx.quantize_layer(Wd, qs.bits, qs.group_size, qs.sym)
            a = {k: v.clone() for k, v in a.items() if v is not None}
            U = ctx.get_factor().cpu().numpy().astype(np.float64)
            b = ctx.quantize_layer(Wd, qs.bits, qs.group_size, qs.sym)
            ctx.synchronize()
        for k in a:
            assert torch.equal(a[k], b[k]), k
        prep = O.prepare(H.cpu().numpy().astype(np.float64), qs.damp, qs.desc_act)
        assert np.abs(U - prep["U"]).max() / np.abs(prep["U"]).max() <= 2e-5
        gpu = {"codes": O.unpack_codes(a["codes"].cpu().numpy().view(np.uint32), layer.n, qs.bits),
               "scales": a["scales"].cpu().numpy(), "zeros": a["zeros"].cpu().numpy()}
        st, rep = GH.check_sweep_replay(W, prep, gpu, qs)
        GH.assert_replay_ok(st, rep, gpu)
