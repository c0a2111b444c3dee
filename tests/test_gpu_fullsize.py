"""Full-size parity on the workload the benchmark times (q_proj 4096 x 4096, 262144 tokens),
in the same launch configuration: H on the full diagonal plus sampled off-diagonal entries
(each an exact float64 dot product over all tokens), the permutation and factor against the
oracle run on the GPU's H, the sweep replayed on sampled rows, and the layer error of the
whole layer against the oracle's own run."""
import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import synth
from post_weight_quantization_16_b200.gptq import GPTQContext
from tests import gpu_helpers as GH

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _sampled_hessian(X_bits, pairs, chunk=16384):
    n = X_bits.shape[1]
    diag = np.zeros(n)
    off = np.zeros(len(pairs))
    I, J = pairs[:, 0], pairs[:, 1]
    for t0 in range(0, X_bits.shape[0], chunk):
        x = synth.bf16_bits_to_f32(X_bits[t0:t0 + chunk]).astype(np.float64)
        diag += np.einsum("ti,ti->i", x, x)
        off += np.einsum("ti,ti->i", x[:, I], x[:, J])
    return 2.0 * diag, 2.0 * off


def test_q_proj_full_size():
    layer, qs = synth.WORKLOADS["q_proj_4096x4096"]
    X = synth.make_x_bf16(layer)
    W = synth.make_w_fp16(layer)
    with GPTQContext(layer.n, layer.m, 0) as ctx:
        Xd = GH.bf16_to_dev(X)
        ctx.accumulate_hessian(Xd)
        del Xd
        H, nt = ctx.get_hessian()
        perm = ctx.prepare(qs.damp, qs.desc_act).cpu().numpy()
        U = ctx.get_factor().cpu().numpy().astype(np.float64)
        out = ctx.quantize_layer(torch.from_numpy(W).to(GH.DEV), qs.bits, qs.group_size, bool(qs.sym))
        ctx.synchronize()
        gpu = {"codes": O.unpack_codes(out["codes"].cpu().numpy().view(np.uint32), layer.n, qs.bits),
               "scales": out["scales"].cpu().numpy(), "zeros": out["zeros"].cpu().numpy(),
               "w_hat": out["w_hat"].cpu().numpy().astype(np.float64), "g_idx": out["g_idx"].cpu().numpy()}
    H = H.cpu().numpy().astype(np.float64)
    assert nt == layer.n_tok

    # S1: the full diagonal and 2048 sampled off-diagonal entries, exact in float64
    rng = np.random.default_rng(123)
    pairs = rng.integers(0, layer.n, size=(2048, 2))
    pairs = pairs[pairs[:, 0] != pairs[:, 1]]
    d_ref, o_ref = _sampled_hessian(X, pairs)
    d_gpu, o_gpu = np.diag(H), H[pairs[:, 0], pairs[:, 1]]
    n_off = layer.n * (layer.n - 1)
    num = np.sum((d_gpu - d_ref) ** 2) + n_off / len(pairs) * np.sum((o_gpu - o_ref) ** 2)
    den = np.sum(d_ref ** 2) + n_off / len(pairs) * np.sum(o_ref ** 2)
    rel_fro = np.sqrt(num / den)
    assert rel_fro <= GH.H_REL_FRO, rel_fro
    assert np.max(np.abs(d_gpu - d_ref) / d_ref) <= 2e-5

    # S2-S4 against the oracle on the GPU's H
    prep = O.prepare(H, qs.damp, qs.desc_act)
    assert np.array_equal(perm, prep["perm"])
    err = np.abs(U - prep["U"]).max() / np.abs(prep["U"]).max()
    assert err <= 2e-5, err

    # S5-S7: replay on 256 sampled rows
    rows = np.sort(rng.choice(layer.m, 256, replace=False))
    st, rep = GH.check_sweep_replay(W, prep, gpu, qs, rows=rows)
    GH.assert_replay_ok(st, rep, gpu, rows=rows)
    assert np.array_equal(gpu["g_idx"], O.g_idx(prep["perm"], qs.group_size))

    # layer error of the whole layer vs the oracle's own run (both measured with the GPU's H)
    own = O.quantize_layer(W.astype(np.float64), H, qs.bits, qs.group_size, bool(qs.sym), qs.damp, qs.desc_act,
                           prep=prep)
    e_gpu = O.layer_error(W, gpu["w_hat"], H)
    e_own = O.layer_error(W, own["what_orig"], H)
    assert abs(e_gpu - e_own) <= GH.LAYER_ERR_REL * e_own, (e_gpu, e_own)
