"""Full-width parity on the benchmarked layer shapes, in the launch configuration the
benchmark uses.  The oracle cannot recompute whole layers of this size in seconds, so each
check takes what it can compute one by one or what holds at any size:

* H: the full diagonal plus sampled off-diagonal entries, each an exact float64 dot product
  over every calibration token (the tokens are streamed batch by batch into both sides);
* perm and the dead columns: the oracle's order on the GPU's H, exactly;
* U: against the oracle's factor of the GPU's H, whole (widths up to 11008) or, at 28672, its
  trailing and leading 1024 x 1024 blocks (exact identities of the factor) and random probes
  of U^T U Hd v = v;
* the sweep: replayed by the oracle on sampled rows (stage-isolated: on the GPU's H; at 28672
  on the GPU's factor, checked above), with the layer error of those rows against the
  oracle's own run on them."""
import time

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import synth
from post_weight_quantization_16_b200.gptq import GPTQContext
from tests import gpu_helpers as GH

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

BATCH = 16384  # calibration tokens per accumulate call (a multiple of the generator's chunk)


def _accumulate_and_sample(ctx, layer, pairs):
    """Stream X into the context batch by batch; meanwhile form the exact diagonal and the
    sampled entries of 2 X^T X in float64 on the host from the same bf16 values."""
    n = layer.n
    diag = np.zeros(n)
    off = np.zeros(len(pairs))
    I, J = pairs[:, 0], pairs[:, 1]
    for t0 in range(0, layer.n_tok, BATCH):
        xb = synth.make_x_bf16(layer, t0, min(layer.n_tok, t0 + BATCH))
        ctx.accumulate_hessian(GH.bf16_to_dev(xb))
        for c0 in range(0, xb.shape[0], 4096):
            x = synth.bf16_bits_to_f32(xb[c0:c0 + 4096]).astype(np.float64)
            diag += np.einsum("ti,ti->i", x, x)
            off += np.einsum("ti,ti->i", x[:, I], x[:, J])
        torch.cuda.current_stream(GH.DEV).synchronize()   # the batch's device copy may be freed
    return 2.0 * diag, 2.0 * off


def _check_sampled_hessian(H, pairs, d_ref, o_ref):
    n = H.shape[0]
    d_gpu, o_gpu = np.diag(H), H[pairs[:, 0], pairs[:, 1]]
    n_off = n * (n - 1)
    num = np.sum((d_gpu - d_ref) ** 2) + n_off / len(pairs) * np.sum((o_gpu - o_ref) ** 2)
    den = np.sum(d_ref ** 2) + n_off / len(pairs) * np.sum(o_ref ** 2)
    rel_fro = np.sqrt(num / den)
    assert rel_fro <= GH.H_REL_FRO, rel_fro
    assert np.max(np.abs(d_gpu - d_ref) / d_ref) <= 2e-5


def _u_probe_residual(U, Hd, rng, probes=8):
    """max over random v of |U Hd U^T v - v| / |v| (float64, O(n^2) per probe).  U Hd U^T = I
    exactly (U = V^-1 with Hd = V V^T), and this form amplifies an error of U by about the
    condition number of U, the square root of that of Hd."""
    worst = 0.0
    for _ in range(probes):
        v = rng.standard_normal(Hd.shape[0])
        r = U @ (Hd @ (U.T @ v)) - v
        worst = max(worst, np.linalg.norm(r) / np.linalg.norm(v))
    return worst


def _gpu_layer(layer, settings, seed=123, n_pairs=2048, full_factor=True, rows=256):
    """Run one layer through the C ABI for each quant setting; check S1-S4 once per damp and
    S5-S7 per setting on sampled rows."""
    rng = np.random.default_rng(seed)
    W = synth.make_w_fp16(layer)
    Wd = torch.from_numpy(W).to(GH.DEV)
    pairs = rng.integers(0, layer.n, size=(n_pairs, 2))
    pairs = pairs[pairs[:, 0] != pairs[:, 1]]
    sample = np.sort(rng.choice(layer.m, min(rows, layer.m), replace=False))
    with GPTQContext(layer.n, layer.m, 0) as ctx:
        t0 = time.perf_counter()
        d_ref, o_ref = _accumulate_and_sample(ctx, layer, pairs)
        print(f"[{layer.name}] X streamed and sampled {time.perf_counter() - t0:.1f} s", flush=True)
        Ht, nt = ctx.get_hessian()
        H = Ht.cpu().numpy().astype(np.float64)
        del Ht
        assert nt == layer.n_tok
        _check_sampled_hessian(H, pairs, d_ref, o_ref)
        preps = {}
        current = None
        for qs in settings:
            key = (qs.damp, qs.desc_act)
            if key != current and key in preps:   # the context holds another damp's factor: redo it
                ctx.prepare(qs.damp, qs.desc_act)
                current = key
            if key not in preps:
                current = key
                t0 = time.perf_counter()
                perm = ctx.prepare(qs.damp, qs.desc_act).cpu().numpy()
                dead = ctx.get_dead_columns().cpu().numpy().astype(bool)
                Ut = ctx.get_factor()
                U = Ut.cpu().numpy().astype(np.float64)
                del Ut
                po = O.prepare_order(H, qs.damp, qs.desc_act)
                assert np.array_equal(perm, po["perm"])
                assert np.array_equal(dead, po["dead"])
                assert np.allclose(np.tril(U, -1), 0)
                if full_factor:
                    Uo = O.upper_cholesky_of_inverse(po["Hd"])
                    err = np.abs(U - Uo).max() / np.abs(Uo).max()
                    assert err <= 2e-5, err
                    uref = Uo
                else:
                    k = 1024
                    for blk, ref in ((U[-k:, -k:], O.upper_cholesky_of_inverse_trailing(po["Hd"], k)),
                                     (U[:k, :k], O.upper_cholesky_of_inverse_leading(po["Hd"], k))):
                        err = np.abs(blk - ref).max() / np.abs(ref).max()
                        assert err <= 2e-5, err
                    uref = U   # the sweep replays on the GPU's factor, checked above
                res = _u_probe_residual(U, po["Hd"], rng)
                assert res <= 1e-3, res
                print(f"[{layer.name}] prepare and factor checks {time.perf_counter() - t0:.1f} s", flush=True)
                preps[key] = {"perm": perm, "dead": dead, "U": uref, "Hd": None}
                del U
            prep = preps[key]
            t0 = time.perf_counter()
            out = ctx.quantize_layer(Wd, qs.bits, qs.group_size, bool(qs.sym))
            ctx.synchronize()
            gpu = {"codes": O.unpack_codes(out["codes"][sample].cpu().numpy().view(np.uint32), layer.n, qs.bits),
                   "scales": out["scales"][sample].cpu().numpy(), "zeros": out["zeros"][sample].cpu().numpy()}
            what = out["w_hat"][sample].cpu().numpy().astype(np.float64)
            g_idx = out["g_idx"].cpu().numpy()
            del out
            st, rep = GH.check_sweep_replay(W[sample], prep, gpu, qs)
            GH.assert_replay_ok(st, rep, gpu)
            assert np.array_equal(g_idx, O.g_idx(prep["perm"], qs.group_size))
            # layer error of the sampled rows against the oracle's own (un-replayed) run on them
            Wf = W[sample].astype(np.float64)
            Wz = Wf.copy()
            Wz[:, prep["dead"]] = 0.0
            own = O.gptq_sweep(Wz[:, prep["perm"]], prep["U"], qs.bits, qs.group_size, bool(qs.sym), block=128)
            own_what = O.unpermute_columns(own["what"], prep["perm"])
            e_gpu = O.layer_error(Wf, what, H)
            e_own = O.layer_error(Wf, own_what, H)
            assert abs(e_gpu - e_own) <= GH.LAYER_ERR_REL * e_own, (qs, e_gpu, e_own)
            print(f"[{layer.name}] {qs} sweep checks {time.perf_counter() - t0:.1f} s", flush=True)


def test_q_proj_full_size():
    layer, qs = synth.WORKLOADS["q_proj_4096x4096"]
    _gpu_layer(layer, [qs])


def test_down_proj_4096x11008_sym_heavy_tails():
    """Student-t(3) weights, |A| B activations, 4-bit symmetric, act-order."""
    layer, qs = synth.WORKLOADS["down_proj_4096x11008"]
    _gpu_layer(layer, [qs])


def test_down_proj_8192x28672():
    """The 70B-shaped layer the benchmark times: 224 diagonal blocks, 28 super-blocks."""
    layer, qs = synth.WORKLOADS["down_proj_8192x28672"]
    _gpu_layer(layer, [qs], full_factor=False, rows=128)


# a spread of the 7B block's bits x group_size x damp grid: every bits, group and damp value
# appears on each width
BLOCK_SPREAD_4096 = [(2, 64, 0.01), (3, -1, 0.1), (4, 128, 0.01), (2, 128, 0.1), (3, 64, 0.01), (4, -1, 0.1)]
BLOCK_SPREAD_11008 = [(4, 64, 0.1), (2, -1, 0.01), (3, 128, 0.1), (4, 128, 0.01)]


def _block_layer(name):
    return next(l for l in synth.block7b_layers() if l.name == name)


def test_block7b_q_4096_settings():
    layer = _block_layer("block7b_q")
    _gpu_layer(layer, [synth.QuantSetting(b, g, False, d, True) for b, g, d in BLOCK_SPREAD_4096], rows=128)


def test_block7b_down_11008_settings():
    layer = _block_layer("block7b_down")
    _gpu_layer(layer, [synth.QuantSetting(b, g, False, d, True) for b, g, d in BLOCK_SPREAD_11008], rows=96)


def test_block7b_gate_11008_rows():
    """11008 output rows (344 row tiles of the sweep) on a 4096-wide input."""
    layer = _block_layer("block7b_gate")
    _gpu_layer(layer, [synth.QuantSetting(3, 128, False, 0.01, True), synth.QuantSetting(4, 64, False, 0.1, True)],
               rows=128)
