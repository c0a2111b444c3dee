"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI on seeded
inputs, bring the results back, and compare them with the oracle."""
from __future__ import annotations

import numpy as np
import torch

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import synth
from post_weight_quantization_16_b200.gptq import GPTQContext

DEV = torch.device("cuda", 0)

# tolerances (the parity bar for this path)
H_REL_FRO = 1e-5        # Hessian, relative Frobenius
SZ_REL = 1e-5           # scales / zeros, relative
CODES_IDENTICAL = 0.999 # fraction of identical codes
BAND = 1e-3             # replay band around rounding boundaries (code units)
LAYER_ERR_REL = 0.01    # relative layer error vs the oracle's own run


def bf16_to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def run_path(layer, qs, X_bits=None, batches=None, chunk=None, W=None, ctx_m=None):
    """Full hot path on the GPU: returns numpy copies of every output."""
    X_bits = synth.make_x_bf16(layer) if X_bits is None else X_bits
    W = synth.make_w_fp16(layer) if W is None else W
    with GPTQContext(layer.n, ctx_m or layer.m, 0) as ctx:
        if chunk:
            ctx.set_hessian_chunk(chunk)
        if batches is None:
            ctx.accumulate_hessian(bf16_to_dev(X_bits))
        else:
            t0 = 0
            for b in batches:
                ctx.accumulate_hessian(bf16_to_dev(X_bits[t0:t0 + b]))
                t0 += b
        H, nt = ctx.get_hessian()
        perm = ctx.prepare(qs.damp, qs.desc_act)
        U = ctx.get_factor()
        out = ctx.quantize_layer(torch.from_numpy(W).to(DEV), qs.bits, qs.group_size, bool(qs.sym))
        ctx.synchronize()
        res = {"H": H.cpu().numpy().astype(np.float64), "n_tok": nt, "perm": perm.cpu().numpy(),
               "U": U.cpu().numpy().astype(np.float64), "packed": out["codes"].cpu().numpy().view(np.uint32),
               "scales": out["scales"].cpu().numpy(), "zeros": out["zeros"].cpu().numpy(),
               "g_idx": out["g_idx"].cpu().numpy(), "w_hat": out["w_hat"].cpu().numpy().astype(np.float64)}
    res["codes"] = O.unpack_codes(res["packed"], layer.n, qs.bits)
    res["W"] = W
    res["X"] = X_bits
    return res


def check_sweep_replay(W, prep, gpu, qs, rows=None):
    """Stage-isolated replay of the sweep (the oracle runs on the GPU's H) on all or some rows.
    Returns (stats, replayed oracle output)."""
    Wf = np.asarray(W, dtype=np.float64).copy()
    Wf[:, prep["dead"]] = 0.0
    Wp = Wf[:, prep["perm"]]
    codes, zeros = gpu["codes"], gpu["zeros"]
    if rows is not None:
        Wp, codes, zeros = Wp[rows], codes[rows], zeros[rows]
    st = O.ReplayStats()
    rep = O.gptq_sweep(Wp, prep["U"], qs.bits, qs.group_size, bool(qs.sym), block=128, ref_codes=codes,
                       ref_zeros=zeros, band=BAND, stats=st)
    return st, rep


def assert_replay_ok(st, rep, gpu, rows=None):
    sc = gpu["scales"] if rows is None else gpu["scales"][rows]
    ze = gpu["zeros"] if rows is None else gpu["zeros"][rows]
    assert st.hard_mismatch == 0, st.as_dict()
    assert st.zero_hard_mismatch == 0, st.as_dict()
    assert st.identical >= CODES_IDENTICAL * st.total, st.as_dict()
    rel = np.abs(sc.astype(np.float64) - rep["scales"]) / np.abs(rep["scales"].astype(np.float64))
    assert rel.max() <= SZ_REL, rel.max()
    assert np.array_equal(ze, rep["zeros"])
