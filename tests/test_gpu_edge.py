"""Degenerate inputs of the path on the GPU, against the oracle: an empty calibration batch
between two real ones, a single-row layer, and a layer with no calibration tokens at all
(every column dead: zero weights, codes at the zero-point)."""
import numpy as np
import pytest

from oracle import gptq_oracle as O
from post_weight_quantization_16_b200 import synth

from tests import gpu_helpers as GH

pytestmark = pytest.mark.gpu
TINY = synth.WORKLOADS["tiny_256x512"][0]


def test_empty_batch_and_single_row():
    layer = synth.scaled_layer(TINY, m=1, n=256, n_tok=500)
    qs = synth.QuantSetting(4, 128, False, 0.01, True)
    gpu = GH.run_path(layer, qs, batches=[300, 0, 200])
    assert gpu["n_tok"] == 500
    Href = O.hessian(synth.bf16_bits_to_f32(gpu["X"]))
    assert np.linalg.norm(gpu["H"] - Href) / np.linalg.norm(Href) <= GH.H_REL_FRO
    prep = O.prepare(gpu["H"], qs.damp, qs.desc_act)
    assert np.array_equal(gpu["perm"], prep["perm"])
    st, rep = GH.check_sweep_replay(gpu["W"], prep, gpu, qs)
    GH.assert_replay_ok(st, rep, gpu)


@pytest.mark.parametrize("sym", [False, True])
def test_no_calibration_tokens(sym):
    layer = synth.scaled_layer(TINY, m=16, n=256, n_tok=64)
    qs = synth.QuantSetting(4, 128, sym, 0.01, True)
    gpu = GH.run_path(layer, qs, batches=[0])  # nothing accumulated: H = 0
    assert gpu["n_tok"] == 0 and not gpu["H"].any()
    prep = O.prepare(gpu["H"], qs.damp, qs.desc_act)
    assert prep["dead"].all()
    assert np.array_equal(gpu["perm"], prep["perm"])  # all diagonals tie: the identity
    assert not gpu["w_hat"].any()
    st, rep = GH.check_sweep_replay(gpu["W"], prep, gpu, qs)
    GH.assert_replay_ok(st, rep, gpu)
