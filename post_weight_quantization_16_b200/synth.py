"""Seeded synthetic inputs for GPTQ's per-layer solve.

This module only draws random numbers and rounds them to the storage types the
path consumes (bf16 calibration activations X, fp16 weights W).  It holds none of
the method's arithmetic, so both the CUDA path and the CPU oracle can be fed from it
without sharing any code of the method.

Recipe (one per workload; all draws are fp32 from numpy's PCG64, then rounded to
nearest-even into bf16 / fp16):

* X is drawn in fixed chunks of ``CHUNK`` tokens; chunk ``c`` of the X stream for
  seed ``s`` uses ``SeedSequence([s, 0, c])``.  Any token range can therefore be
  regenerated on its own, and host memory stays bounded for large N.
* Outlier channels (the "1 % of channels x20" of the workloads) are chosen without
  replacement from ``SeedSequence([s, 2])``; their fp32 draws are multiplied by the
  outlier factor before rounding.
* W comes from ``SeedSequence([s, 1])``.

The calibration sets of the pages (WikiText-2 / C4 / Alpaca samples pushed through
Llama-2 / Qwen layers) are not available; these draws stand in for them with the
same layer shapes.
"""
from __future__ import annotations

import dataclasses
import numpy as np

CHUNK = 8192  # tokens per independently seeded X chunk


# ----------------------------------------------------------------------------------
# storage-type rounding
# ----------------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even); return the raw uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    u = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Layer:
    """One synthetic linear layer plus its calibration activations."""
    name: str
    m: int                      # out features (rows of W)
    n: int                      # in features (columns of W, channels of X)
    n_tok: int                  # calibration tokens (rows of X)
    w_dist: str                 # "normal" | "student_t3"
    w_sigma: float
    x_dist: str                 # "normal" | "relu_like"
    n_outliers: int             # outlier channels of X
    outlier_scale: float
    x_seed: int
    w_seed: int


@dataclasses.dataclass(frozen=True)
class QuantSetting:
    bits: int
    group_size: int             # -1 = one group per row (per-channel)
    sym: bool
    damp: float
    desc_act: bool


def _outlier_count(n: int, frac: float) -> int:
    return int(round(frac * n))


WORKLOADS = {
    # tiny single layer: 256x512, N=2048, 1 % outlier channels x20
    "tiny_256x512": (Layer("tiny_256x512", 256, 512, 2048, "normal", 0.02, "normal",
                           _outlier_count(512, 0.01), 20.0, 0, 0),
                     QuantSetting(4, 128, False, 0.01, False)),
    # Llama-7B-shaped q_proj: 4096x4096, N=262144 (128 x 2048), 0.5 % outlier channels x30
    "q_proj_4096x4096": (Layer("q_proj_4096x4096", 4096, 4096, 262144, "normal", 0.02, "normal",
                               _outlier_count(4096, 0.005), 30.0, 0, 0),
                         QuantSetting(4, 128, False, 0.01, True)),
    # MLP down_proj: 4096x11008, heavy-tailed W, ReLU-like X
    "down_proj_4096x11008": (Layer("down_proj_4096x11008", 4096, 11008, 131072, "student_t3", 0.01,
                                   "relu_like", 0, 1.0, 0, 0),
                             QuantSetting(4, 128, True, 0.01, True)),
    # 70B-shaped down_proj: 8192x28672, N=65536, 1 % outlier channels x20
    "down_proj_8192x28672": (Layer("down_proj_8192x28672", 8192, 28672, 65536, "normal", 0.01, "normal",
                                   _outlier_count(28672, 0.01), 20.0, 0, 0),
                             QuantSetting(4, 128, False, 0.01, True)),
}


def block7b_layers():
    """The 7B-shaped block: seven independent layers, N=65536 each, 1 % outliers x20.

    Layer k uses seed k for X and 1000+k for W.
    """
    shapes = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
              ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
    out = []
    for k, (nm, m, n) in enumerate(shapes):
        out.append(Layer(f"block7b_{nm}", m, n, 65536, "normal", 0.02, "normal",
                         _outlier_count(n, 0.01), 20.0, k, 1000 + k))
    return out


def _register_block7b():
    """Name each 7B-block layer as a workload too (4-bit, asymmetric, group 128, damp 0.01, act-order)."""
    for lay in block7b_layers():
        WORKLOADS[f"{lay.name}_{lay.m}x{lay.n}"] = (lay, QuantSetting(4, 128, False, 0.01, True))


_register_block7b()


def block7b_settings():
    """bits x group_size x damp grid of the 7B block sweep (desc_act on)."""
    out = []
    for bits in (2, 3, 4):
        for g in (64, 128, -1):
            for damp in (0.01, 0.1):
                out.append(QuantSetting(bits, g, False, damp, True))
    return out


# ----------------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------------
def outlier_channels(layer: Layer) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([layer.x_seed, 2])))
    return np.sort(rng.choice(layer.n, size=layer.n_outliers, replace=False)) if layer.n_outliers else \
        np.zeros(0, dtype=np.int64)


def _x_chunk_f32(layer: Layer, c: int, channel_scale: np.ndarray) -> np.ndarray:
    rows = min(CHUNK, layer.n_tok - c * CHUNK)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([layer.x_seed, 0, c])))
    if layer.x_dist == "normal":
        a = rng.standard_normal((rows, layer.n), dtype=np.float32)
    elif layer.x_dist == "relu_like":
        # product of an independent half-normal and a standard normal draw
        a = np.abs(rng.standard_normal((rows, layer.n), dtype=np.float32))
        a *= rng.standard_normal((rows, layer.n), dtype=np.float32)
    else:
        raise ValueError(layer.x_dist)
    if channel_scale is not None:
        a *= channel_scale[None, :]
    return a


def _channel_scale(layer: Layer):
    if layer.n_outliers == 0:
        return None
    s = np.ones(layer.n, dtype=np.float32)
    s[outlier_channels(layer)] = np.float32(layer.outlier_scale)
    return s


def make_x_bf16(layer: Layer, t0: int = 0, t1: int | None = None, out: np.ndarray | None = None) -> np.ndarray:
    """Tokens [t0, t1) of the layer's calibration activations as bf16 bits, shape [t1-t0, n]."""
    t1 = layer.n_tok if t1 is None else t1
    assert 0 <= t0 <= t1 <= layer.n_tok
    if out is None:
        out = np.empty((t1 - t0, layer.n), dtype=np.uint16)
    cs = _channel_scale(layer)
    c0, c1 = t0 // CHUNK, (t1 + CHUNK - 1) // CHUNK
    for c in range(c0, c1):
        a = _x_chunk_f32(layer, c, cs)
        base = c * CHUNK
        lo, hi = max(t0, base), min(t1, base + a.shape[0])
        out[lo - t0:hi - t0] = f32_to_bf16_bits(a[lo - base:hi - base])
    return out


def iter_x_bf16(layer: Layer, batch_tokens: int):
    """Yield the calibration set in batches of ``batch_tokens`` rows (bf16 bits)."""
    for t0 in range(0, layer.n_tok, batch_tokens):
        yield make_x_bf16(layer, t0, min(layer.n_tok, t0 + batch_tokens))


def make_w_fp16(layer: Layer) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([layer.w_seed, 1])))
    if layer.w_dist == "normal":
        a = rng.standard_normal((layer.m, layer.n), dtype=np.float32) * np.float32(layer.w_sigma)
    elif layer.w_dist == "student_t3":
        a = rng.standard_t(3, size=(layer.m, layer.n)).astype(np.float32) * np.float32(layer.w_sigma)
    else:
        raise ValueError(layer.w_dist)
    return a.astype(np.float16)


def scaled_layer(layer: Layer, m: int | None = None, n: int | None = None, n_tok: int | None = None,
                 name: str | None = None) -> Layer:
    """Same recipe at another size (for parity cases the oracle finishes in seconds)."""
    n2 = layer.n if n is None else n
    frac = layer.n_outliers / layer.n
    return dataclasses.replace(layer, name=name or f"{layer.name}_scaled",
                               m=layer.m if m is None else m, n=n2,
                               n_tok=layer.n_tok if n_tok is None else n_tok,
                               n_outliers=_outlier_count(n2, frac) if layer.n_outliers else 0)
