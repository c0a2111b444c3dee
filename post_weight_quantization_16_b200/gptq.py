"""Python binding of libgptq (ctypes).  Argument marshalling only: every step of the
solve runs in the library's CUDA kernels; PyTorch provides device memory and the stream.

The object mirrors the three-call lifecycle of the GPTQ quantizer on the page
"模型量化实战：从 INT8 PTQ 到 GPTQ 的精度保持与推理加速全解析" (§3.2: accumulate the Hessian
over calibration batches, prepare the inverse factor, quantize the layer), with the
quantizer settings named as in AutoGPTQ's quantize_config ("GPTQ算法原理深度解析" §3.3).
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgptq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "gptq.h")
HEADERS = [HEADER, os.path.join(os.path.dirname(HERE), "include", "gptq_testing.h")]

STATUS = {0: "GPTQ_OK", 1: "GPTQ_ERR_ARG", 2: "GPTQ_ERR_STATE", 3: "GPTQ_ERR_NOT_PD", 4: "GPTQ_ERR_OOM",
          5: "GPTQ_ERR_CUDA", 6: "GPTQ_ERR_TIMEOUT", 7: "GPTQ_ERR_UNSUPPORTED"}
OK, ERR_ARG, ERR_STATE, ERR_NOT_PD, ERR_OOM, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED = range(8)


class GPTQError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{call}: {self.name} ({lib().gptq_status_string(status).decode()})")


class QParams(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group_size", ctypes.c_int), ("sym", ctypes.c_int)]


class LayerJob(ctypes.Structure):
    _fields_ = [("X_bf16", ctypes.c_void_p), ("n_tok", ctypes.c_int64), ("ld_x", ctypes.c_int64),
                ("W_fp16", ctypes.c_void_p), ("m", ctypes.c_int64), ("n", ctypes.c_int64), ("qp", QParams),
                ("damp", ctypes.c_double), ("desc_act", ctypes.c_int), ("codes_out", ctypes.c_void_p),
                ("scales_out", ctypes.c_void_p), ("zeros_out", ctypes.c_void_p), ("g_idx_out", ctypes.c_void_p),
                ("perm_out", ctypes.c_void_p), ("W_hat_out", ctypes.c_void_p)]


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 40), ("launches", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


_LIB = None
_P = ctypes.c_void_p
_SIGS = {
    "gptq_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "gptq_create": (ctypes.c_int, [ctypes.POINTER(_P), ctypes.c_int64, ctypes.c_int64, ctypes.c_int, _P]),
    "gptq_hessian_accumulate": (ctypes.c_int, [_P, _P, ctypes.c_int64, ctypes.c_int64]),
    "gptq_get_hessian": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int64)]),
    "gptq_set_hessian": (ctypes.c_int, [_P, _P, ctypes.c_int64]),
    "gptq_prepare": (ctypes.c_int, [_P, ctypes.c_double, ctypes.c_int, _P]),
    "gptq_get_factor": (ctypes.c_int, [_P, _P]),
    "gptq_quantize_layer": (ctypes.c_int, [_P, _P, ctypes.c_int64, QParams, _P, _P, _P, _P, _P]),
    "gptq_synchronize": (ctypes.c_int, [_P]),
    "gptq_reset": (ctypes.c_int, [_P]),
    "gptq_destroy": (ctypes.c_int, [_P]),
    "gptq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "gptq_set_hessian_chunk": (ctypes.c_int, [_P, ctypes.c_int64]),
    "gptq_launch_count": (ctypes.c_int64, [_P]),
    "gptq_get_dead_columns": (ctypes.c_int, [_P, _P]),
    "gptq_set_profiling": (ctypes.c_int, [_P, ctypes.c_int]),
    "gptq_get_profile": (ctypes.c_int, [_P, ctypes.POINTER(KernelStat), ctypes.c_int, ctypes.POINTER(ctypes.c_int)]),
    "gptq_test_bounded_wait": (ctypes.c_int, [_P, ctypes.c_uint64]),
    "gptq_dequant_matmul_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                              ctypes.c_int]),
    "gptq_dequant_matmul": (ctypes.c_int, [_P, ctypes.c_int64, _P, _P, _P, _P, ctypes.c_int64, ctypes.c_int64,
                                           QParams, _P, _P, ctypes.c_size_t, ctypes.c_int, _P]),
    "gptq_dequant_matmul_check": (ctypes.c_int, [_P, ctypes.c_int, _P]),
    "gptq_quantize_layers": (ctypes.c_int, [ctypes.POINTER(LayerJob), ctypes.c_int, ctypes.c_int, _P]),
    "gptq_pipeline_create": (ctypes.c_int, [ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_int64),
                                            ctypes.POINTER(ctypes.c_int64), ctypes.c_int, ctypes.c_int, _P]),
    "gptq_pipeline_run": (ctypes.c_int, [_P, ctypes.POINTER(LayerJob), ctypes.c_int]),
    "gptq_pipeline_destroy": (ctypes.c_int, [_P]),
    "gptq_activation_convert": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, _P, _P, ctypes.c_int,
                                               _P]),
    "gptq_awq_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64]),
    "gptq_awq_quantize": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int64, _P, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_float, QParams, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                         ctypes.c_int, _P]),
    "gptq_rtn_quantize": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int64, QParams, ctypes.c_float, _P, _P, _P, _P,
                                         _P, ctypes.c_int, _P]),
    "gptq_quantize_layer_noalloc": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int64, _P, _P, _P, QParams,
                                                   _P, _P, _P, _P, _P, ctypes.c_int, _P]),
    "gptq_test_gemm_tf32x3": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, ctypes.c_int, _P, _P,
                                             ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, _P, ctypes.c_int, _P, _P, ctypes.c_int, _P, _P,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             _P]),
    "gptq_test_div_rn": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_int64, ctypes.POINTER(ctypes.c_uint64),
                                        ctypes.POINTER(ctypes.c_float), ctypes.c_int, _P]),
    "gptq_test_pick_tile_n": (ctypes.c_int, [ctypes.c_int] * 7),
    "gptq_test_tile_schedule": (ctypes.c_int, [ctypes.c_int] * 8),
    "gptq_test_factor_plan": (ctypes.c_int, [ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                             ctypes.POINTER(ctypes.c_int)]),
    "gptq_test_pct_position": (ctypes.c_int, [ctypes.c_double, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                              ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float),
                                              ctypes.POINTER(ctypes.c_float)]),
}


def lib():
    """Load libgptq.so (built in-tree).  Fails loudly when it is missing: there is no fallback."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgptq.so is not built ({LIB_PATH}); run "
                               "`python -m post_weight_quantization_16_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def header_functions():
    """Names of the functions the headers under include/ declare."""
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(gptq_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def _check(status: int, call: str):
    if status != OK:
        raise GPTQError(status, call)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class GPTQContext:
    """One layer width n: accumulate H over calibration batches, prepare, quantize layers."""

    def __init__(self, n: int, m_max: int, device: int | torch.device = 0, stream: torch.cuda.Stream | None = None):
        self.device = torch.device("cuda", device if isinstance(device, int) else device.index)
        self.n, self.m_max = int(n), int(m_max)
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        h = ctypes.c_void_p()
        _check(lib().gptq_create(ctypes.byref(h), self.n, self.m_max, self.device.index,
                                 ctypes.c_void_p(self.stream.cuda_stream)), "gptq_create")
        self._h = h

    # -- lifecycle ---------------------------------------------------------------------------
    def close(self):
        if getattr(self, "_h", None):
            st = lib().gptq_destroy(self._h)
            self._h = None
            _check(st, "gptq_destroy")

    def __del__(self):
        try:
            if getattr(self, "_h", None):
                lib().gptq_destroy(self._h)
                self._h = None
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    # -- S1 ----------------------------------------------------------------------------------
    def set_hessian_chunk(self, tokens: int):
        _check(lib().gptq_set_hessian_chunk(self._h, int(tokens)), "gptq_set_hessian_chunk")

    def accumulate_hessian(self, X: torch.Tensor):
        """H += 2 X^T X for a bf16 batch X [tokens, n] on the device (row stride may exceed n)."""
        if X.dtype != torch.bfloat16 or X.device != self.device or X.dim() != 2 or X.stride(1) != 1:
            raise ValueError("X must be a bf16 [tokens, n] device tensor with unit column stride")
        _check(lib().gptq_hessian_accumulate(self._h, _ptr(X), X.shape[0], X.stride(0)), "gptq_hessian_accumulate")

    def get_hessian(self):
        H = torch.empty((self.n, self.n), dtype=torch.float32, device=self.device)
        nt = ctypes.c_int64()
        _check(lib().gptq_get_hessian(self._h, _ptr(H), ctypes.byref(nt)), "gptq_get_hessian")
        return H, nt.value

    def set_hessian(self, H: torch.Tensor, n_tok: int):
        if H.dtype != torch.float32 or H.shape != (self.n, self.n) or not H.is_contiguous() or H.device != self.device:
            raise ValueError("H must be a contiguous fp32 [n, n] device tensor")
        _check(lib().gptq_set_hessian(self._h, _ptr(H), int(n_tok)), "gptq_set_hessian")

    # -- S2-S4 -------------------------------------------------------------------------------
    def prepare(self, damp: float = 0.01, desc_act: bool = False) -> torch.Tensor:
        perm = torch.empty(self.n, dtype=torch.int32, device=self.device)
        _check(lib().gptq_prepare(self._h, float(damp), int(bool(desc_act)), _ptr(perm)), "gptq_prepare")
        return perm

    def get_dead_columns(self) -> torch.Tensor:
        """uint8 [n] mask (original column order) of the columns the last prepare found unexcited."""
        d = torch.empty(self.n, dtype=torch.uint8, device=self.device)
        _check(lib().gptq_get_dead_columns(self._h, _ptr(d)), "gptq_get_dead_columns")
        return d

    def get_factor(self) -> torch.Tensor:
        U = torch.empty((self.n, self.n), dtype=torch.float32, device=self.device)
        _check(lib().gptq_get_factor(self._h, _ptr(U)), "gptq_get_factor")
        return U

    # -- S5-S7 -------------------------------------------------------------------------------
    def quantize_layer(self, W: torch.Tensor, bits: int = 4, group_size: int = 128, sym: bool = False,
                       want_w_hat: bool = True, out: dict | None = None) -> dict:
        """Quantize fp16 W [m, n] (original column order).  Returns device tensors
        codes [m, n*bits/32] int32-viewed uint32 words, scales/zeros [m, G], g_idx [n], w_hat [m, n]."""
        if W.dtype != torch.float16 or W.dim() != 2 or W.shape[1] != self.n or not W.is_contiguous() \
                or W.device != self.device:
            raise ValueError("W must be a contiguous fp16 [m, n] device tensor")
        m = W.shape[0]
        g = self.n if group_size == -1 else group_size
        G = self.n // g if g > 0 and self.n % g == 0 else 1
        if out is None:
            out = {
                "codes": torch.empty((m, self.n * bits // 32), dtype=torch.int32, device=self.device),
                "scales": torch.empty((m, G), dtype=torch.float32, device=self.device),
                "zeros": torch.empty((m, G), dtype=torch.float32, device=self.device),
                "g_idx": torch.empty(self.n, dtype=torch.int32, device=self.device),
                "w_hat": torch.empty((m, self.n), dtype=torch.float32, device=self.device) if want_w_hat else None,
            }
        qp = QParams(int(bits), int(group_size), int(bool(sym)))
        _check(lib().gptq_quantize_layer(self._h, _ptr(W), m, qp, _ptr(out["codes"]), _ptr(out["scales"]),
                                         _ptr(out["zeros"]), _ptr(out["g_idx"]), _ptr(out.get("w_hat"))),
               "gptq_quantize_layer")
        return out

    def synchronize(self):
        _check(lib().gptq_synchronize(self._h), "gptq_synchronize")

    # -- instrumentation ---------------------------------------------------------------------
    def set_profiling(self, on: bool):
        _check(lib().gptq_set_profiling(self._h, int(bool(on))), "gptq_set_profiling")

    def get_profile(self) -> dict:
        """{role: {"launches", "ms", "flops", "bytes"}} of the launches recorded since the last call."""
        cap = 64
        arr = (KernelStat * cap)()
        cnt = ctypes.c_int()
        _check(lib().gptq_get_profile(self._h, arr, cap, ctypes.byref(cnt)), "gptq_get_profile")
        return {arr[i].name.decode(): {"launches": int(arr[i].launches), "ms": arr[i].ms, "flops": arr[i].flops,
                                      "bytes": arr[i].bytes} for i in range(min(cap, cnt.value))}

    def launch_count(self) -> int:
        return int(lib().gptq_launch_count(self._h))

    def reset(self):
        _check(lib().gptq_reset(self._h), "gptq_reset")


def allreduce_hessian(ctx, group=None) -> int:
    """Token-split calibration across the ranks of a torch.distributed group: each rank has
    accumulated 2 X^T X over its own share of the tokens ("模型量化实战…" §3.2 accumulate_hessian:
    the Hessian is a sum over tokens, so partial sums add).  The partial H and token counts are
    summed with one all-reduce each (n^2 fp32 on the group's backend: NCCL over NVLink between
    GPUs) and every rank's context continues from the full H.  Returns the total token count.
    Every rank must call it, in the same order as its other collectives."""
    import torch.distributed as dist
    H, nt = ctx.get_hessian()
    dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)
    t = torch.tensor([nt], dtype=torch.int64, device=H.device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    total = int(t.item())
    ctx.set_hessian(H, total)
    return total


def workspace_bytes(n: int, m_max: int) -> int:
    return int(lib().gptq_workspace_bytes(int(n), int(m_max)))


def dequant_matmul(X: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                   perm: torch.Tensor | None, bits: int, group_size: int, out: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Y = X W16^T from the packed result (gptq_dequant_matmul).  X: fp16 [T, n] device tensor in
    original column order; codes/scales/zeros as gptq_quantize_layer wrote them; perm or None.
    Returns fp32 Y [T, m] (asynchronous on `stream`)."""
    if X.dtype != torch.float16 or X.dim() != 2 or not X.is_contiguous():
        raise ValueError("X must be a contiguous fp16 [T, n] device tensor")
    T, n = X.shape
    m = codes.shape[0]
    dev = X.device
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    need = int(lib().gptq_dequant_matmul_workspace_bytes(T, m, n, int(perm is not None)))
    if need == 0:
        raise GPTQError(ERR_ARG, "gptq_dequant_matmul_workspace_bytes")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((T, m), dtype=torch.float32, device=dev)
    qp = QParams(int(bits), int(group_size), 0)
    _check(lib().gptq_dequant_matmul(_ptr(X), T, _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(perm), m, n, qp,
                                     _ptr(out), _ptr(workspace), workspace.numel(), dev.index,
                                     ctypes.c_void_p(stream.cuda_stream)), "gptq_dequant_matmul")
    return out


def _jobs(layers: list, dev: torch.device):
    jobs = (LayerJob * len(layers))()
    outs = []
    for i, L in enumerate(layers):
        X, W = L["X"], L["W"]
        m, n = W.shape
        g = n if L["group_size"] == -1 else L["group_size"]
        o = L.get("out") or {
            "codes": torch.empty((m, n * L["bits"] // 32), dtype=torch.int32, device=dev),
            "scales": torch.empty((m, n // g), dtype=torch.float32, device=dev),
            "zeros": torch.empty((m, n // g), dtype=torch.float32, device=dev),
            "g_idx": torch.empty(n, dtype=torch.int32, device=dev),
            "perm": torch.empty(n, dtype=torch.int32, device=dev),
            "w_hat": torch.empty((m, n), dtype=torch.float32, device=dev) if L.get("want_w_hat") else None}
        outs.append(o)
        j = jobs[i]
        j.X_bf16, j.n_tok, j.ld_x = X.data_ptr(), X.shape[0], X.stride(0)
        j.W_fp16, j.m, j.n = W.data_ptr(), m, n
        j.qp = QParams(int(L["bits"]), int(L["group_size"]), int(bool(L["sym"])))
        j.damp, j.desc_act = float(L["damp"]), int(bool(L["desc_act"]))
        j.codes_out, j.scales_out, j.zeros_out = o["codes"].data_ptr(), o["scales"].data_ptr(), o["zeros"].data_ptr()
        j.g_idx_out, j.perm_out = o["g_idx"].data_ptr(), o["perm"].data_ptr()
        j.W_hat_out = o["w_hat"].data_ptr() if o.get("w_hat") is not None else None
    return jobs, outs


class Pipeline:
    """Contexts kept between batches of layers (gptq_pipeline_*): `widths` maps each input width
    to the largest number of rows its layers have."""

    def __init__(self, widths: dict, device: int = 0, stream: torch.cuda.Stream | None = None):
        self.device = torch.device("cuda", device)
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        ws = (ctypes.c_int64 * len(widths))(*[int(w) for w in widths])
        ms = (ctypes.c_int64 * len(widths))(*[int(m) for m in widths.values()])
        h = ctypes.c_void_p()
        _check(lib().gptq_pipeline_create(ctypes.byref(h), ws, ms, len(widths), self.device.index,
                                          ctypes.c_void_p(self.stream.cuda_stream)), "gptq_pipeline_create")
        self._h = h

    def run(self, layers: list) -> list:
        jobs, outs = _jobs(layers, self.device)
        _check(lib().gptq_pipeline_run(self._h, jobs, len(layers)), "gptq_pipeline_run")
        return outs

    def close(self):
        if getattr(self, "_h", None):
            st = lib().gptq_pipeline_destroy(self._h)
            self._h = None
            _check(st, "gptq_pipeline_destroy")

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()


def quantize_layers(layers: list, device: int = 0, stream: torch.cuda.Stream | None = None) -> list:
    """Quantize many layers in one pipelined call (gptq_quantize_layers).  `layers` is a list of
    dicts with X (bf16 [n_tok, n] device tensor; the same tensor object for layers that share an
    input), W (fp16 [m, n]), bits, group_size, sym, damp, desc_act and optional want_w_hat.
    Returns one dict of device outputs per layer (codes, scales, zeros, g_idx, perm, w_hat)."""
    dev = torch.device("cuda", device)
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    jobs, outs = _jobs(layers, dev)
    _check(lib().gptq_quantize_layers(jobs, len(layers), dev.index, ctypes.c_void_p(stream.cuda_stream)),
           "gptq_quantize_layers")
    return outs


def awq_quantize(X: torch.Tensor | None, W: torch.Tensor, s_protect: float = 2.0, bits: int = 4, group_size: int = 128,
                 sym: bool = False, want_w_hat: bool = True, stream: torch.cuda.Stream | None = None) -> dict:
    """AWQ channel scaling plus round-to-nearest (gptq_awq_quantize).  X: bf16 [n_tok, n] device
    tensor (or None: no calibration tokens), W: fp16 [m, n].  Returns device tensors codes,
    scales, zeros, channel_scale and (optionally) w_hat, all in original column order."""
    m, n = W.shape
    dev = W.device
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    g = n if group_size == -1 else group_size
    out = {"codes": torch.empty((m, n * bits // 32), dtype=torch.int32, device=dev),
           "scales": torch.empty((m, n // g), dtype=torch.float32, device=dev),
           "zeros": torch.empty((m, n // g), dtype=torch.float32, device=dev),
           "channel_scale": torch.empty(n, dtype=torch.float32, device=dev),
           "w_hat": torch.empty((m, n), dtype=torch.float32, device=dev) if want_w_hat else None}
    ws = torch.empty(int(lib().gptq_awq_workspace_bytes(n)), dtype=torch.uint8, device=dev)
    n_tok, ld = (0, n) if X is None else (X.shape[0], X.stride(0))
    qp = QParams(int(bits), int(group_size), int(bool(sym)))
    _check(lib().gptq_awq_quantize(_ptr(X), n_tok, ld, _ptr(W), m, n, float(s_protect), qp, _ptr(out["codes"]),
                                   _ptr(out["scales"]), _ptr(out["zeros"]), _ptr(out["channel_scale"]),
                                   _ptr(out["w_hat"]), _ptr(ws), ws.numel(), dev.index,
                                   ctypes.c_void_p(stream.cuda_stream)), "gptq_awq_quantize")
    return out


def rtn_quantize(W: torch.Tensor, bits: int = 8, group_size: int = -1, sym: bool = True, clip_ratio: float = 1.0,
                 channel_scale: torch.Tensor | None = None, want_w_hat: bool = True,
                 stream: torch.cuda.Stream | None = None) -> dict:
    """Round-to-nearest with a clipped range (gptq_rtn_quantize; the page's INT8 LinearQuantizer
    is bits 8, per-channel, symmetric, clip_ratio 0.99).  W: fp16 [m, n]; channel_scale: fp32 [n]
    or None.  Returns device tensors codes, scales, zeros and (optionally) w_hat, in original
    column order."""
    m, n = W.shape
    dev = W.device
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    g = n if group_size == -1 else group_size
    out = {"codes": torch.empty((m, n * bits // 32), dtype=torch.int32, device=dev),
           "scales": torch.empty((m, n // g), dtype=torch.float32, device=dev),
           "zeros": torch.empty((m, n // g), dtype=torch.float32, device=dev),
           "w_hat": torch.empty((m, n), dtype=torch.float32, device=dev) if want_w_hat else None}
    qp = QParams(int(bits), int(group_size), int(bool(sym)))
    _check(lib().gptq_rtn_quantize(_ptr(W), m, n, qp, float(clip_ratio), _ptr(channel_scale), _ptr(out["codes"]),
                                   _ptr(out["scales"]), _ptr(out["zeros"]), _ptr(out["w_hat"]), dev.index,
                                   ctypes.c_void_p(stream.cuda_stream)), "gptq_rtn_quantize")
    return out


def activation_convert(Y: torch.Tensor, act: int = 1, want_bf16: bool = True, want_fp16: bool = True,
                       stream: torch.cuda.Stream | None = None):
    """x = act(y) (0 identity, 1 ReLU) of an fp32 or bf16 device tensor, as bf16 and fp16 copies
    (gptq_activation_convert)."""
    if Y.dtype not in (torch.float32, torch.bfloat16) or not Y.is_contiguous():
        raise ValueError("Y must be a contiguous fp32 or bf16 device tensor")
    dev = Y.device
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    xb = torch.empty(Y.shape, dtype=torch.bfloat16, device=dev) if want_bf16 else None
    xh = torch.empty(Y.shape, dtype=torch.float16, device=dev) if want_fp16 else None
    _check(lib().gptq_activation_convert(_ptr(Y), int(Y.dtype == torch.bfloat16), Y.numel(), int(act), _ptr(xb),
                                         _ptr(xh), dev.index, ctypes.c_void_p(stream.cuda_stream)),
           "gptq_activation_convert")
    return xb, xh


def _sequential_context(contexts: dict | None, n: int, m: int, dev: torch.device,
                        stream: torch.cuda.Stream) -> "GPTQContext":
    """A context of width n for at least m rows on this stream: kept in `contexts` when given."""
    if contexts is None:
        return GPTQContext(n, m, dev.index, stream)
    key = (n, dev.index, stream.cuda_stream)
    ctx = contexts.get(key)
    if ctx is not None and ctx.m_max < m:
        ctx.close()
        ctx = None
    if ctx is None:
        ctx = GPTQContext(n, m, dev.index, stream)
        contexts[key] = ctx
    return ctx


def close_contexts(contexts: dict) -> None:
    """Close the contexts that quantize_sequential kept in `contexts`."""
    for ctx in contexts.values():
        ctx.close()
    contexts.clear()


def quantize_sequential(X0: torch.Tensor, layers: list, act: int = 1, stream: torch.cuda.Stream | None = None,
                        keep_hessian: bool = False, contexts: dict | None = None) -> list:
    """Sequential quantization of a stack of linear layers ("GPTQ算法原理深度解析" §2.1: the error
    of a layer reaches the next one through its input).  X0: bf16 [N, n0] calibration inputs of
    layer 0; layers: dicts with W (fp16 [m_l, n_l], n_{l+1} = m_l), bits, group_size, sym, damp,
    desc_act.  Layer l is calibrated on X_l; X_{l+1} = act(X_l W16_l^T), the product taken with
    layer l's quantized weights (gptq_dequant_matmul on the fp16 copy of X_l).  Every step runs in
    the library's kernels; this function only sequences the calls.  Returns, per layer, its
    outputs (codes, scales, zeros, g_idx, perm), its calibration inputs X (bf16) and X16 (the
    fp16 copy its product reads), and with keep_hessian its H (fp32 [n, n]).  contexts: an optional
    dict in which the contexts (one per layer width and stream) stay between calls, so that repeated
    calls skip their creation (workspace allocation, the factorization's graph); the caller closes
    them with close_contexts.  Without it, each layer's context is created and closed here."""
    dev = X0.device
    stream = stream if stream is not None else torch.cuda.current_stream(dev)
    xb = X0
    _, xh = activation_convert(X0, act=0, want_bf16=False, stream=stream)
    res = []
    for li, L in enumerate(layers):
        W = L["W"]
        m, n = W.shape
        if xb.shape[1] != n:
            raise ValueError(f"layer {li}: {n} inputs, but the previous layer gives {xb.shape[1]}")
        ctx = _sequential_context(contexts, n, m, dev, stream)
        try:
            ctx.reset()
            ctx.accumulate_hessian(xb)
            H = ctx.get_hessian()[0] if keep_hessian else None
            perm = ctx.prepare(L["damp"], L["desc_act"])
            out = ctx.quantize_layer(W, L["bits"], L["group_size"], L["sym"], want_w_hat=False)
            ctx.synchronize()
        finally:
            if contexts is None:
                ctx.close()
        out = dict(out, perm=perm, X=xb, X16=xh, H=H)
        res.append(out)
        if li + 1 < len(layers):
            Y = dequant_matmul(xh, out["codes"], out["scales"], out["zeros"], perm, L["bits"], L["group_size"],
                               stream=stream)
            xb, xh = activation_convert(Y, act=act, stream=stream)
    return res
